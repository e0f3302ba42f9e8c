"""Float64 CPU oracle for paged FP8-KV MLA decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
reference leg use it.  It shares no code with the CUDA path.

What it computes, step by step, in the order the pages lay out the data:

1. Page-table gather ("generic_get_paged_cache_with_scales", Args: blocks,
   cache_lengths, lookup_table, scales, scales_lookup_table).  Logical token t
   of request b lives in physical block lookup_table[b, t // page_size], slot
   t % page_size, of the 6-D blocks tensor at [blk, 0, layer_idx, slot, 0, :].
   Its scale lives at the same slot of the 6-D scales tensor, in block
   scales_lookup_table[b, t // page_size] when that table is given, else in
   the value block id (the page says the shared id is right only while both
   pools share one id space).  kv_dim index 0 is the latent ("k cache").
2. Per-token dequantisation ("KVCacheScalesMHAOperand", description: MLA k_s
   per-token scales, quantization_granularity = head_size):
   K[t, d] = bf16_rn( f32_rn( e4m3(code[t, d]) * scale[t] ) ).
   The e4m3 value is decoded from its bit fields (OCP FP8 E4M3: bias 7, no
   infinities, S.1111.111 = NaN, subnormals m * 2^-9).
3. Attention (the textbook definition; the pages give no formula):
   x[t] = f32(softmax_scale) * sum_d q[d] K[t, d]   over keys t the query sees,
   lse = log(sum_t exp(x[t]))  (natural log),  w[t] = exp(x[t] - lse),
   out[v] = sum_t w[t] V[t, v]   with V[t, :] = K[t, :512].
   Keys per request: n_b = cache_lengths[b] + max_prompt_length (the step's
   new tokens are already in the cache); query i of request b sees keys
   t <= cache_lengths[b] + i (causal among the new tokens).

4. The KV-store step that produces this path's input (the per-token FP8
   recipe that also generates the test workloads: scale f32(amax) / 448, e4m3
   codes with round-to-nearest and saturation).  For new token i of request b, at
   position t = cache_lengths[b] + i (reading R1), with x the 576 bf16 values:
   scale = f32(max_d |x_d|) / 448 rounded to fp32 (1.0 for an all-zero row),
   code_d = e4m3_rn_sat(f32_rn(x_d / scale)), written to blocks[blk, 0,
   layer_idx, t % page_size, 0, :] and scale to the same slot of scales, with
   blk (and the scale block) from the page tables as in step 1.

5. The scale-folding variant (per-token scales): the same gather and attention, with the
   key and value elements left as the exact e4m3 values and the per-token scale applied to
   score column t and to weight column t instead (attend_scale_folded).  Exactly, this is
   attention over the unrounded products e4m3 * s_t; it differs from step 2's rounded keys by
   the fp32 and bf16 roundings of the dequant (reading R18).

6. The FP8 P.V variant (per-token scales): scores and softmax as in steps 1-3, and the value
   product taken with the exact e4m3 values and the scale folded into the weights, each weight
   split into two e4m3 terms (attend_fp8_pv, reading R21).

Everything after the e4m3 decode is float64 (the dequantised bf16 values are
exact in float64).  Points the pages leave open and the reading taken here:
cache_lengths count only tokens cached before this step (R1); query i sees
keys t <= L_b + i (R2); the dequant rounds twice, product to fp32 then to
bf16, both to nearest even, no flush to zero (R3); e4m3 is the OCP "fn"
encoding (R4); lse is the natural log (R5); the scales tensor is the 6-D one
and the page's 4-D shape is its (kv_dim 0, layer) slice (R7); kv_dim index 0
is read (R8); slots past n_b and unused table entries are never read (R9).
"""
from __future__ import annotations

import numpy as np

HEAD_DIM = 576
V_DIM = 512
INVALID_PAGE = 0xFFFFFFFF


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 byte (OCP E4M3, 'fn' flavour) as float64.

    sign s = bit 7, exponent field e = bits 6..3 (bias 7), mantissa m = bits 2..0.
    e == 0: subnormal (-1)^s * 2^-6 * m/8;  e == 15 and m == 7: NaN;
    otherwise (-1)^s * 2^(e-7) * (1 + m/8).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    sign = np.where(s == 1, -1.0, 1.0)
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return v.astype(np.float64)


def f32_bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32).view(np.uint32)


def bf16_round_f32(x) -> np.ndarray:
    """Round float32 values to bfloat16 with round-to-nearest-even; returns float64.

    Works on the bit pattern: add 0x7FFF plus the lowest kept bit, then drop the
    low 16 bits.  NaN stays NaN; overflow past the largest bf16 becomes inf, as
    in IEEE rounding.
    """
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    with np.errstate(invalid="ignore"):
        out = (r.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.where(np.isnan(f), np.nan, out)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """float64 value of bf16 numbers given as uint16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def dequant_rows(codes, scale) -> np.ndarray:
    """bf16_rn(f32_rn(e4m3(code) * scale)) for a [n, d] code block and [n] or [n, g] scales.

    The product of an e4m3 value (4 significant bits) and an fp32 scale (24
    bits) is exact in float64, so rounding it to float32 here is the single
    fp32 rounding of the product; the second rounding is to bf16 (reading R3).
    With g > 1 scales per row, dim d uses scale d // (d_total // g).
    """
    v = e4m3_decode(codes)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    if s.ndim == v.ndim - 1:
        s = s[..., None]
    if s.shape[-1] != 1 and s.shape[-1] != v.shape[-1]:
        g = s.shape[-1]
        s = np.repeat(s, v.shape[-1] // g, axis=-1)
    prod = v * s
    with np.errstate(over="ignore", invalid="ignore"):
        p32 = prod.astype(np.float32)
    return bf16_round_f32(p32)


def e4m3_encode_rn_sat(y) -> np.ndarray:
    """e4m3 byte nearest to each finite float32 value y, ties to even mantissa, saturated to +-448.

    Written from the format: |y| is clamped to 448, then for |y| >= 2^-6 (normal range) the
    exponent is e = floor(log2 |y|) and the mantissa steps are 2^(e-3); below 2^-6 the steps are
    the subnormal 2^-9.  A mantissa that rounds up to 8 carries into the exponent.  The sign bit is
    kept (so -0.0 -> 0x80).  Scaling by powers of two is exact in float64, so the rounding here is
    the single round-to-nearest-even of the format.
    """
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    sign = (np.signbit(y)).astype(np.int64)
    a = np.minimum(np.abs(y), 448.0)
    code = np.zeros(a.shape, dtype=np.int64)
    normal = a >= 2.0 ** -6
    # subnormal range: value = m * 2^-9, m in 0..8 (8 carries into the smallest normal)
    m_sub = np.rint(a * 2.0 ** 9).astype(np.int64)            # rint: round half to even
    code = np.where(~normal, m_sub, code)                     # m_sub == 8 -> 0x08 = 2^-6, correct
    # normal range
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(normal, a, 1.0))).astype(np.int64)
    # guard against log2 rounding at exact powers of two
    e = np.where(np.ldexp(1.0, e) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, e + 1) <= a, e + 1, e)
    m = np.rint((a / np.ldexp(1.0, e) - 1.0) * 8.0).astype(np.int64)
    carry = m == 8
    e = np.where(carry, e + 1, e)
    m = np.where(carry, 0, m)
    code_n = ((e + 7) << 3) | m
    code = np.where(normal, code_n, code)
    return ((sign << 7) | code).astype(np.uint8)


def quantize_token(x_bf16_bits):
    """(codes [576] uint8, scale float32) of one token's latent given as bf16 bit patterns."""
    x = bf16_bits_to_f64(x_bf16_bits).astype(np.float32)       # exact
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    scale = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    y = (x / scale).astype(np.float32)                         # IEEE fp32 division, RN
    return e4m3_encode_rn_sat(y), scale


def kv_store(latent_bits, cache_lengths, lookup_table, scales_lookup_table, layer_idx, blocks, scales):
    """Write the new tokens' codes and scales into copies of blocks / scales; returns the copies.

    latent_bits: bf16 bit patterns [B, T, 576]; token i of request b goes to position
    cache_lengths[b] + i.  Only kv_dim 0 and scale column 0 are written.
    """
    lat = np.asarray(latent_bits, dtype=np.uint16)
    B, T, _ = lat.shape
    blocks = np.array(blocks, copy=True)
    scales = np.array(scales, copy=True)
    L = np.asarray(cache_lengths, dtype=np.int64)
    lut = np.asarray(lookup_table, dtype=np.uint32)
    slut = None if scales_lookup_table is None else np.asarray(scales_lookup_table, dtype=np.uint32)
    P = blocks.shape[3]
    for b in range(B):
        for i in range(T):
            t = int(L[b]) + i
            page, slot = t // P, t % P
            blk = int(lut[b, page])
            sblk = int(slut[b, page]) if slut is not None else blk
            codes, sc = quantize_token(lat[b, i])
            blocks[blk, 0, layer_idx, slot, 0, :] = codes
            scales[sblk, 0, layer_idx, slot, 0, 0] = sc
    return blocks, scales


# ----------------------------------------------------------------------------
# page-table gather
# ----------------------------------------------------------------------------
def num_keys(cache_lengths, max_prompt_length) -> np.ndarray:
    """Keys stored for each request this step: n_b = L_b + T (reading R1)."""
    return np.asarray(cache_lengths, dtype=np.int64) + int(max_prompt_length)


def gather_request(blocks, scales, lookup_table, scales_lookup_table, b, n, layer_idx):
    """Codes [n, D] and scales [n, g] of the first n logical tokens of request b."""
    blocks = np.asarray(blocks)
    scales = np.asarray(scales)
    P = blocks.shape[3]
    lut = np.asarray(lookup_table).astype(np.int64) & 0xFFFFFFFF
    slut = None if scales_lookup_table is None else (np.asarray(scales_lookup_table).astype(np.int64) & 0xFFFFFFFF)
    t = np.arange(n, dtype=np.int64)
    page = t // P
    slot = t % P
    blk = lut[b, page]
    sblk = blk if slut is None else slut[b, page]
    if n and (blk.max() >= blocks.shape[0] or sblk.max() >= scales.shape[0]):
        raise IndexError("page id outside the block pool")
    codes = blocks[blk, 0, layer_idx, slot, 0, :]
    sc = scales[sblk, 0, layer_idx, slot, 0, :]
    return codes, sc


def dequant_request(blocks, scales, lookup_table, scales_lookup_table, b, n, layer_idx):
    codes, sc = gather_request(blocks, scales, lookup_table, scales_lookup_table, b, n, layer_idx)
    return dequant_rows(codes, sc)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def attend(q, K, softmax_scale, return_weights=False):
    """Softmax attention of queries q [H, D] over keys K [n, D], V = K[:, :512].

    Returns out [H, 512] and natural-log lse [H] (and weights [H, n]).
    """
    q = np.asarray(q, dtype=np.float64)
    s = float(np.float32(softmax_scale))
    x = s * (q @ K.T)                                  # [H, n]
    mx = x.max(axis=1, keepdims=True)
    e = np.exp(x - mx)
    tot = e.sum(axis=1, keepdims=True)
    lse = (mx + np.log(tot))[:, 0]
    w = np.exp(x - lse[:, None])
    out = w @ K[:, :V_DIM]
    if return_weights:
        return out, lse, w
    return out, lse


def decode(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table,
           max_prompt_length, layer_idx, softmax_scale, requests=None, heads=None,
           return_weights=False):
    """Full decode: out [B, T, H, 512] float64, lse [B, T, H] float64.

    `requests` / `heads` restrict the work to a subset (rows not computed are NaN).
    q: [B, T, H, 576] float values (bf16-exact), or uint16 bf16 bit patterns.
    """
    q = np.asarray(q)
    if q.dtype == np.uint16:
        q = bf16_bits_to_f64(q)
    q = q.astype(np.float64)
    B, T, H, D = q.shape
    assert D == HEAD_DIM
    T = int(max_prompt_length)
    L = np.asarray(cache_lengths).astype(np.int64) & 0xFFFFFFFF
    n_all = num_keys(L, T)
    out = np.full((B, T, H, V_DIM), np.nan)
    lse = np.full((B, T, H), np.nan)
    weights = {}
    reqs = range(B) if requests is None else requests
    hs = np.arange(H) if heads is None else np.asarray(heads)
    for b in reqs:
        K = dequant_request(blocks, scales, lookup_table, scales_lookup_table, b, int(n_all[b]), layer_idx)
        for i in range(T):
            vis = int(L[b]) + i + 1                    # query i sees keys t <= L_b + i (R2)
            r = attend(q[b, i, hs], K[:vis], softmax_scale, return_weights)
            out[b, i, hs] = r[0]
            lse[b, i, hs] = r[1]
            if return_weights:
                weights[(b, i)] = r[2]
    if return_weights:
        return out, lse, weights
    return out, lse


# ----------------------------------------------------------------------------
# scale-folding variant (per-token scales only)
# ----------------------------------------------------------------------------
def attend_scale_folded(q, codes, scale, softmax_scale):
    """Attention with the per-token scale folded out of the keys and values.

    The key and value elements stay the exact e4m3 values C[t, d]; the scale s_t multiplies
    column t of the scores and column t of the softmax weights instead:
      x[t] = f32(softmax_scale) * s_t * sum_d q[d] C[t, d],
      lse = log sum_t exp(x[t]),  w[t] = exp(x[t] - lse),
      out[v] = sum_t (w[t] s_t) C[t, v]   (v < 512).
    In exact arithmetic this is attention over the unrounded keys K[t, d] = s_t C[t, d] (no fp32
    or bf16 rounding of the dequantised values), which the tests check.
    """
    q = np.asarray(q, dtype=np.float64)
    C = e4m3_decode(codes)                             # [n, 576], exact
    s = np.asarray(scale, dtype=np.float32).astype(np.float64).reshape(-1)
    ss = float(np.float32(softmax_scale))
    x = ss * (q @ C.T) * s[None, :]                    # score columns scaled by s_t
    mx = x.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.exp(x - mx).sum(axis=1, keepdims=True)))[:, 0]
    w = np.exp(x - lse[:, None])
    out = (w * s[None, :]) @ C[:, :V_DIM]              # weight columns scaled by s_t
    return out, lse


def decode_scale_folded(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table,
                        max_prompt_length, layer_idx, softmax_scale, requests=None, heads=None):
    """decode() with the scale-folding variant's arithmetic (one fp32 scale per token).

    Same gather and visibility rules as decode(); rows not computed are NaN.
    """
    q = np.asarray(q)
    if q.dtype == np.uint16:
        q = bf16_bits_to_f64(q)
    q = q.astype(np.float64)
    B, T, H, D = q.shape
    assert D == HEAD_DIM
    if np.asarray(scales).shape[-1] != 1:
        raise ValueError("the scale-folding variant takes one scale per token")
    T = int(max_prompt_length)
    L = np.asarray(cache_lengths).astype(np.int64) & 0xFFFFFFFF
    n_all = num_keys(L, T)
    out = np.full((B, T, H, V_DIM), np.nan)
    lse = np.full((B, T, H), np.nan)
    reqs = range(B) if requests is None else requests
    hs = np.arange(H) if heads is None else np.asarray(heads)
    for b in reqs:
        codes, sc = gather_request(blocks, scales, lookup_table, scales_lookup_table, b, int(n_all[b]), layer_idx)
        for i in range(T):
            vis = int(L[b]) + i + 1
            r = attend_scale_folded(q[b, i, hs], codes[:vis], sc[:vis, 0], softmax_scale)
            out[b, i, hs] = r[0]
            lse[b, i, hs] = r[1]
    return out, lse


# ----------------------------------------------------------------------------
# FP8 P.V variant (per-token scales only)
# ----------------------------------------------------------------------------
E4M3_MAX = 448.0
FP8_PV_HEADROOM = 112.0


def fp8_pv_sigma(s_max):
    """Power-of-two exponent of the folded weights: the largest integer sigma with
    s_max * 2^sigma <= 112 = 448 / 4.  Every weight p * s * 2^sigma then stays at or below 448
    for p <= 4, which leaves an implementation room for a running maximum that trails the true
    one by up to 2 (log2 units); here p <= 1, so the largest weight lies in (56, 112] and the
    weights fill the top of the e4m3 range (the normal range, 4 significant bits, reaches down to
    2^-6, i.e. 2^-13 of the largest weight)."""
    return int(np.floor(np.log2(FP8_PV_HEADROOM / float(s_max))))


def e4m3_split2(w):
    """Two-term e4m3 split of float32 values w (all >= 0): hi = e4m3_rn_sat(w), lo = e4m3_rn_sat(w - hi)
    (the residual is exact in float32).  Returns (hi, lo) as float64 values."""
    w = np.asarray(w, dtype=np.float32)
    hi = e4m3_decode(e4m3_encode_rn_sat(w))
    r = (w.astype(np.float64) - hi).astype(np.float32)       # exact: hi is w rounded to 4 significant bits
    lo = e4m3_decode(e4m3_encode_rn_sat(r))
    return hi, lo


def attend_fp8_pv(q, codes, scale, softmax_scale):
    """Attention whose P.V product is taken in e4m3 (the scope table's FP8-MMA variant, reading R21).

    Scores and softmax are the decode's (keys dequantised by R3); the value rows are the exact e4m3
    values C[t, :512] without their scale, and the scale moves into the weights:
      x[t] = f32(softmax_scale) * q . K[t],   p[t] = exp(x[t] - max x),   l = sum_t p[t],
      w[t] = f32(p[t] * s_t * 2^sigma)  with sigma = fp8_pv_sigma(max_t s_t),
      (hi[t], lo[t]) = e4m3_split2(w[t]),
      out[v] = 2^-sigma * sum_t (hi[t] + lo[t]) * C[t, v] / l,   lse = max x + ln l.
    hi + lo is w to within 2^-8 of w (normal range), so out is attention over V[t] = s_t C[t]
    (unrounded) up to that relative error of each weight.
    """
    q = np.asarray(q, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64).reshape(-1)
    K = dequant_rows(codes, s.astype(np.float32)[:, None])    # R3 dequant (bf16 values)
    C = e4m3_decode(codes)
    ss = float(np.float32(softmax_scale))
    x = ss * (q @ K.T)
    mx = x.max(axis=1, keepdims=True)
    p = np.exp(x - mx)
    l = p.sum(axis=1)
    sigma = fp8_pv_sigma(s.max())
    w = p * s[None, :] * 2.0 ** sigma
    hi, lo = e4m3_split2(w)
    out = ((hi + lo) @ C[:, :V_DIM]) * 2.0 ** (-sigma) / l[:, None]
    lse = mx[:, 0] + np.log(l)
    return out, lse


def decode_fp8_pv(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table,
                  max_prompt_length, layer_idx, softmax_scale, requests=None, heads=None):
    """decode() with the FP8 P.V variant's arithmetic (one fp32 scale per token).

    Same gather and visibility rules as decode(); rows not computed are NaN.
    """
    q = np.asarray(q)
    if q.dtype == np.uint16:
        q = bf16_bits_to_f64(q)
    q = q.astype(np.float64)
    B, T, H, D = q.shape
    assert D == HEAD_DIM
    if np.asarray(scales).shape[-1] != 1:
        raise ValueError("the FP8 P.V variant takes one scale per token")
    T = int(max_prompt_length)
    L = np.asarray(cache_lengths).astype(np.int64) & 0xFFFFFFFF
    n_all = num_keys(L, T)
    out = np.full((B, T, H, V_DIM), np.nan)
    lse = np.full((B, T, H), np.nan)
    reqs = range(B) if requests is None else requests
    hs = np.arange(H) if heads is None else np.asarray(heads)
    for b in reqs:
        codes, sc = gather_request(blocks, scales, lookup_table, scales_lookup_table, b, int(n_all[b]), layer_idx)
        for i in range(T):
            vis = int(L[b]) + i + 1
            r = attend_fp8_pv(q[b, i, hs], codes[:vis], sc[:vis, 0], softmax_scale)
            out[b, i, hs] = r[0]
            lse[b, i, hs] = r[1]
    return out, lse


# ----------------------------------------------------------------------------
# split-KV combine (used to pin that any split of the keys reaches the same result)
# ----------------------------------------------------------------------------
def attend_partial(q, K, softmax_scale, t0, t1):
    """Normalised partial result over keys [t0, t1): (out_s [H, 512], lse_s [H]); empty -> lse -inf."""
    if t1 <= t0:
        H = np.asarray(q).shape[0]
        return np.zeros((H, V_DIM)), np.full(H, -np.inf)
    return attend(q, K[t0:t1], softmax_scale)


def combine(parts):
    """LSE-weighted merge of partial results: lse = log sum_s e^{lse_s}, out = sum_s e^{lse_s - lse} out_s."""
    lses = np.stack([p[1] for p in parts])            # [S, H]
    outs = np.stack([p[0] for p in parts])            # [S, H, 512]
    mx = lses.max(axis=0)
    w = np.exp(lses - mx)
    tot = w.sum(axis=0)
    lse = mx + np.log(tot)
    out = (w[..., None] * outs).sum(axis=0) / tot[:, None]
    return out, lse

"""Pins for the float64 oracle: each check ties it to something other than itself.

Library routines (ml_dtypes, torch casts, torch SDPA), closed forms, invariants
the page layouts imply, brute force on tiny inputs, and hand-derived values.
The last tests plant plausible mistakes in the oracle and check that a pin
catches each one.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- formats
def test_e4m3_decode_matches_ml_dtypes_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    th = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for ref in (ml, th):
        assert np.array_equal(np.isnan(ours), np.isnan(ref))
        ok = ~np.isnan(ref)
        assert np.array_equal(ours[ok], ref[ok])
        assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e4m3_golden_hand_values():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            code, val = line.split()[:2]
            rows.append((int(code, 16), float(val)))
    assert len(rows) >= 12
    for code, val in rows:
        got = O.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def _tie_heavy_f32(n, rng):
    u = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    # force a share of exact ties (low 16 bits = 0x8000) and near-ties
    u[: n // 4] = (u[: n // 4] & 0xFFFF0000) | 0x8000
    u[n // 4: n // 2] = (u[n // 4: n // 2] & 0xFFFF0000) | 0x7FFF
    return u.view(np.float32)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    f = _tie_heavy_f32(1_000_000, rng)
    extra = np.array([0.0, -0.0, 1e-45, -1e-45, 1.1754942e-38, 3.4028235e38, -3.4028235e38,
                      np.inf, -np.inf, 65504.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8], dtype=np.float32)
    f = np.concatenate([f, extra])
    ours = O.bf16_round_f32(f)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def _scales_for_exhaustive(n, rng):
    s = np.concatenate([
        rng.uniform(1e-3, 2.0, n // 2).astype(np.float32),
        (2.0 ** rng.integers(-40, 20, n // 8)).astype(np.float32),
        rng.uniform(1e-30, 1e-28, n // 8).astype(np.float32),      # products near/below f32 normal range
        rng.uniform(1e30, 1e35, n // 8).astype(np.float32),        # products past bf16/f32 max
        np.frombuffer(rng.integers(0, 2**31, n // 8, dtype=np.uint32).tobytes(), dtype=np.float32),
    ])
    return s[np.isfinite(s) & (s > 0)]


def test_dequant_matches_torch_exhaustive_codes():
    """bf16(f32(e4m3 * scale)) against torch's own fp8 decode, fp32 multiply and bf16 cast."""
    rng = np.random.default_rng(2)
    scales = _scales_for_exhaustive(10_000, rng)
    codes = np.arange(256, dtype=np.uint8)
    C = np.broadcast_to(codes[None, :], (scales.size, 256))
    ours = O.dequant_rows(C, scales)
    tc = torch.from_numpy(np.ascontiguousarray(C)).view(torch.float8_e4m3fn).to(torch.float32)
    ts = torch.from_numpy(scales.copy())[:, None]
    ref = (tc * ts).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def test_dequant_power_of_two_scale_is_exact_scaling():
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes)
    for k in (-12, -3, 0, 5):
        d = O.dequant_rows(codes[None], np.array([2.0 ** k], dtype=np.float32))[0]
        ok = ~np.isnan(v)
        assert np.array_equal(d[ok], v[ok] * 2.0 ** k)


# --------------------------------------------------------------------------- gather
def _tiny_paged(n_tokens, P, NB, layers, layer_idx, rng, kv_dim=1, separate=False):
    codes = rng.integers(0, 256, size=(n_tokens, O.HEAD_DIM), dtype=np.uint8)
    codes[codes == 0x7F] = 0x7E
    codes[codes == 0xFF] = 0xFE
    sc = rng.uniform(0.01, 0.1, size=n_tokens).astype(np.float32)
    pages = (n_tokens + P - 1) // P
    perm = rng.permutation(NB)[:pages]
    blocks = np.full((NB, kv_dim, layers, P, 1, O.HEAD_DIM), 0x7F, dtype=np.uint8)
    NSB = NB + 3 if separate else NB
    scales = np.full((NSB, kv_dim, layers, P, 1, 1), np.nan, dtype=np.float32)
    sperm = rng.permutation(NSB)[:pages] if separate else perm
    for t in range(n_tokens):
        blocks[perm[t // P], 0, layer_idx, t % P, 0, :] = codes[t]
        scales[sperm[t // P], 0, layer_idx, t % P, 0, 0] = sc[t]
    lut = np.full((1, pages + 2), O.INVALID_PAGE, dtype=np.int64)
    lut[0, :pages] = perm
    slut = None
    if separate:
        slut = np.full((1, pages + 2), O.INVALID_PAGE, dtype=np.int64)
        slut[0, :pages] = sperm
    return codes, sc, blocks, scales, lut, slut


@pytest.mark.parametrize("P,separate,layers,layer_idx,kv_dim", [
    (16, False, 1, 0, 1), (64, False, 3, 2, 1), (16, True, 2, 1, 2), (48, True, 1, 0, 1)])
def test_gather_equals_direct_contiguous(P, separate, layers, layer_idx, kv_dim):
    """Brute force: paging through permuted blocks equals reading the rows directly."""
    rng = np.random.default_rng(3)
    n = 150
    codes, sc, blocks, scales, lut, slut = _tiny_paged(n, P, 20, layers, layer_idx, rng, kv_dim, separate)
    got = O.dequant_request(blocks, scales, lut, slut, 0, n, layer_idx)
    direct = O.dequant_rows(codes, sc)
    assert np.array_equal(got, direct)
    assert np.isfinite(got).all()


def test_page_permutation_invariance_oracle():
    inp = W.make_inputs(W.CONFIGS[0])
    out1, lse1 = oracle_decode(inp)
    out2, lse2 = oracle_decode(W.permute_pages(inp, seed=5))
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_scale_id_space_invariance_oracle():
    inp = W.make_inputs(W.CONFIGS[0])
    out1, lse1 = oracle_decode(inp)
    sep = W.separate_scale_space(inp, extra=9, seed=4)
    out2, lse2 = oracle_decode(sep)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)
    # and separated + permuted
    out3, lse3 = oracle_decode(W.permute_pages(sep, seed=8))
    assert np.array_equal(out1, out3) and np.array_equal(lse1, lse3)


def poison_unread(inp):
    """Copy of `inp` with every byte the decode must not read set to NaN / invalid ids."""
    a = to_numpy(inp)
    blocks = np.full_like(a["blocks"], 0x7F)
    scales = np.full_like(a["scales"], np.nan)
    P = blocks.shape[3]
    lut = a["lookup_table"].copy()
    slut = None if a["scales_lookup_table"] is None else a["scales_lookup_table"].copy()
    n = O.num_keys(a["cache_lengths"], a["max_prompt_length"])
    li = a["layer_idx"]
    for b in range(lut.shape[0]):
        t = np.arange(n[b])
        blk = lut[b, t // P]
        sblk = blk if slut is None else slut[b, t // P]
        blocks[blk, 0, li, t % P] = a["blocks"][blk, 0, li, t % P]
        scales[sblk, 0, li, t % P] = a["scales"][sblk, 0, li, t % P]
        pages = (n[b] + P - 1) // P
        lut[b, pages:] = O.INVALID_PAGE
        if slut is not None:
            slut[b, pages:] = O.INVALID_PAGE
    a.update(blocks=blocks, scales=scales, lookup_table=lut, scales_lookup_table=slut)
    return a


@pytest.mark.parametrize("cfg_i", [0, 1])
def test_poisoned_unread_bytes_do_not_change_oracle(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i])
    req = [0, 1]
    out1, lse1 = oracle_decode(inp, requests=req)
    a = poison_unread(inp)
    out2, lse2 = O.decode(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                          a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"],
                          a["softmax_scale"], requests=req)
    assert np.array_equal(out1[req], out2[req]) and np.isfinite(out2[req]).all()
    assert np.array_equal(lse1[req], lse2[req])


# --------------------------------------------------------------------------- attention
def _sdpa(q, K, scale, mask=None):
    tq = torch.from_numpy(q)[None, None]                  # [1,1,H,D]
    tk = torch.from_numpy(K)[None, None]
    tv = torch.from_numpy(np.ascontiguousarray(K[:, :O.V_DIM]))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    return o[0, 0].numpy()


def test_attend_matches_torch_sdpa_float64():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((8, O.HEAD_DIM))
    K = rng.standard_normal((37, O.HEAD_DIM))
    s = float(np.float32(W.SOFTMAX_SCALE))
    out, lse = O.attend(q, K, W.SOFTMAX_SCALE)
    ref = _sdpa(q, K, s)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    lref = torch.logsumexp(torch.from_numpy(s * (q @ K.T)), dim=1).numpy()
    assert np.allclose(lse, lref, rtol=0, atol=1e-12)


def test_decode_matches_sdpa_with_causal_mask_t2():
    cfg = W.DecodeConfig("t2", batch=2, q_len=2, num_q_heads=4, page_size=16, num_layers=1,
                         layer_idx=0, length_kind="list", length_args=(5, 20), pool_kind="fixed",
                         num_blocks=6, seed=77)
    inp = W.make_inputs(cfg)
    a = to_numpy(inp)
    out, lse = oracle_decode(inp)
    q = O.bf16_bits_to_f64(a["q"])
    s = float(np.float32(inp.softmax_scale))
    for b in range(2):
        n = int(a["cache_lengths"][b]) + 2
        K = O.dequant_request(a["blocks"], a["scales"], a["lookup_table"], None, b, n, 0)
        qb = q[b]                                             # [T, H, D]
        tq = torch.from_numpy(qb.transpose(1, 0, 2))[None]   # [1, H, T, D]
        tk = torch.from_numpy(K)[None, None]
        tv = torch.from_numpy(np.ascontiguousarray(K[:, :512]))[None, None]
        L = int(a["cache_lengths"][b])
        mask = torch.from_numpy(np.arange(n)[None, :] <= (L + np.arange(2))[:, None])
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=s)
        assert np.allclose(out[b], ref[0].numpy().transpose(1, 0, 2), rtol=1e-12, atol=1e-12)


def test_weights_sum_to_one():
    inp = W.make_inputs(W.CONFIGS[0])
    _, _, w = oracle_decode(inp, return_weights=True)
    for key, wb in w.items():
        assert np.allclose(wb.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert (wb >= 0).all()


def test_closed_form_q_zero_mean_of_v():
    inp = W.make_inputs(W.CONFIGS[0], q_zero=True)
    out, lse = oracle_decode(inp)
    a = to_numpy(inp)
    for b in range(2):
        n = int(a["cache_lengths"][b]) + 1
        K = O.dequant_request(a["blocks"], a["scales"], a["lookup_table"], None, b, n, 0)
        assert np.allclose(out[b, 0], K[:, :512].mean(axis=0)[None], rtol=1e-12, atol=1e-13)
        assert np.allclose(lse[b, 0], math.log(n), rtol=0, atol=1e-12)


def test_closed_form_equal_scores():
    """q_nope = 0 and identical rope rows on every key: scores are equal, out = mean V."""
    rng = np.random.default_rng(5)
    n, P = 40, 16
    codes = rng.integers(0, 0x70, size=(n, O.HEAD_DIM), dtype=np.uint8)
    codes[:, 512:] = codes[0, 512:]
    sc = np.ones(n, dtype=np.float32)
    pages = (n + P - 1) // P
    blocks = np.zeros((pages, 1, 1, P, 1, O.HEAD_DIM), dtype=np.uint8)
    scales = np.ones((pages, 1, 1, P, 1, 1), dtype=np.float32)
    for t in range(n):
        blocks[t // P, 0, 0, t % P, 0] = codes[t]
        scales[t // P, 0, 0, t % P, 0, 0] = sc[t]
    lut = np.arange(pages)[None]
    q = np.zeros((1, 1, 3, O.HEAD_DIM))
    q[..., 512:] = O.bf16_round_f32(rng.standard_normal((1, 1, 3, 64)).astype(np.float32))
    out, lse = O.decode(q, blocks, scales, np.array([n - 1]), lut, None, 1, 0, W.SOFTMAX_SCALE)
    K = O.dequant_rows(codes, sc)
    x = float(np.float32(W.SOFTMAX_SCALE)) * (q[0, 0] @ K[0])
    assert np.allclose(out[0, 0], K[:, :512].mean(axis=0)[None], rtol=1e-12, atol=1e-13)
    assert np.allclose(lse[0, 0], x + math.log(n), rtol=0, atol=1e-12)


def test_single_key_returns_v0():
    cfg = W.DecodeConfig("one", batch=1, q_len=1, num_q_heads=4, page_size=16, num_layers=1,
                         layer_idx=0, length_kind="list", length_args=(0,), pool_kind="fixed",
                         num_blocks=2, seed=9)
    inp = W.make_inputs(cfg)
    out, lse = oracle_decode(inp)
    a = to_numpy(inp)
    K = O.dequant_request(a["blocks"], a["scales"], a["lookup_table"], None, 0, 1, 0)
    q = O.bf16_bits_to_f64(a["q"])[0, 0]
    assert np.array_equal(out[0, 0], np.broadcast_to(K[0, :512], (4, 512)))
    assert np.allclose(lse[0, 0], float(np.float32(W.SOFTMAX_SCALE)) * (q @ K[0]), rtol=0, atol=1e-12)


def test_t2_query0_equals_t1_run():
    cfg2 = W.DecodeConfig("t2", batch=2, q_len=2, num_q_heads=8, page_size=16, num_layers=1,
                          layer_idx=0, length_kind="list", length_args=(9, 33), pool_kind="fixed",
                          num_blocks=8, seed=21)
    inp = W.make_inputs(cfg2)
    a = to_numpy(inp)
    out2, lse2 = oracle_decode(inp)
    # the same cache read as a q_len = 1 step: query 0's visible keys are the first L+1
    q1 = a["q"][:, :1]
    out1, lse1 = O.decode(q1, a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"], None,
                          1, 0, inp.softmax_scale)
    assert np.array_equal(out1[:, 0], out2[:, 0]) and np.array_equal(lse1[:, 0], lse2[:, 0])
    # query 1 equals a q_len = 1 step whose cache holds one more token
    out1b, lse1b = O.decode(a["q"][:, 1:], a["blocks"], a["scales"], a["cache_lengths"] + 1,
                            a["lookup_table"], None, 1, 0, inp.softmax_scale)
    assert np.array_equal(out1b[:, 0], out2[:, 1]) and np.array_equal(lse1b[:, 0], lse2[:, 1])


def test_split_combine_equals_unsplit():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((16, O.HEAD_DIM))
    K = rng.standard_normal((300, O.HEAD_DIM)) * 3
    full = O.attend(q, K, W.SOFTMAX_SCALE)
    for cuts in ([0, 300], [0, 150, 300], [0, 1, 2, 299, 300], [0, 64, 64, 128, 192, 300],
                 sorted([0, 300] + list(rng.integers(0, 300, 9)))):
        parts = [O.attend_partial(q, K, W.SOFTMAX_SCALE, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
        out, lse = O.combine(parts)
        assert np.allclose(out, full[0], rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, full[1], rtol=0, atol=1e-12)


def test_oracle_config1_sampled_is_finite_and_bounded():
    inp = W.make_inputs(W.CONFIGS[1])
    out, lse = oracle_decode(inp, requests=[0, 31], heads=[0, 127])
    v = out[[0, 31]][:, :, [0, 127]]
    assert np.isfinite(v).all()
    # a convex combination of V rows lies inside their range
    a = to_numpy(inp)
    for b in (0, 31):
        n = int(a["cache_lengths"][b]) + 1
        K = O.dequant_request(a["blocks"], a["scales"], a["lookup_table"], None, b, n, 1)
        assert (out[b, 0, [0, 127]] <= K[:, :512].max(axis=0) + 1e-12).all()
        assert (out[b, 0, [0, 127]] >= K[:, :512].min(axis=0) - 1e-12).all()


# --------------------------------------------------------------------------- planted mistakes
def _dequant_single_rounding(codes, scale):
    v = O.e4m3_decode(codes)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    if s.ndim == v.ndim - 1:
        s = s[..., None]
    # mistake: one rounding of the exact product straight to bf16 (no fp32 step)
    prod = v * s
    mant, ex = np.frexp(prod)
    return np.ldexp(np.round(mant * 256) / 256, ex)


def test_planted_single_rounding_is_caught(monkeypatch):
    monkeypatch.setattr(O, "dequant_rows", _dequant_single_rounding)
    with pytest.raises(AssertionError):
        test_dequant_matches_torch_exhaustive_codes()


def test_planted_causal_off_by_one_is_caught(monkeypatch):
    real = O.attend

    def decode_wrong(q, blocks, scales, cache_lengths, lookup_table, slut, T, li, ss, **kw):
        # mistake: query i sees keys t < L_b + i (one key short)
        q = O.bf16_bits_to_f64(q) if np.asarray(q).dtype == np.uint16 else np.asarray(q, dtype=np.float64)
        B, T_, H, _ = q.shape
        out = np.zeros((B, T_, H, 512))
        lse = np.zeros((B, T_, H))
        for b in range(B):
            n = int(cache_lengths[b]) + T
            K = O.dequant_request(blocks, scales, lookup_table, slut, b, n, li)
            for i in range(T_):
                vis = max(1, int(cache_lengths[b]) + i)
                out[b, i], lse[b, i] = real(q[b, i], K[:vis], ss)
        return out, lse

    monkeypatch.setattr(O, "decode", decode_wrong)
    with pytest.raises(AssertionError):
        test_decode_matches_sdpa_with_causal_mask_t2()


def test_planted_scale_table_ignored_is_caught(monkeypatch):
    real = O.gather_request

    def gather_wrong(blocks, scales, lut, slut, b, n, li):
        return real(blocks, scales, lut, None, b, n, li)   # mistake: scales through lookup_table

    monkeypatch.setattr(O, "gather_request", gather_wrong)
    with pytest.raises((AssertionError, IndexError)):
        test_scale_id_space_invariance_oracle()


def test_planted_v_slice_is_caught(monkeypatch):
    def attend_wrong(q, K, softmax_scale, return_weights=False):
        q = np.asarray(q, dtype=np.float64)
        x = float(np.float32(softmax_scale)) * (q @ K.T)
        mx = x.max(axis=1, keepdims=True)
        lse = (mx + np.log(np.exp(x - mx).sum(axis=1, keepdims=True)))[:, 0]
        w = np.exp(x - lse[:, None])
        out = w @ K[:, 64:]                                  # mistake: V = last 512 dims
        return (out, lse, w) if return_weights else (out, lse)

    monkeypatch.setattr(O, "attend", attend_wrong)
    with pytest.raises(AssertionError):
        test_attend_matches_torch_sdpa_float64()

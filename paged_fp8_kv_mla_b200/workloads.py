"""Seeded synthetic inputs for paged FP8-KV MLA decode.

This module only *creates* inputs: it draws random numbers, builds page
tables and stores the KV latent as e4m3 bytes with one fp32 scale per token.
It holds none of the decode arithmetic (no dequantisation, no attention), so
the CUDA path and the float64 oracle can both read what it writes without
sharing any of the method's code.

Layouts follow the Modular page "generic_get_paged_cache_with_scales" (Args):
  blocks  [num_blocks, kv_dim, num_layers, page_size, num_heads, head_dim]  (e4m3 bytes)
  scales  [num_scale_blocks, kv_dim, num_layers, page_size, num_heads, head_dim_granularity] (fp32)
  cache_lengths [batch] uint32, lookup_table [batch, max_pages] uint32,
  optional scales_lookup_table [batch, max_pages] uint32 (own block-id space).
The per-token scale (quantization_granularity = head_size) is the layout the
page "KVCacheScalesMHAOperand" describes for MLA k_s.

Quantiser used to *build* the cache (data generation, not the decode path):
each token's 576-wide bf16 row x gets scale = f32(amax|x|) / 448 (1.0 for an
all-zero row) and codes = e4m3(clamp(x / scale, -448, 448)) with
round-to-nearest-even, done by torch's float8_e4m3fn cast.

Randomness comes from torch generators seeded with 1000 + config id.  The CPU
and CUDA generators produce different streams, so a (config, device) pair is
reproducible, not a config alone.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

HEAD_DIM = 576          # 512 latent + 64 rope
V_DIM = 512             # V = first 512 latent dims of each token
E4M3_MAX = 448.0
INVALID_PAGE = 0xFFFFFFFF
SOFTMAX_SCALE = float(torch.tensor(1.0 / math.sqrt(192.0), dtype=torch.float32).item())


@dataclass(frozen=True)
class DecodeConfig:
    """One decode workload: shapes, length recipe and page-pool recipe."""
    name: str
    batch: int
    q_len: int
    num_q_heads: int
    page_size: int
    num_layers: int
    layer_idx: int
    length_kind: str                 # "fixed" | "uniform" | "loguniform"
    length_args: tuple
    pool_kind: str = "permuted"      # "permuted" (pool = pool_factor * pages needed) | "exact"
    pool_factor: float = 1.0
    pool_extra: int = 0
    num_blocks: Optional[int] = None  # fixed pool size (the tiny two-request workload)
    separate_scales: bool = False     # scales paged through their own id space
    scales_pool_extra: int = 0
    outlier_rate: float = 0.0
    outlier_mult: float = 1.0
    kv_dim: int = 1
    seed: int = 1000
    softmax_scale: float = SOFTMAX_SCALE
    scale_blocks: int = 1             # scales per token (head_dim_granularity); each covers 576 / g dims

    @property
    def head_dim(self) -> int:
        return HEAD_DIM


CONFIGS = [
    # 0: tiny, the oracle finishes it in milliseconds
    DecodeConfig("tiny_b2_h16_p16", batch=2, q_len=1, num_q_heads=16, page_size=16,
                 num_layers=1, layer_idx=0, length_kind="list", length_args=(37, 64),
                 pool_kind="fixed", num_blocks=16, seed=1000),
    # 1: moderate batch, lengths uniform in [1024, 4096], pool 2x pages needed, layer 1 of 2
    DecodeConfig("moderate_b32_h128_l1k-4k", batch=32, q_len=1, num_q_heads=128, page_size=64,
                 num_layers=2, layer_idx=1, length_kind="uniform", length_args=(1024, 4096),
                 pool_kind="permuted", pool_factor=2.0, seed=1001),
    # 2: bandwidth-bound steady state, all lengths 8192, 1% outlier tokens x20
    DecodeConfig("steady_b128_h128_l8k", batch=128, q_len=1, num_q_heads=128, page_size=64,
                 num_layers=1, layer_idx=0, length_kind="fixed", length_args=(8192,),
                 pool_kind="permuted", pool_factor=1.0, outlier_rate=0.01, outlier_mult=20.0,
                 seed=1002),
    # 3: ragged speculative decode, q_len 2, log-uniform lengths, scales paged separately
    DecodeConfig("ragged_spec_b64_t2_h128", batch=64, q_len=2, num_q_heads=128, page_size=64,
                 num_layers=1, layer_idx=0, length_kind="loguniform", length_args=(1, 32768),
                 pool_kind="permuted", pool_factor=1.0, separate_scales=True, scales_pool_extra=37,
                 seed=1003),
    # 4: long context, split-KV across SMs
    DecodeConfig("long_b4_h128_l128k", batch=4, q_len=1, num_q_heads=128, page_size=128,
                 num_layers=1, layer_idx=0, length_kind="fixed", length_args=(131072,),
                 pool_kind="permuted", pool_factor=1.0, seed=1004),
]


def config_by_index(i: int) -> DecodeConfig:
    return CONFIGS[i]


@dataclass
class DecodeInputs:
    """Tensors of one decode call (all on one device) plus the host scalars."""
    cfg: DecodeConfig
    q: torch.Tensor                 # bf16 [B, T, H, 576]
    blocks: torch.Tensor            # uint8 [NB, kv_dim, L, P, 1, 576]
    scales: torch.Tensor            # fp32  [NSB, kv_dim, L, P, 1, 1]
    cache_lengths: torch.Tensor     # int32 view of uint32 [B]
    lookup_table: torch.Tensor      # int32 view of uint32 [B, max_pages]
    scales_lookup_table: Optional[torch.Tensor]
    max_prompt_length: int
    max_cache_length: int
    layer_idx: int
    softmax_scale: float
    extra: dict = field(default_factory=dict)

    @property
    def num_keys(self):
        """Keys stored per request: cached tokens plus this step's q_len tokens."""
        return self.cache_lengths.to(torch.int64) + self.max_prompt_length

    def kv_scale_bytes(self) -> int:
        """Algorithmic KV+scale bytes: each visible key's 576 e4m3 bytes + 4 B scale, read once."""
        return int(self.num_keys.sum().item()) * (HEAD_DIM + 4)

    def flops(self) -> int:
        """2*H*(576+512) per (query token, visible key) pair; query i sees L_b + i + 1 keys."""
        L = self.cache_lengths.to(torch.int64)
        T = self.max_prompt_length
        vis = sum(int((L + i + 1).sum().item()) for i in range(T))
        return 2 * self.cfg.num_q_heads * (HEAD_DIM + V_DIM) * vis


def u32_as_i32(t: torch.Tensor) -> torch.Tensor:
    """Store uint32 values (given as int64) in an int32 tensor with the same bit pattern."""
    v = t.to(torch.int64) & 0xFFFFFFFF
    return torch.where(v >= (1 << 31), v - (1 << 32), v).to(torch.int32)


def i32_as_u32(t: torch.Tensor) -> torch.Tensor:
    """Read an int32 tensor holding uint32 bit patterns back as int64 values."""
    return t.to(torch.int64) & 0xFFFFFFFF


def _lengths(cfg: DecodeConfig, g: torch.Generator) -> torch.Tensor:
    B = cfg.batch
    if cfg.length_kind == "list":
        return torch.tensor(cfg.length_args, dtype=torch.int64)
    if cfg.length_kind == "fixed":
        return torch.full((B,), int(cfg.length_args[0]), dtype=torch.int64)
    if cfg.length_kind == "uniform":
        lo, hi = cfg.length_args
        return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)
    if cfg.length_kind == "loguniform":
        lo, hi = cfg.length_args
        u = torch.rand((B,), generator=g, dtype=torch.float64)
        v = torch.floor(torch.exp(u * math.log(hi + 1))).to(torch.int64)
        return v.clamp(lo, hi)
    raise ValueError(cfg.length_kind)


def quantize_rows_e4m3(x: torch.Tensor, blocks: int = 1):
    """amax/448 fp32 scales (one per row, or one per each of `blocks` equal slices of a row) and
    saturating RNE e4m3 codes (data generation only).  Returns (codes uint8 like x, scales [..., blocks]
    or [...] when blocks == 1)."""
    xf = x.to(torch.float32)
    xb = xf.reshape(*xf.shape[:-1], blocks, xf.shape[-1] // blocks)
    amax = xb.abs().amax(dim=-1)
    scale = amax / E4M3_MAX
    scale = torch.where(amax > 0, scale, torch.ones_like(scale))
    codes = (xb / scale[..., None]).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    codes = codes.reshape(xf.shape).view(torch.uint8)
    return codes, (scale[..., 0] if blocks == 1 else scale)


@dataclass
class StoreInputs:
    """Tensors of one KV-store call: new tokens' latent and the (pre-assigned) pages they go to."""
    latent: torch.Tensor            # bf16 [B, T, 576]
    cache_lengths: torch.Tensor     # int32 view of uint32 [B]
    lookup_table: torch.Tensor      # int32 view of uint32 [B, max_pages]
    scales_lookup_table: Optional[torch.Tensor]
    blocks: torch.Tensor            # uint8 [NB, 1, L, P, 1, 576]
    scales: torch.Tensor            # fp32 [NSB, 1, L, P, 1, 1]
    layer_idx: int

    def algorithmic_bytes(self) -> int:
        """bf16 latent read (1152 B) + e4m3 row (576 B) + fp32 scale (4 B) written, per token."""
        B, T, _ = self.latent.shape
        return B * T * (2 * HEAD_DIM + HEAD_DIM + 4)


def make_store_inputs(batch: int, new_tokens: int, page_size: int, max_cached: int, seed: int, device="cpu",
                      num_layers: int = 1, layer_idx: int = 0) -> StoreInputs:
    """Seeded inputs of the KV-store step: cached lengths uniform in [0, max_cached], every page a
    request needs for its cached plus new tokens assigned from a randomly permuted pool, latent
    N(0, 1) in bf16.  The pool's bytes start as zeros (the store writes the new rows)."""
    gc = torch.Generator()
    gc.manual_seed(seed)
    L = torch.randint(0, max_cached + 1, (batch,), generator=gc)
    pages = (L + new_tokens + page_size - 1) // page_size
    max_pages = int(pages.max().item())
    nb = int(pages.sum().item())
    perm = torch.randperm(nb, generator=gc).to(torch.int64)
    lut = torch.full((batch, max_pages), INVALID_PAGE, dtype=torch.int64)
    k = 0
    for b in range(batch):
        n = int(pages[b])
        lut[b, :n] = perm[k:k + n]
        k += n
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed + 1)
    latent = torch.randn((batch, new_tokens, HEAD_DIM), generator=g, device=device).to(torch.bfloat16)
    blocks = torch.zeros((nb, 1, num_layers, page_size, 1, HEAD_DIM), dtype=torch.uint8, device=device)
    scales = torch.zeros((nb, 1, num_layers, page_size, 1, 1), dtype=torch.float32, device=device)
    return StoreInputs(latent=latent, cache_lengths=u32_as_i32(L).to(device), lookup_table=u32_as_i32(lut).to(device),
                       scales_lookup_table=None, blocks=blocks, scales=scales, layer_idx=layer_idx)


def make_inputs(cfg: DecodeConfig, device="cpu", *, poison: bool = False,
                lengths: Optional[torch.Tensor] = None, seed: Optional[int] = None,
                q_zero: bool = False, chunk_tokens: int = 1 << 20) -> DecodeInputs:
    """Build one seeded decode problem for `cfg` on `device`.

    poison=True fills every byte the decode must never read (unused page slots,
    unreferenced pages, other layers, kv_dim > 0 slices, unused page-table
    entries) with NaN codes (0x7F), NaN scales and invalid ids.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed if seed is None else seed)
    gc = torch.Generator()  # small host-side draws (lengths, permutations)
    gc.manual_seed((cfg.seed if seed is None else seed) + 7919)

    B, T, H, P = cfg.batch, cfg.q_len, cfg.num_q_heads, cfg.page_size
    L = _lengths(cfg, gc) if lengths is None else lengths.to(torch.int64).cpu()
    n = L + T                                    # keys stored per request
    pages_per_req = (n + P - 1) // P
    max_pages = int(pages_per_req.max().item())
    total_pages = int(pages_per_req.sum().item())

    if cfg.pool_kind == "fixed":
        NB = int(cfg.num_blocks)
    else:
        NB = int(math.ceil(total_pages * cfg.pool_factor)) + cfg.pool_extra
    assert NB >= total_pages
    perm = torch.randperm(NB, generator=gc)
    lut = torch.full((B, max_pages), INVALID_PAGE, dtype=torch.int64)
    off = 0
    for b in range(B):
        k = int(pages_per_req[b])
        lut[b, :k] = perm[off:off + k]
        off += k

    slut = None
    NSB = NB
    if cfg.separate_scales:
        NSB = total_pages + cfg.scales_pool_extra
        sperm = torch.randperm(NSB, generator=gc)
        slut = torch.full((B, max_pages), INVALID_PAGE, dtype=torch.int64)
        off = 0
        for b in range(B):
            k = int(pages_per_req[b])
            slut[b, :k] = sperm[off:off + k]
            off += k

    KVD, NL, li = cfg.kv_dim, cfg.num_layers, cfg.layer_idx
    D = HEAD_DIM
    SG = cfg.scale_blocks
    if poison:
        blocks = torch.full((NB, KVD, NL, P, 1, D), 0x7F, dtype=torch.uint8, device=dev)
        scales = torch.full((NSB, KVD, NL, P, 1, SG), float("nan"), dtype=torch.float32, device=dev)
    else:
        blocks = torch.empty((NB, KVD, NL, P, 1, D), dtype=torch.uint8, device=dev)
        scales = torch.empty((NSB, KVD, NL, P, 1, SG), dtype=torch.float32, device=dev)
        # every slot gets real random data (other layers, spare pages, tails)
        flat_b = blocks.view(-1, D)
        flat_s = scales.view(-1)
        for s0 in range(0, flat_b.shape[0], chunk_tokens):
            s1 = min(flat_b.shape[0], s0 + chunk_tokens)
            x = torch.randn((s1 - s0, D), generator=g, device=dev).to(torch.bfloat16)
            c, s = quantize_rows_e4m3(x)
            flat_b[s0:s1] = c
        for s0 in range(0, flat_s.shape[0], chunk_tokens):
            s1 = min(flat_s.shape[0], s0 + chunk_tokens)
            flat_s[s0:s1] = torch.rand((s1 - s0,), generator=g, device=dev) * 0.01 + 0.001

    # the visible tokens of every request, written in logical order
    req = torch.repeat_interleave(torch.arange(B), n)
    tok = torch.cat([torch.arange(int(x)) for x in n]) if B else torch.zeros(0, dtype=torch.int64)
    blk = lut[req, tok // P]
    sblk = (slut if slut is not None else lut)[req, tok // P]
    slot = tok % P
    ntok = int(n.sum().item())
    blk_d, sblk_d, slot_d = blk.to(dev), sblk.to(dev), slot.to(dev)
    for s0 in range(0, ntok, chunk_tokens):
        s1 = min(ntok, s0 + chunk_tokens)
        x = torch.randn((s1 - s0, D), generator=g, device=dev)
        if cfg.outlier_rate > 0:
            m = torch.rand((s1 - s0,), generator=g, device=dev) < cfg.outlier_rate
            x = torch.where(m[:, None], x * cfg.outlier_mult, x)
        c, s = quantize_rows_e4m3(x.to(torch.bfloat16), SG)
        blocks[blk_d[s0:s1], 0, li, slot_d[s0:s1], 0, :] = c
        scales[sblk_d[s0:s1], 0, li, slot_d[s0:s1], 0, :] = s.reshape(s1 - s0, SG)

    if q_zero:
        q = torch.zeros((B, T, H, D), dtype=torch.bfloat16, device=dev)
    else:
        q = torch.randn((B, T, H, D), generator=g, device=dev).to(torch.bfloat16)

    def u32(t):
        return None if t is None else u32_as_i32(t).to(dev)

    return DecodeInputs(
        cfg=cfg, q=q, blocks=blocks, scales=scales,
        cache_lengths=u32(L), lookup_table=u32(lut), scales_lookup_table=u32(slut),
        max_prompt_length=T, max_cache_length=int(L.max().item()) if B else 0,
        layer_idx=li, softmax_scale=cfg.softmax_scale,
        extra={"num_keys": n, "pages_per_req": pages_per_req},
    )


def to_device(inp: DecodeInputs, device) -> DecodeInputs:
    def mv(t):
        return None if t is None else t.to(device)
    return replace(inp, q=mv(inp.q), blocks=mv(inp.blocks), scales=mv(inp.scales),
                   cache_lengths=mv(inp.cache_lengths), lookup_table=mv(inp.lookup_table),
                   scales_lookup_table=mv(inp.scales_lookup_table))


def permute_pages(inp: DecodeInputs, seed: int = 7) -> DecodeInputs:
    """Physically permute the value pool (and the scale pool) and relabel the tables.

    The logical content every request sees is unchanged, so decode results must
    not change.
    """
    g = torch.Generator()
    g.manual_seed(seed)
    NB = inp.blocks.shape[0]
    pv = torch.randperm(NB, generator=g)           # new position of old block j: pv[j]
    dev = inp.blocks.device
    nb = torch.empty_like(inp.blocks)
    nb[pv.to(dev)] = inp.blocks
    lut = inp.lookup_table.to(torch.int64) & 0xFFFFFFFF
    valid = lut != INVALID_PAGE
    nlut = torch.where(valid.cpu(), pv[lut.cpu().clamp(max=NB - 1)], lut.cpu())
    out = replace(inp, blocks=nb, lookup_table=u32_as_i32(nlut).to(dev))
    if inp.scales_lookup_table is None:
        ns = torch.empty_like(inp.scales)
        ns[pv.to(dev)] = inp.scales
        return replace(out, scales=ns)
    NSB = inp.scales.shape[0]
    ps = torch.randperm(NSB, generator=g)
    ns = torch.empty_like(inp.scales)
    ns[ps.to(dev)] = inp.scales
    slut = inp.scales_lookup_table.to(torch.int64) & 0xFFFFFFFF
    sval = slut != INVALID_PAGE
    nslut = torch.where(sval.cpu(), ps[slut.cpu().clamp(max=NSB - 1)], slut.cpu())
    return replace(out, scales=ns, scales_lookup_table=u32_as_i32(nslut).to(dev))


def separate_scale_space(inp: DecodeInputs, extra: int = 5, seed: int = 11) -> DecodeInputs:
    """Move the scales into their own, independently permuted block-id space.

    Only valid on inputs whose scales share the value pool's ids.  Logical
    content is unchanged.
    """
    assert inp.scales_lookup_table is None
    g = torch.Generator()
    g.manual_seed(seed)
    NB = inp.scales.shape[0]
    NSB = NB + extra
    ps = torch.randperm(NSB, generator=g)[:NB]      # old id j -> new id ps[j]
    dev = inp.scales.device
    ns = torch.full((NSB,) + tuple(inp.scales.shape[1:]), float("nan"),
                    dtype=inp.scales.dtype, device=dev)
    ns[ps.to(dev)] = inp.scales
    lut = inp.lookup_table.to(torch.int64) & 0xFFFFFFFF
    valid = lut != INVALID_PAGE
    slut = torch.where(valid.cpu(), ps[lut.cpu().clamp(max=NB - 1)], lut.cpu())
    return replace(inp, scales=ns, scales_lookup_table=u32_as_i32(slut).to(dev))

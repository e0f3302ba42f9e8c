"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerances of the method: per element
|out - ref| <= 2e-2 * max|ref| + 1e-2, and |lse - ref| <= 1e-3.  The dequantised
bf16 tiles must be bit-exact.  Page permutation and scale id space must not
change the GPU result at all (the reduction order depends only on logical token
order and lengths).
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy

pytestmark = pytest.mark.gpu

OUT_RTOL = 2e-2
OUT_ATOL = 1e-2
LSE_ATOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield
    M.set_num_clusters(0)


def bf16_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check_against(out, lse, ref_out, ref_lse, rows=None, heads=None):
    o = O.bf16_bits_to_f64(bf16_bits(out))
    l = lse.detach().cpu().double().numpy()
    if rows is not None:
        o, l, ref_out, ref_lse = o[rows], l[rows], ref_out[rows], ref_lse[rows]
    if heads is not None:
        o, l, ref_out, ref_lse = o[:, :, heads], l[:, :, heads], ref_out[:, :, heads], ref_lse[:, :, heads]
    assert np.isfinite(o).all() and np.isfinite(l).all()
    tol = OUT_RTOL * np.abs(ref_out).max() + OUT_ATOL
    err = np.abs(o - ref_out)
    assert err.max() <= tol, f"max |err| {err.max():.4g} > {tol:.4g}"
    lerr = np.abs(l - ref_lse).max()
    assert lerr <= LSE_ATOL, f"max |dlse| {lerr:.4g}"
    return err.max(), lerr


def run(inp, **kw):
    out, lse = M.decode_inputs(inp, **kw)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    return out, lse


# ----------------------------------------------------------------------------- dequant (steps A + C)
def test_dequant_bit_exact_all_codes_many_scales():
    """Every e4m3 code times >= 10^4 scales through the real page gather: bit-exact bf16."""
    rng = np.random.default_rng(11)
    n = 10240
    scales = np.concatenate([
        rng.uniform(1e-3, 2.0, n // 2), 2.0 ** rng.integers(-40, 20, n // 8),
        rng.uniform(1e-30, 1e-28, n // 8), rng.uniform(1e30, 1e35, n // 8),
        rng.uniform(1e-40, 1e-38, n // 8)]).astype(np.float32)
    scales = scales[:n]
    codes = rng.integers(0, 256, size=(n, 576), dtype=np.uint8)
    codes[:, :256] = np.arange(256, dtype=np.uint8)[None]
    codes[:, 256:512] = np.roll(np.arange(256, dtype=np.uint8), 77)[None]
    P = 64
    pages = n // P
    perm = rng.permutation(pages + 5)[:pages]
    blocks = np.zeros((pages + 5, 1, 1, P, 1, 576), dtype=np.uint8)
    sc = np.zeros((pages + 5, 1, 1, P, 1, 1), dtype=np.float32)
    for t in range(n):
        blocks[perm[t // P], 0, 0, t % P, 0] = codes[t]
        sc[perm[t // P], 0, 0, t % P, 0, 0] = scales[t]
    lut = perm[None].astype(np.int64)
    dev = "cuda"
    tb = torch.from_numpy(blocks).to(dev)
    ts = torch.from_numpy(sc).to(dev)
    tl = W.u32_as_i32(torch.tensor([n - 1])).to(dev)
    tlut = W.u32_as_i32(torch.from_numpy(lut)).to(dev)
    k = M.gather_dequant(tb, ts, tl, tlut, None, 1, 1, n - 1, 0)
    torch.cuda.synchronize()
    got = bf16_bits(k)[0]
    ref = O.dequant_rows(codes, scales)
    ref_bits = ref.astype(np.float32).view(np.uint32) >> 16
    nan_ref = np.isnan(ref)
    gv = O.bf16_bits_to_f64(got)
    assert np.array_equal(np.isnan(gv), nan_ref)
    assert np.array_equal(got[~nan_ref], ref_bits[~nan_ref].astype(np.uint16))


@pytest.mark.parametrize("cfg_i", [0, 1, 3])
def test_dequant_gather_configs_bit_exact(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    k = M.gather_dequant(inp.blocks, inp.scales, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table,
                         inp.cfg.batch, inp.max_prompt_length, inp.max_cache_length, inp.layer_idx)
    torch.cuda.synchronize()
    a = to_numpy(inp)
    got = O.bf16_bits_to_f64(bf16_bits(k))
    n = O.num_keys(a["cache_lengths"], a["max_prompt_length"])
    for b in list(range(min(4, len(n)))) + [len(n) - 1]:
        ref = O.dequant_request(a["blocks"], a["scales"], a["lookup_table"], a["scales_lookup_table"], b,
                                int(n[b]), a["layer_idx"])
        assert np.array_equal(got[b, :n[b]], ref)


# ----------------------------------------------------------------------------- full decode
@pytest.mark.parametrize("cfg_i", [0, 1, 3])
def test_decode_config_full_parity(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    out, lse = run(inp)
    ref_out, ref_lse = oracle_decode(inp)
    check_against(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("cfg_i,reqs,heads", [
    (2, [int(x) for x in np.linspace(0, 127, 16)], None),     # 16 spread requests, every head
    (4, [0, 1, 2, 3], None),                                   # the whole long-context workload
])
def test_decode_full_size_sampled(cfg_i, reqs, heads):
    """Full-size configs in the bench's launch configuration against the oracle: config 4 whole
    (4 requests x 128 heads, 131 073 keys each), config 2 on 16 of its 128 requests."""
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    out, lse = run(inp)
    ref_out, ref_lse = oracle_decode(inp, requests=reqs, heads=heads)
    check_against(out, lse, ref_out, ref_lse, rows=reqs, heads=heads)
    # every row: finite, and lse at least the largest single score bound is plausible
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("nc", [1, 2, 7, 200])
def test_forced_split_counts(nc):
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    ref_out, ref_lse = oracle_decode(inp)
    M.set_num_clusters(nc)
    try:
        out, lse = run(inp)
    finally:
        M.set_num_clusters(0)
    check_against(out, lse, ref_out, ref_lse)


def test_page_permutation_invariance_bitwise():
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run(inp)
    o2, l2 = run(W.permute_pages(inp, seed=3))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_scale_id_space_invariance_bitwise():
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run(inp)
    sep = W.separate_scale_space(inp, extra=13, seed=2)
    o2, l2 = run(sep)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o3, l3 = run(W.permute_pages(sep, seed=9))
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_poisoned_unread_bytes_bitwise():
    from tests.test_oracle_pins import poison_unread
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run(inp)
    a = poison_unread(inp)
    pz = W.DecodeInputs(cfg=inp.cfg, q=inp.q, blocks=torch.from_numpy(a["blocks"]).cuda(),
                        scales=torch.from_numpy(a["scales"]).cuda(), cache_lengths=inp.cache_lengths,
                        lookup_table=W.u32_as_i32(torch.from_numpy(a["lookup_table"])).cuda(),
                        scales_lookup_table=None, max_prompt_length=inp.max_prompt_length,
                        max_cache_length=inp.max_cache_length, layer_idx=inp.layer_idx,
                        softmax_scale=inp.softmax_scale)
    o2, l2 = run(pz)
    assert torch.isfinite(o2.float()).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _custom(B, T, H, P, lengths, layers=1, layer_idx=0, kv_dim=1, seed=5, separate=False, q_zero=False):
    cfg = W.DecodeConfig("edge", batch=B, q_len=T, num_q_heads=H, page_size=P, num_layers=layers,
                         layer_idx=layer_idx, length_kind="list", length_args=tuple(lengths),
                         pool_kind="permuted", pool_factor=1.5, pool_extra=3, kv_dim=kv_dim, seed=seed,
                         separate_scales=separate, scales_pool_extra=7)
    return W.make_inputs(cfg, device="cuda", q_zero=q_zero)


@pytest.mark.parametrize("case", [
    dict(B=3, T=1, H=128, P=64, lengths=(0, 63, 64)),               # 1 key, tile edge, tile edge + 1
    dict(B=2, T=2, H=128, P=64, lengths=(0, 127)),                   # causal among new tokens
    dict(B=2, T=3, H=32, P=16, lengths=(5, 200)),
    dict(B=2, T=1, H=16, P=48, lengths=(100, 333)),                  # page size not dividing the tile
    dict(B=2, T=1, H=192, P=128, lengths=(700, 129)),                # two head groups, second partial
    dict(B=2, T=1, H=128, P=256, lengths=(1000, 4000), layers=3, layer_idx=2, kv_dim=2),
    dict(B=4, T=1, H=128, P=16, lengths=(1, 2, 3, 4), separate=True),
    dict(B=1, T=1, H=1, P=64, lengths=(5000,)),
    dict(B=2, T=2, H=256, P=80, lengths=(300, 77)),                 # G = 2 and T = 2 together, page size 80
])
def test_edge_cases(case):
    inp = _custom(**case)
    out, lse = run(inp)
    ref_out, ref_lse = oracle_decode(inp)
    check_against(out, lse, ref_out, ref_lse)


def test_q_zero_closed_form_on_gpu():
    inp = _custom(B=2, T=1, H=128, P=64, lengths=(300, 1234), q_zero=True)
    out, lse = run(inp)
    n = (inp.cache_lengths.cpu().double() + 1).numpy()
    assert np.allclose(lse.cpu().numpy()[:, 0, :], np.log(n)[:, None], atol=LSE_ATOL)


def test_repeat_calls_identical():
    inp = W.make_inputs(W.CONFIGS[3], device="cuda")
    o1, l1 = run(inp)
    for _ in range(3):
        o2, l2 = run(inp)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_page_id_sets_device_status_without_fault():
    inp = W.make_inputs(W.CONFIGS[0], device="cuda")
    lut = inp.lookup_table.clone()
    lut[0, 0] = 1000            # >= num_blocks (16): the kernel must skip and flag it
    bad = W.DecodeInputs(**{**inp.__dict__, "lookup_table": lut})
    M.decode_inputs(bad)
    st = M.device_status()
    assert st == 6
    # the context still works afterwards
    out, lse = run(inp)
    ref_out, ref_lse = oracle_decode(inp)
    check_against(out, lse, ref_out, ref_lse)

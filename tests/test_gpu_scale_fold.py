"""GPU parity of the scale-folding decode (mla_decode_paged_fp8_scale_folded).

Against its own float64 oracle (decode_scale_folded) at the decode's stated tolerances
(|out - ref| <= 2e-2 * max|ref| + 1e-2 per element, |lse - ref| <= 1e-3).  Against the pages'
rounded decode the bar widens by the distance between the two oracles (the dequant's rounding,
which this variant leaves out).  With power-of-two scales the two kernels must agree bit for bit:
then bf16(e4m3 * 2^k) = e4m3 * 2^k and bf16(p * 2^k) = bf16(p) * 2^k exactly, so every MMA sees
the same products and the softmax the same scores.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy
from tests.test_gpu_parity import _custom, check_against

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield
    M.set_num_clusters(0)


def run_fold(inp):
    out, lse = M.decode_inputs(inp, fold_scales=True)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    return out, lse


def fold_oracle(inp, **kw):
    a = to_numpy(inp)
    return O.decode_scale_folded(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                                 a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"],
                                 a["softmax_scale"], **kw)


@pytest.mark.parametrize("cfg_i", [0, 1, 3])
def test_fold_config_full_parity(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    out, lse = run_fold(inp)
    ref_out, ref_lse = fold_oracle(inp)
    check_against(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("cfg_i,reqs,heads", [(2, [0, 77, 127], None), (4, [2], list(range(0, 128, 9)))])
def test_fold_full_size_sampled(cfg_i, reqs, heads):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    out, lse = run_fold(inp)
    ref_out, ref_lse = fold_oracle(inp, requests=reqs, heads=heads)
    check_against(out, lse, ref_out, ref_lse, rows=reqs, heads=heads)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_fold_distance_to_the_pages_decode():
    """Against the pages' rounded decode the variant is off by the dequant's bf16 rounding (the
    distance between the two oracles, a few 1e-3 in lse here) plus the kernel tolerance, no more."""
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    out, lse = run_fold(inp)
    ref_out, ref_lse = oracle_decode(inp)
    f_out, f_lse = fold_oracle(inp)
    o = O.bf16_bits_to_f64(out.cpu().view(torch.int16).numpy().view(np.uint16))
    l = lse.cpu().double().numpy()
    gap_o, gap_l = np.abs(f_out - ref_out).max(), np.abs(f_lse - ref_lse).max()
    assert np.abs(o - ref_out).max() <= gap_o + 2e-2 * np.abs(ref_out).max() + 1e-2
    assert np.abs(l - ref_lse).max() <= gap_l + 1e-3


@pytest.mark.parametrize("cfg_i", [1, 3])
def test_fold_bitwise_equal_to_decode_for_power_of_two_scales(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    e = torch.round(torch.log2(inp.scales.clamp_min(1e-30)))
    p2 = W.DecodeInputs(**{**inp.__dict__, "scales": torch.exp2(e).to(torch.float32).contiguous()})
    o1, l1 = M.decode_inputs(p2)
    o2, l2 = run_fold(p2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("nc", [1, 7, 200])
def test_fold_forced_split_counts(nc):
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    rows = [0, 11, 31]
    ref_out, ref_lse = fold_oracle(inp, requests=rows)
    M.set_num_clusters(nc)
    try:
        out, lse = run_fold(inp)
    finally:
        M.set_num_clusters(0)
    check_against(out, lse, ref_out, ref_lse, rows=rows)


@pytest.mark.parametrize("case", [
    dict(B=3, T=1, H=128, P=64, lengths=(0, 63, 64)),
    dict(B=2, T=3, H=32, P=16, lengths=(5, 200)),
    dict(B=2, T=1, H=16, P=48, lengths=(100, 333)),
    dict(B=2, T=1, H=192, P=128, lengths=(700, 129)),
    dict(B=2, T=1, H=128, P=256, lengths=(1000, 4000), layers=3, layer_idx=2, kv_dim=2),
    dict(B=4, T=1, H=128, P=16, lengths=(1, 2, 3, 4), separate=True),
    dict(B=2, T=2, H=256, P=80, lengths=(300, 77)),
])
def test_fold_edge_cases(case):
    inp = _custom(**case)
    out, lse = run_fold(inp)
    ref_out, ref_lse = fold_oracle(inp)
    check_against(out, lse, ref_out, ref_lse)


def test_fold_invariant_to_pages_and_poisoned_unread_bytes():
    from tests.test_oracle_pins import poison_unread
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run_fold(inp)
    o2, l2 = run_fold(W.permute_pages(W.separate_scale_space(inp, extra=13, seed=2), seed=9))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    a = poison_unread(inp)
    pz = W.DecodeInputs(cfg=inp.cfg, q=inp.q, blocks=torch.from_numpy(a["blocks"]).cuda(),
                        scales=torch.from_numpy(a["scales"]).cuda(), cache_lengths=inp.cache_lengths,
                        lookup_table=W.u32_as_i32(torch.from_numpy(a["lookup_table"])).cuda(),
                        scales_lookup_table=None, max_prompt_length=inp.max_prompt_length,
                        max_cache_length=inp.max_cache_length, layer_idx=inp.layer_idx,
                        softmax_scale=inp.softmax_scale)
    o3, l3 = run_fold(pz)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_fold_bad_page_id_sets_device_status_without_fault():
    inp = W.make_inputs(W.CONFIGS[0], device="cuda")
    lut = inp.lookup_table.clone()
    lut[0, 0] = 1000
    M.decode_inputs(W.DecodeInputs(**{**inp.__dict__, "lookup_table": lut}), fold_scales=True)
    assert M.device_status() == 6
    out, lse = run_fold(inp)
    ref_out, ref_lse = fold_oracle(inp)
    check_against(out, lse, ref_out, ref_lse)


def test_fold_rejects_block_scales():
    from dataclasses import replace
    inp = W.make_inputs(replace(W.CONFIGS[0], scale_blocks=9), device="cuda")
    with pytest.raises(M.MlaError):
        M.decode_inputs(inp, fold_scales=True)

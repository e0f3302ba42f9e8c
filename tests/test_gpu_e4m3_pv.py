"""GPU parity of the e4m3 P.V decode (mla_decode_paged_fp8_e4m3_pv).

Against its own float64 oracle (decode_fp8_pv) element by element, at a bound taken from the
oracle's own terms: both sides represent every weight w_t = p_t s_t 2^sigma by two e4m3 terms,
each within e_t = max(2^-8 w_t, min(w_t, 2^-10)) of it (the kernel, whose running maximum and
sigma only make its weights larger, within less), so the two results are within
    2 * sum_t e_t |C[t, v]| 2^-sigma / l      (B below)
of each other, plus the bf16 rounding of the kernel's output and the fp32 score noise (both a
fraction of A = sum_t w_t |C[t, v]| 2^-sigma / l, the scale of the element).  The rms of the
difference must also stay below 4e-3 of the rms of the output (the bf16 output rounding alone is
about 1.1e-3).  A test shows that both have teeth: the oracle with the residual term dropped fails
them on the same inputs.  The lse is the decode's own (the variant changes only the value
product).  Against the pages' rounded decode the decode's stated tolerances hold.  With q = 0 and
power-of-two scales every weight is an exact e4m3 value, so the output is the mean of s_t C[t] up
to the tensor cores' summation and bf16 output rounding (the summation is allowed 2^-12 of the
mean absolute value: the precision the e4m3 MMA keeps while it adds is not stated here).
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy
from tests.test_gpu_parity import _custom, bf16_bits, check_against

pytestmark = pytest.mark.gpu

LSE_ATOL = 1e-3
NOISE = 1e-3 + 2.0 ** -8      # fp32 score noise + bf16 output rounding, as a fraction of A
RMS_REL = 4e-3                # rms(out - oracle) / rms(oracle)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield
    M.set_num_clusters(0)


def run_pv(inp):
    out, lse = M.decode_inputs(inp, e4m3_pv=True)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    return out, lse


def pv_oracle(inp, **kw):
    a = to_numpy(inp)
    return O.decode_fp8_pv(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                           a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"], a["softmax_scale"], **kw)


def split_terms(inp, rows, heads=None):
    """Per output element, B = sum_t e_t |C[t, v]| 2^-sigma / l and A = sum_t w_t |C[t, v]| 2^-sigma / l
    from the oracle's weights (NaN where not computed)."""
    a = to_numpy(inp)
    q = O.bf16_bits_to_f64(a["q"])
    B, T, H, _ = q.shape
    hs = np.arange(H) if heads is None else np.asarray(heads)
    L = a["cache_lengths"].astype(np.int64)
    n_all = O.num_keys(L, int(a["max_prompt_length"]))
    Bd = np.full((B, T, H, 512), np.nan)
    Ad = np.full((B, T, H, 512), np.nan)
    ss = float(np.float32(a["softmax_scale"]))
    for b in rows:
        codes, sc = O.gather_request(a["blocks"], a["scales"], a["lookup_table"], a["scales_lookup_table"], b,
                                     int(n_all[b]), a["layer_idx"])
        for i in range(T):
            vis = int(L[b]) + i + 1
            s = sc[:vis, 0].astype(np.float32).astype(np.float64)
            K = O.dequant_rows(codes[:vis], sc[:vis, :1].astype(np.float32))
            C = np.abs(O.e4m3_decode(codes[:vis])[:, :512])
            x = ss * (q[b, i, hs] @ K.T)
            p = np.exp(x - x.max(axis=1, keepdims=True))
            l = p.sum(axis=1, keepdims=True)
            sg = O.fp8_pv_sigma(s.max())
            w = p * s[None, :] * 2.0 ** sg
            e = np.maximum(2.0 ** -8 * w, np.minimum(w, 2.0 ** -10))
            Bd[b, i, hs] = (e @ C) * 2.0 ** (-sg) / l
            Ad[b, i, hs] = (w @ C) * 2.0 ** (-sg) / l
    return Bd, Ad


def pv_excess(o, ref, Bd, Ad):
    """max over elements of |o - ref| / tolerance (<= 1 passes)."""
    tol = 2.0 * Bd + NOISE * Ad + 1e-6
    m = np.isfinite(ref)
    return (np.abs(o - ref)[m] / tol[m]).max()


def rms_rel(o, ref):
    m = np.isfinite(ref)
    return np.sqrt(np.mean((o[m] - ref[m]) ** 2) / np.mean(ref[m] ** 2))


def check_pv(out, lse, inp, rows=None, heads=None):
    B = inp.q.shape[0]
    rows = list(range(B)) if rows is None else rows
    ref_out, ref_lse = pv_oracle(inp, requests=rows, heads=heads)
    Bd, Ad = split_terms(inp, rows, heads)
    o = O.bf16_bits_to_f64(bf16_bits(out))
    l = lse.detach().cpu().double().numpy()
    hs = slice(None) if heads is None else heads
    o, ref_out, Bd, Ad = o[rows][:, :, hs], ref_out[rows][:, :, hs], Bd[rows][:, :, hs], Ad[rows][:, :, hs]
    l, ref_lse = l[rows][:, :, hs], ref_lse[rows][:, :, hs]
    assert np.isfinite(o).all() and np.isfinite(l).all()
    ex = pv_excess(o, ref_out, Bd, Ad)
    assert ex <= 1.0, f"|out - oracle| reaches {ex:.3g} x the split bound"
    rr = rms_rel(o, ref_out)
    assert rr <= RMS_REL, f"rms(out - oracle) / rms(oracle) = {rr:.3g}"
    lerr = np.abs(l - ref_lse).max()
    assert lerr <= LSE_ATOL, f"max |dlse| {lerr:.4g}"
    return ex


@pytest.mark.parametrize("cfg_i", [0, 1, 3])
def test_pv_config_full_parity(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    out, lse = run_pv(inp)
    check_pv(out, lse, inp)


@pytest.mark.parametrize("cfg_i,reqs,heads", [(2, [0, 77, 127], None), (4, [2], list(range(0, 128, 9)))])
def test_pv_full_size_sampled(cfg_i, reqs, heads):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    out, lse = run_pv(inp)
    check_pv(out, lse, inp, rows=reqs, heads=heads)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_pv_bound_catches_a_dropped_residual(monkeypatch):
    """Planted in the oracle, on the CPU: without the lo term the oracle leaves the bound that the
    kernel meets on the same inputs (config 1)."""
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    out, lse = run_pv(inp)
    rows = [0, 5, 9, 30]
    ex = check_pv(out, lse, inp, rows=rows)
    ref_out, _ = pv_oracle(inp, requests=rows)
    real = O.e4m3_split2
    monkeypatch.setattr(O, "e4m3_split2", lambda w: (real(w)[0], np.zeros_like(real(w)[1])))
    bad_out, _ = pv_oracle(inp, requests=rows)
    monkeypatch.undo()
    Bd, Ad = split_terms(inp, rows)
    bad_ex = pv_excess(bad_out[rows], ref_out[rows], Bd[rows], Ad[rows])
    assert bad_ex > 1.0 and bad_ex > 4 * ex, (bad_ex, ex)
    assert rms_rel(bad_out[rows], ref_out[rows]) > 2 * RMS_REL


def test_pv_within_the_decode_tolerance_of_the_pages_decode():
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    out, lse = run_pv(inp)
    ref_out, ref_lse = oracle_decode(inp)
    check_against(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("P,lengths", [(64, (0, 63, 64, 700)), (16, (5, 200, 4096, 1))])
def test_pv_q_zero_power_of_two_scales_is_the_scaled_mean(P, lengths):
    inp = _custom(B=len(lengths), T=1, H=128, P=P, lengths=lengths, q_zero=True)
    e = torch.round(torch.log2(inp.scales.clamp_min(1e-30)))
    inp = W.DecodeInputs(**{**inp.__dict__, "scales": torch.exp2(e).to(torch.float32).contiguous()})
    out, lse = run_pv(inp)
    a = to_numpy(inp)
    o = O.bf16_bits_to_f64(bf16_bits(out))
    L = a["cache_lengths"].astype(np.int64)
    for b in range(len(lengths)):
        n = int(L[b]) + 1
        codes, sc = O.gather_request(a["blocks"], a["scales"], a["lookup_table"], a["scales_lookup_table"], b, n,
                                     a["layer_idx"])
        V = sc[:n, :1].astype(np.float64) * O.e4m3_decode(codes[:n])[:, :512]
        mean = V.mean(axis=0)
        scale = np.abs(V).mean(axis=0)
        err = np.abs(o[b, 0] - mean[None, :])
        assert (err <= 2.0 ** -8 * np.abs(mean) + 2.0 ** -12 * scale + 1e-7).all(), (err / scale).max()
        assert np.allclose(lse.cpu().double().numpy()[b, 0], np.log(n), atol=1e-5)


@pytest.mark.parametrize("nc", [1, 7, 200])
def test_pv_forced_split_counts(nc):
    """Splitting a request's keys across clusters gives each split its own sigma and running max;
    the combined result stays within the bound."""
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    rows = [0, 11, 31]
    M.set_num_clusters(nc)
    try:
        out, lse = run_pv(inp)
    finally:
        M.set_num_clusters(0)
    check_pv(out, lse, inp, rows=rows)


@pytest.mark.parametrize("case", [
    dict(B=3, T=1, H=128, P=64, lengths=(0, 63, 64)),
    dict(B=2, T=3, H=32, P=16, lengths=(5, 200)),
    dict(B=2, T=1, H=16, P=48, lengths=(100, 333)),
    dict(B=2, T=1, H=192, P=128, lengths=(700, 129)),
    dict(B=2, T=1, H=128, P=256, lengths=(1000, 4000), layers=3, layer_idx=2, kv_dim=2),
    dict(B=4, T=1, H=128, P=16, lengths=(1, 2, 3, 4), separate=True),
    dict(B=2, T=2, H=256, P=80, lengths=(300, 77)),
])
def test_pv_edge_cases(case):
    inp = _custom(**case)
    out, lse = run_pv(inp)
    check_pv(out, lse, inp)


def test_pv_invariant_to_pages_and_scale_ids():
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run_pv(inp)
    o2, l2 = run_pv(W.permute_pages(W.separate_scale_space(inp, extra=13, seed=2), seed=9))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_pv_bad_page_id_sets_device_status_without_fault():
    inp = W.make_inputs(W.CONFIGS[0], device="cuda")
    lut = inp.lookup_table.clone()
    lut[0, 0] = 1000
    M.decode_inputs(W.DecodeInputs(**{**inp.__dict__, "lookup_table": lut}), e4m3_pv=True)
    assert M.device_status() == 6
    out, lse = run_pv(inp)
    check_pv(out, lse, inp)


def test_pv_rejects_block_scales():
    from dataclasses import replace
    inp = W.make_inputs(replace(W.CONFIGS[0], scale_blocks=9), device="cuda")
    with pytest.raises(M.MlaError):
        M.decode_inputs(inp, e4m3_pv=True)

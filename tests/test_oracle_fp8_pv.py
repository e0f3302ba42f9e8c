"""Pins of the oracle's FP8 P.V variant (attend_fp8_pv, decode_fp8_pv), on the CPU.

The variant keeps the decode's scores and softmax and takes the value product in e4m3: value rows
are the exact e4m3 values, each weight carries its token's scale and a power-of-two headroom
factor 2^sigma and is split into two e4m3 terms.  Pinned here against things the oracle does not
compute the same way: a brute-force nearest-code search for the split, the split's error bound
from the format, a closed form (q = 0 with power-of-two scales, where the split is exact), the
unrounded attention the variant approximates, and planted mistakes that the pins must catch.
"""
import numpy as np
import pytest

from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import to_numpy

ALL_CODES = np.arange(256, dtype=np.uint8)
FINITE = ALL_CODES[(ALL_CODES & 0x7F) != 0x7F]
FINITE_VALUES = O.e4m3_decode(FINITE)


def nearest_e4m3(y):
    """Brute force: the finite e4m3 value nearest to y (ties to the even mantissa, saturating)."""
    y = float(np.float32(y))
    d = np.abs(FINITE_VALUES - y)
    best = d.min()
    cand = FINITE[d == best]
    if len(cand) > 1:
        cand = cand[(cand & 1) == 0]          # tie: even mantissa (the last code bit)
    vals = O.e4m3_decode(cand)
    # +0 and -0 both represent 0: take the one with y's sign
    if vals[0] == 0.0:
        return -0.0 if np.signbit(y) else 0.0
    return float(vals[0])


def test_split_equals_brute_force_nearest_pair():
    rng = np.random.default_rng(5)
    w = np.concatenate([rng.uniform(0, 448, 400), 2.0 ** rng.uniform(-12, 8.8, 600),
                        FINITE_VALUES[FINITE_VALUES >= 0] * 1.03]).astype(np.float32)
    w = np.minimum(w, 448.0).astype(np.float32)
    hi, lo = O.e4m3_split2(w)
    for k in range(len(w)):
        h = nearest_e4m3(w[k])
        r = np.float32(np.float64(w[k]) - h)
        assert hi[k] == h, (w[k], hi[k], h)
        assert lo[k] == nearest_e4m3(r), (w[k], lo[k], r)


def test_split_error_bound_from_the_format():
    """|hi + lo - w| <= max(2^-8 w, 2^-10): hi is within 2^-4 of w's binade, the residual is below
    2^(e-4) and its own rounding is within 2^-4 of it (or 2^-10 absolute in the subnormal range)."""
    rng = np.random.default_rng(6)
    w = np.concatenate([2.0 ** rng.uniform(-14, np.log2(448), 200000), np.linspace(0, 448, 20001)]).astype(np.float32)
    hi, lo = O.e4m3_split2(w)
    err = np.abs(hi + lo - w.astype(np.float64))
    assert (err <= np.maximum(2.0 ** -8 * w, 2.0 ** -10)).all()
    # and the bound is not loose by orders of magnitude: the worst case reaches a quarter of it
    assert (err / np.maximum(2.0 ** -8 * w, 2.0 ** -10)).max() > 0.25


def test_sigma_is_the_largest_power_that_fits():
    rng = np.random.default_rng(7)
    for s_max in np.concatenate([2.0 ** rng.uniform(-30, 10, 500), [112.0, 56.0, 1.75, 0.875, 1.0, 448.0]]):
        sg = O.fp8_pv_sigma(s_max)
        assert s_max * 2.0 ** sg <= 112.0 < s_max * 2.0 ** (sg + 1)
        assert 4.0 * s_max * 2.0 ** sg <= O.E4M3_MAX


def _row(n, rng, pow2_scales=False):
    codes = rng.integers(0, 256, size=(n, 576), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] ^= 1                    # no NaN codes
    if pow2_scales:
        s = 2.0 ** rng.integers(-9, -3, n)
    else:
        s = rng.uniform(2e-3, 2e-2, n) * np.where(rng.random(n) < 0.05, 20.0, 1.0)
    return codes, s.astype(np.float32)


def test_q_zero_with_power_of_two_scales_is_exact():
    """q = 0: every p is 1, w = s_t 2^sigma is a power of two (an e4m3 value), lo = 0, and the
    result is the mean over keys of s_t C[t] (the scale-folded oracle's value) with lse = ln n."""
    rng = np.random.default_rng(8)
    codes, s = _row(300, rng, pow2_scales=True)
    q = np.zeros((4, 576))
    out, lse = O.attend_fp8_pv(q, codes, s, 1 / np.sqrt(192))
    ref = (s.astype(np.float64)[:, None] * O.e4m3_decode(codes)[:, :512]).mean(axis=0)
    assert np.allclose(out, ref[None, :], rtol=0, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(lse, np.log(300), atol=1e-12)
    fo, fl = O.attend_scale_folded(q, codes, s, 1 / np.sqrt(192))
    assert np.allclose(out, fo, rtol=0, atol=1e-12 * np.abs(ref).max())


def _unrounded(q, codes, s, softmax_scale):
    """Scores of the decode (R3 keys), values s_t C[t] unrounded, float64; and the bound the
    two-term split allows per output element: weight w_t = p_t s_t 2^sigma is represented within
    max(2^-8 w_t, min(w_t, 2^-10)) (the format's bound, test_split_error_bound_from_the_format),
    so out moves by at most sum_t that * |C[t, v]| * 2^-sigma / l."""
    K = O.dequant_rows(codes, s[:, None])
    C = O.e4m3_decode(codes)
    x = float(np.float32(softmax_scale)) * (q @ K.T)
    p = np.exp(x - x.max(axis=1, keepdims=True))
    l = p.sum(axis=1, keepdims=True)
    V = s.astype(np.float64)[:, None] * C[:, :512]
    sigma = O.fp8_pv_sigma(s.max())
    w = p * s.astype(np.float64)[None, :] * 2.0 ** sigma
    e = np.maximum(2.0 ** -8 * w, np.minimum(w, 2.0 ** -10))
    bound = (e @ np.abs(C[:, :512])) * 2.0 ** (-sigma) / l
    return (p @ V) / l, bound * 1.0001 + 1e-13 * (p @ np.abs(V)) / l


def test_within_the_split_bound_of_the_unrounded_attention():
    rng = np.random.default_rng(9)
    codes, s = _row(777, rng)
    q = rng.standard_normal((8, 576))
    out, lse = O.attend_fp8_pv(q, codes, s, 1 / np.sqrt(192))
    exact, bound = _unrounded(q, codes, s, 1 / np.sqrt(192))
    assert (np.abs(out - exact) <= bound).all()
    # the bound is not loose by orders of magnitude
    assert (np.abs(out - exact) / bound).max() > 0.01
    # and close to the decode itself (bf16 V rows) at the method's tolerance
    ref_out, ref_lse = O.attend(q, O.dequant_rows(codes, s[:, None]), 1 / np.sqrt(192))
    assert np.abs(out - ref_out).max() <= 2e-2 * np.abs(ref_out).max() + 1e-2
    assert np.abs(lse - ref_lse).max() <= 1e-12


def test_decode_fp8_pv_through_the_page_tables():
    """decode_fp8_pv reads the same gathered rows as decode (config 3: its own scale id space)."""
    inp = W.make_inputs(W.CONFIGS[3], device="cpu")
    a = to_numpy(inp)
    reqs = [0, 17, 63]
    out, lse = O.decode_fp8_pv(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                               a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"], a["softmax_scale"],
                               requests=reqs)
    ref_out, ref_lse = O.decode(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                                a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"], a["softmax_scale"],
                                requests=reqs)
    assert np.isfinite(out[reqs]).all()
    assert np.abs(out[reqs] - ref_out[reqs]).max() <= 2e-2 * np.abs(ref_out[reqs]).max() + 1e-2
    assert np.abs(lse[reqs] - ref_lse[reqs]).max() <= 1e-9


@pytest.mark.parametrize("mistake", ["no_lo", "no_sigma_undo", "scale_not_folded"])
def test_planted_mistakes_are_caught(mistake, monkeypatch):
    rng = np.random.default_rng(10)
    codes, s = _row(500, rng)
    q = rng.standard_normal((4, 576))
    real_split, real_sigma = O.e4m3_split2, O.fp8_pv_sigma

    if mistake == "no_lo":
        monkeypatch.setattr(O, "e4m3_split2", lambda w: (real_split(w)[0], np.zeros_like(real_split(w)[1])))
    elif mistake == "no_sigma_undo":
        # the weights are scaled but the result is not scaled back (sigma read as 0 on the way out)
        def bad_attend(q, codes, scale, ss):
            out, lse = O.__dict__["_attend_fp8_pv_real"](q, codes, scale, ss)
            return out * 2.0 ** real_sigma(np.max(scale)), lse
        monkeypatch.setattr(O, "_attend_fp8_pv_real", O.attend_fp8_pv, raising=False)
        monkeypatch.setattr(O, "attend_fp8_pv", bad_attend)
    else:
        s_used = np.ones_like(s)
        monkeypatch.setattr(O, "fp8_pv_sigma", lambda s_max: real_sigma(1.0))
        out, lse = O.attend_fp8_pv(q, codes, s_used, 1 / np.sqrt(192))
        exact, bound = _unrounded(q, codes, s, 1 / np.sqrt(192))
        assert np.abs(out - exact).max() > 2e-2 * np.abs(exact).max()
        return
    out, lse = O.attend_fp8_pv(q, codes, s, 1 / np.sqrt(192))
    monkeypatch.undo()
    exact, bound = _unrounded(q, codes, s, 1 / np.sqrt(192))
    assert not (np.abs(out - exact) <= bound).all()

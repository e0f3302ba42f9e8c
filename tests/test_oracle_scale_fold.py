"""Pins for the oracle of the scale-folding variant (attend_scale_folded / decode_scale_folded).

The variant keeps key and value elements as exact e4m3 values and applies the per-token scale to
score column t and to weight column t.  In exact arithmetic that is attention over the unrounded
keys s_t * e4m3(code); with power-of-two scales the pages' rounded dequant is exact too, so there
the variant must agree with the pinned per-token decode; and its distance from the rounded decode
is the size of the dequant's bf16 rounding.  A fold that forgets the weight columns, scales the
scores twice or drops the softmax scale fails one of these.
"""
import math

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy


def _codes(rng, n, d=576):
    c = rng.integers(0, 256, size=(n, d), dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x30                               # no NaN codes
    return c


def _q(rng, H):
    x = torch.from_numpy(rng.standard_normal((H, 576))).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fold_equals_attention_over_unrounded_keys(seed):
    rng = np.random.default_rng(seed)
    n, H = 40, 6
    codes = _codes(rng, n)
    s = (rng.random(n) * 0.05 + 1e-3).astype(np.float32)
    q = _q(rng, H)
    K = O.e4m3_decode(codes) * s.astype(np.float64)[:, None]   # exact products, no rounding
    ref_out, ref_lse = O.attend(q, K, 0.0721)
    out, lse = O.attend_scale_folded(q, codes, s, 0.0721)
    assert np.allclose(out, ref_out, rtol=1e-12, atol=1e-14 * np.abs(ref_out).max())
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_fold_brute_force_tiny():
    """Per-element Python loops (math.exp / sums in Python floats) on 3 keys, 2 heads."""
    rng = np.random.default_rng(7)
    n, H = 3, 2
    codes = _codes(rng, n)
    s = np.array([0.5, 0.0078125, 3.25], dtype=np.float32)
    q = _q(rng, H)
    sm = float(np.float32(0.1))
    C = O.e4m3_decode(codes)
    out, lse = O.attend_scale_folded(q, codes, s, 0.1)
    for h in range(H):
        x = []
        for t in range(n):
            acc = 0.0
            for d in range(576):
                acc += float(q[h, d]) * float(C[t, d]) * float(s[t])
            x.append(sm * acc)
        m = max(x)
        tot = sum(math.exp(v - m) for v in x)
        want_lse = m + math.log(tot)
        assert abs(lse[h] - want_lse) < 1e-9
        for v in (0, 1, 200, 511):
            want = sum(math.exp(x[t] - want_lse) * float(s[t]) * float(C[t, v]) for t in range(n))
            assert abs(out[h, v] - want) <= 1e-9 * max(1.0, abs(want))


def _pow2_scales(inp):
    sc = inp.scales.clone()
    e = torch.round(torch.log2(sc.clamp_min(1e-30)))
    return W.DecodeInputs(**{**inp.__dict__, "scales": torch.exp2(e).to(torch.float32)})


@pytest.mark.parametrize("cfg_i", [0, 3])
def test_fold_matches_pinned_decode_for_power_of_two_scales(cfg_i):
    """With scales 2^k the rounded dequant is exact, so both oracles compute the same numbers
    (through the same page tables, including a separate scale id space for config 3)."""
    inp = _pow2_scales(W.make_inputs(W.CONFIGS[cfg_i]))
    a = to_numpy(inp)
    rows = None if cfg_i == 0 else [0, 9, 40]
    ref_out, ref_lse = oracle_decode(inp, requests=rows)
    out, lse = O.decode_scale_folded(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                                     a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"],
                                     a["softmax_scale"], requests=rows)
    sel = slice(None) if rows is None else rows
    assert np.allclose(out[sel], ref_out[sel], rtol=1e-11, atol=1e-12)
    assert np.allclose(lse[sel], ref_lse[sel], rtol=0, atol=1e-11)


def test_fold_differs_from_rounded_decode_by_the_dequant_rounding():
    """General fp32 scales: the two oracles differ, but by no more than bf16 rounding of the keys
    (relative 2^-8 per element) can move the result."""
    inp = W.make_inputs(W.CONFIGS[0])
    a = to_numpy(inp)
    ref_out, ref_lse = oracle_decode(inp)
    out, lse = O.decode_scale_folded(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                                     a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"],
                                     a["softmax_scale"])
    d = np.abs(out - ref_out).max()
    assert 0 < d <= 2.0 ** -7 * np.abs(ref_out).max()
    assert 0 < np.abs(lse - ref_lse).max() <= 1e-2


def test_fold_rejects_block_scales():
    from dataclasses import replace
    inp = W.make_inputs(replace(W.CONFIGS[0], scale_blocks=9))
    a = to_numpy(inp)
    with pytest.raises(ValueError):
        O.decode_scale_folded(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                              a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"], a["softmax_scale"])


def test_fold_visibility_is_causal_among_new_tokens():
    """q_len 2: query 0 must not see the step's second token; replacing that token's codes changes
    query 1's result only."""
    cfg = W.DecodeConfig("fold_vis", batch=1, q_len=2, num_q_heads=4, page_size=16, num_layers=1, layer_idx=0,
                         length_kind="list", length_args=(20,), pool_kind="fixed", num_blocks=4, seed=5)
    inp = W.make_inputs(cfg)
    a = to_numpy(inp)
    args = lambda blk: (a["q"], blk, a["scales"], a["cache_lengths"], a["lookup_table"], a["scales_lookup_table"],
                        a["max_prompt_length"], a["layer_idx"], a["softmax_scale"])
    o1, l1 = O.decode_scale_folded(*args(a["blocks"]))
    blk2 = a["blocks"].copy()
    t = 21                                                     # position of the second new token
    page = int(a["lookup_table"][0, t // 16])
    blk2[page, 0, 0, t % 16, 0, :] = 0x38                     # all 1.0
    o2, l2 = O.decode_scale_folded(*args(blk2))
    assert np.array_equal(o1[0, 0], o2[0, 0]) and np.array_equal(l1[0, 0], l2[0, 0])
    assert not np.allclose(o1[0, 1], o2[0, 1])

"""Pins for the oracle with sub-token block scales (head_dim_granularity g > 1).

Scale j of a token covers dims [j * 576 / g, (j + 1) * 576 / g) ("KVCacheScalesMHAOperand":
quantization granularity; "generic_get_paged_cache_with_scales": the scales tensor's last dim).
The dequant is tied to a per-element loop and to torch's fp8 decode / fp32 multiply / bf16 cast;
equal block scales must reproduce the per-token result bit for bit, end to end.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy

GRANULARITIES = [2, 3, 4, 6, 9, 12, 18, 36]


@pytest.mark.parametrize("g", GRANULARITIES)
def test_block_dequant_matches_per_element_loop(g):
    rng = np.random.default_rng(g)
    codes = rng.integers(0, 256, size=(5, 576), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                       # no NaN codes
    sc = (rng.random((5, g)) * 0.02 + 1e-4).astype(np.float32)
    got = O.dequant_rows(codes, sc)
    bs = 576 // g
    want = np.empty((5, 576))
    for t in range(5):
        for d in range(576):
            prod = np.float32(O.e4m3_decode(codes[t, d]) * np.float64(sc[t, d // bs]))
            want[t, d] = O.bf16_round_f32(prod)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("g", [9, 36])
def test_block_dequant_matches_torch(g):
    rng = np.random.default_rng(100 + g)
    codes = rng.integers(0, 256, size=(64, 576), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01
    sc = (rng.random((64, g)) * 3.0 + 1e-3).astype(np.float32)
    ours = O.dequant_rows(codes, sc)
    v = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32)
    s = torch.from_numpy(sc).repeat_interleave(576 // g, dim=1)
    ref = (v * s).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_equal_block_scales_reproduce_per_token_decode():
    base = W.make_inputs(W.CONFIGS[0])
    g = 9
    sc9 = base.scales.repeat(1, 1, 1, 1, 1, g).contiguous()
    blk = W.DecodeInputs(**{**base.__dict__, "scales": sc9})
    o1, l1 = oracle_decode(base)
    o9, l9 = oracle_decode(blk)
    assert np.array_equal(o1, o9) and np.array_equal(l1, l9)


def test_generator_block_scales_cover_their_slices():
    """Each of the g scales is the amax of its own slice / 448, so the slice's largest |value| codes to 448."""
    cfg = replace(W.CONFIGS[0], scale_blocks=9)
    inp = W.make_inputs(cfg)
    a = to_numpy(inp)
    codes, sc = O.gather_request(a["blocks"], a["scales"], a["lookup_table"], a["scales_lookup_table"], 0, 20,
                                 a["layer_idx"])
    assert sc.shape == (20, 9)
    v = O.e4m3_decode(codes).reshape(20, 9, 64)
    assert np.all(np.abs(v).max(axis=-1) == 448.0)
    assert len(np.unique(sc[0])) > 1                            # the scales really differ per slice

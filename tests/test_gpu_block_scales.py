"""GPU parity with sub-token block scales (head_dim_granularity g > 1: g fp32 scales per token,
scale j covering dims [j * 576 / g, (j + 1) * 576 / g)).

The dequantised tiles must be bit-exact against the oracle; the decode within the stated
tolerances; and g copies of each per-token scale must give bitwise the same decode as g = 1 (the
converted tiles are identical, so every MMA is).
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy
from tests.test_gpu_parity import bf16_bits, check_against, run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield


def _cfg(base_i, g, **kw):
    return replace(W.CONFIGS[base_i], scale_blocks=g, **kw)


@pytest.mark.parametrize("g", [2, 3, 9, 36])
def test_block_scale_dequant_bit_exact(g):
    inp = W.make_inputs(_cfg(0, g), device="cuda")
    k = M.gather_dequant(inp.blocks, inp.scales, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table,
                         inp.cfg.batch, inp.max_prompt_length, inp.max_cache_length, inp.layer_idx)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    a = to_numpy(inp)
    got = O.bf16_bits_to_f64(bf16_bits(k))
    n = O.num_keys(a["cache_lengths"], a["max_prompt_length"])
    for b in range(len(n)):
        ref = O.dequant_request(a["blocks"], a["scales"], a["lookup_table"], a["scales_lookup_table"], b,
                                int(n[b]), a["layer_idx"])
        assert np.array_equal(got[b, :n[b]], ref)


@pytest.mark.parametrize("g", [9, 36])
def test_block_scale_decode_parity_small(g):
    inp = W.make_inputs(_cfg(0, g), device="cuda")
    out, lse = run(inp)
    ref_out, ref_lse = oracle_decode(inp)
    check_against(out, lse, ref_out, ref_lse)


def test_block_scale_decode_parity_ragged_separate_scales():
    """q_len 2, log-uniform lengths, scales paged through their own id space, g = 9 (64-dim blocks)."""
    inp = W.make_inputs(_cfg(3, 9), device="cuda")
    out, lse = run(inp)
    rows = [0, 7, 31, 63]
    ref_out, ref_lse = oracle_decode(inp, requests=rows)
    check_against(out, lse, ref_out, ref_lse, rows=rows)


def test_replicated_block_scales_are_bitwise_per_token():
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run(inp)
    rep = W.DecodeInputs(**{**inp.__dict__, "scales": inp.scales.repeat(1, 1, 1, 1, 1, 9).contiguous()})
    o9, l9 = run(rep)
    assert torch.equal(o1, o9) and torch.equal(l1, l9)


def test_block_scale_forced_splits():
    inp = W.make_inputs(_cfg(1, 9), device="cuda")
    rows = [0, 13, 31]
    ref_out, ref_lse = oracle_decode(inp, requests=rows)
    try:
        for nc in (1, 7, 200):
            M.set_num_clusters(nc)
            out, lse = run(inp)
            check_against(out, lse, ref_out, ref_lse, rows=rows)
    finally:
        M.set_num_clusters(0)

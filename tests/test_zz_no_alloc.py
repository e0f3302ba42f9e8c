"""The no-allocation decode entry point, checked against the regular one.

mla_decode_paged_fp8_noalloc exists for callers that may not allocate device memory while they run
(a CUDA graph being captured, an allocator that owns the device, a service that forbids allocation
after start-up).  It keeps its split plan and partial results in a fixed array built into the
library instead of the lazily allocated workspace, so this test calls it twice in a row with
different problems (the second call finds the first call's leftovers in the array) and compares each
result with mla_decode_paged_fp8 on the same inputs: the same kernels with the same split, so the
results must be equal bit for bit, and both must match the float64 oracle at the parity tests'
tolerances.  A second test captures the call in a CUDA graph and replays it with new inputs.

The file name sorts last so that a run stopping at the first failure has run every other test
first; the test also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import _lib
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode

pytestmark = pytest.mark.gpu

OUT_RTOL = 2e-2
OUT_ATOL = 1e-2
LSE_ATOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield


def _bf16_to_f64(t):
    return O.bf16_bits_to_f64(t.detach().cpu().view(torch.int16).numpy().view(np.uint16))


def _close_oracle(out, lse, ref_out, ref_lse):
    a = _bf16_to_f64(out)
    assert np.isfinite(a).all()
    tol = OUT_RTOL * np.abs(ref_out).max() + OUT_ATOL
    assert np.abs(a - ref_out).max() <= tol
    assert np.abs(lse.detach().cpu().double().numpy() - ref_lse).max() <= LSE_ATOL


@pytest.mark.parametrize("first,second", [(1, 3), (0, 2)])
def test_noalloc_matches_regular_entry_two_calls_in_a_row(first, second):
    for cfg_i in (first, second):
        inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
        out_ref, lse_ref = M.decode_inputs(inp)
        out = torch.full_like(out_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        _lib.decode_noalloc(inp.q, inp.blocks, inp.scales, inp.cache_lengths, inp.lookup_table,
                            inp.scales_lookup_table, inp.max_prompt_length, inp.max_cache_length,
                            inp.layer_idx, inp.softmax_scale, out, lse)
        torch.cuda.synchronize()
        assert M.device_status() == 0
        assert torch.equal(out, out_ref) and torch.equal(lse, lse_ref)
        if cfg_i in (0, 1, 3):               # the oracle finishes these whole workloads in seconds
            ref_out, ref_lse = oracle_decode(inp)
            _close_oracle(out, lse, ref_out, ref_lse)


def test_noalloc_captured_in_a_cuda_graph_replays_with_new_inputs():
    """Capture the no-allocation decode once, then change q and the cache lengths in place (same
    shapes, lengths within the captured max_cache_length, same page tables and pool) and replay:
    the replay must equal the regular entry on the new inputs bit for bit (same kernels, same split)."""
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    q = inp.q.clone()
    lens = inp.cache_lengths.clone()
    out = torch.empty((inp.cfg.batch, 1, inp.cfg.num_q_heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((inp.cfg.batch, 1, inp.cfg.num_q_heads), dtype=torch.float32, device="cuda")
    args = (inp.blocks, inp.scales, lens, inp.lookup_table, inp.scales_lookup_table, 1, inp.max_cache_length,
            inp.layer_idx, inp.softmax_scale, out, lse)
    _lib.decode_noalloc(q, *args)                      # first call outside capture (sets up the scratch)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _lib.decode_noalloc(q, *args)
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    for step in range(2):
        q.copy_(torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16))
        lens.copy_((inp.cache_lengths.to(torch.int64) - 37 * (step + 1)).clamp_min(0).to(torch.int32))
        graph.replay()
        torch.cuda.synchronize()
        assert M.device_status() == 0
        ref_out, ref_lse = M.decode(q, inp.blocks, inp.scales, lens, inp.lookup_table, inp.scales_lookup_table, 1,
                                    inp.max_cache_length, inp.layer_idx, inp.softmax_scale)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    del graph


@pytest.mark.parametrize("g", [9, 36])
def test_noalloc_block_scales_match_regular_entry(g):
    """Block scales take two kernel modes (g <= 9 through the ring, larger g by per-thread loads);
    the no-allocation entry must pick the same one and agree bit for bit."""
    from dataclasses import replace
    inp = W.make_inputs(replace(W.CONFIGS[1], scale_blocks=g), device="cuda")
    out_ref, lse_ref = M.decode_inputs(inp)
    out = torch.full_like(out_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    _lib.decode_noalloc(inp.q, inp.blocks, inp.scales, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table,
                        inp.max_prompt_length, inp.max_cache_length, inp.layer_idx, inp.softmax_scale, out, lse)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    assert torch.equal(out, out_ref) and torch.equal(lse, lse_ref)

"""GPU tests of mla_decode_paged_fp8_host (inputs and outputs in host memory, copies overlapped
with the decode of other groups of requests).

With one chunk it must equal the device entry point bit for bit; with n chunks it must equal the
device entry point called on each group of requests alone, bit for bit (each group is its own
decode call), and the oracle at the decode's tolerances.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode
from tests.test_gpu_parity import check_against

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield
    M.set_num_clusters(0)


def host_inputs(inp, pinned=True):
    def h(t):
        if t is None:
            return None
        c = t.detach().cpu().contiguous()
        return c.pin_memory() if pinned else c
    return h(inp.q), h(inp.cache_lengths), h(inp.lookup_table), h(inp.scales_lookup_table)


def run_host(inp, variant=M.VARIANT_DECODE, chunks=0, pinned=True, want_lse=True):
    hq, hl, hlut, hslut = host_inputs(inp, pinned)
    B, T, H, _ = inp.q.shape
    out = torch.empty((B, T, H, 512), dtype=torch.bfloat16, pin_memory=pinned)
    lse = torch.empty((B, T, H), dtype=torch.float32, pin_memory=pinned) if want_lse else None
    M.decode_host(hq, inp.blocks, inp.scales, hl, hlut, hslut, inp.max_prompt_length, inp.max_cache_length,
                  inp.layer_idx, inp.softmax_scale, out, lse, variant=variant, num_chunks=chunks)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    return out, lse


def device_by_groups(inp, n, **kw):
    """The device entry point on each of the n contiguous request groups the host entry cuts."""
    B = inp.q.shape[0]
    outs, lses = [], []
    for i in range(n):
        b0, b1 = B * i // n, B * (i + 1) // n
        sl = slice(b0, b1)
        o, l = M.decode(inp.q[sl].contiguous(), inp.blocks, inp.scales, inp.cache_lengths[sl].contiguous(),
                        inp.lookup_table[sl].contiguous(),
                        None if inp.scales_lookup_table is None else inp.scales_lookup_table[sl].contiguous(),
                        inp.max_prompt_length, inp.max_cache_length, inp.layer_idx, inp.softmax_scale, **kw)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    return torch.cat(outs).cpu(), torch.cat(lses).cpu()


@pytest.mark.parametrize("cfg_i", [0, 1, 3])
def test_one_chunk_equals_the_device_entry(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    o1, l1 = run_host(inp, chunks=1)
    o2, l2 = M.decode_inputs(inp)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2.cpu()) and torch.equal(l1, l2.cpu())


@pytest.mark.parametrize("cfg_i,chunks", [(1, 3), (1, 0), (3, 4), (3, 16)])
def test_chunks_equal_the_device_entry_per_group_and_the_oracle(cfg_i, chunks):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    B = inp.q.shape[0]
    n = chunks if chunks > 0 else (4 if B >= 64 else 2 if B >= 16 else 1)
    o1, l1 = run_host(inp, chunks=chunks)
    o2, l2 = device_by_groups(inp, min(n, B))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    rows = [0, B // 2, B - 1]
    ref_out, ref_lse = oracle_decode(inp, requests=rows)
    check_against(o1, l1, ref_out, ref_lse, rows=rows)


@pytest.mark.parametrize("variant,kw", [(M.VARIANT_E4M3_PV, dict(e4m3_pv=True)),
                                        (M.VARIANT_SCALE_FOLDED, dict(fold_scales=True))])
def test_variants_by_group(variant, kw):
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    o1, l1 = run_host(inp, variant=variant, chunks=2)
    o2, l2 = device_by_groups(inp, 2, **kw)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_pageable_buffers_and_no_lse():
    inp = W.make_inputs(W.CONFIGS[0], device="cuda")
    o1, _ = run_host(inp, chunks=2, pinned=False, want_lse=False)
    o2, _ = device_by_groups(inp, 2)
    assert torch.equal(o1, o2)


def test_back_to_back_calls_reuse_the_staging_area():
    """Two calls on one stream without a synchronisation between them: the second call's copies
    into the staging area wait for the first call's decodes."""
    a = W.make_inputs(W.CONFIGS[1], device="cuda")
    b = W.make_inputs(W.CONFIGS[1], device="cuda", seed=77)
    outs = []
    for inp in (a, b):
        hq, hl, hlut, hslut = host_inputs(inp)
        B, T, H, _ = inp.q.shape
        out = torch.empty((B, T, H, 512), dtype=torch.bfloat16, pin_memory=True)
        lse = torch.empty((B, T, H), dtype=torch.float32, pin_memory=True)
        M.decode_host(hq, inp.blocks, inp.scales, hl, hlut, hslut, inp.max_prompt_length, inp.max_cache_length,
                      inp.layer_idx, inp.softmax_scale, out, lse, num_chunks=4)
        outs.append((out, lse, inp))
    torch.cuda.synchronize()
    for out, lse, inp in outs:
        o2, l2 = device_by_groups(inp, 4)
        assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_device_tensors_are_rejected():
    inp = W.make_inputs(W.CONFIGS[0], device="cuda")
    B, T, H, _ = inp.q.shape
    out = torch.empty((B, T, H, 512), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        M.decode_host(inp.q, inp.blocks, inp.scales, inp.cache_lengths.cpu(), inp.lookup_table.cpu(), None,
                      inp.max_prompt_length, inp.max_cache_length, inp.layer_idx, inp.softmax_scale, out)


def test_block_scales_through_the_host_entry():
    from dataclasses import replace
    inp = W.make_inputs(replace(W.CONFIGS[1], scale_blocks=9), device="cuda")
    o1, l1 = run_host(inp, chunks=2)
    o2, l2 = device_by_groups(inp, 2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)

"""GPU side of context parallelism: the LSE merge kernel against the oracle's combine, and the whole
scheme with the ranks emulated one after another on one GPU (each rank's part is the ordinary
decode of its local page table; the parts are merged by mla_merge_lse_parts_bf16) against the
oracle decode of the whole request, at the decode tolerances.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import context_parallel as CP
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy
from tests.test_gpu_parity import check_against

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield


def test_merge_kernel_against_oracle_combine():
    g = torch.Generator().manual_seed(3)
    R, rows = 4, 777
    outs = torch.randn((R, rows, 512), generator=g).to(torch.bfloat16)
    lses = torch.randn((R, rows), generator=g) * 5
    lses[1, ::3] = float("-inf")                      # empty parts
    lses[:, 10] = float("-inf")                       # a row with no keys at all
    out, lse = M.merge_parts(outs.cuda(), lses.cuda())
    torch.cuda.synchronize()
    o = out.float().cpu().double().numpy()
    l = lse.cpu().double().numpy()
    of = outs.double().numpy()
    lf = lses.double().numpy()
    for row in range(rows):
        if row == 10:
            assert np.all(o[row] == 0) and l[row] == -np.inf
            continue
        parts = [(of[r, row][None], lf[r, row][None]) for r in range(R) if lf[r, row] > -np.inf]
        ref_o, ref_l = O.combine(parts)
        assert np.abs(o[row] - ref_o[0]).max() <= 1e-2 * np.abs(ref_o).max() + 1e-3
        assert abs(l[row] - ref_l[0]) <= 1e-4


def _emulate(inp, world):
    a = to_numpy(inp)
    outs, lses = [], []
    for r in range(world):
        shard = CP.local_shard(a["lookup_table"], a["cache_lengths"], inp.cfg.page_size, world, r,
                               scales_lookup_table=a["scales_lookup_table"], device="cuda")
        out, lse = CP.decode_local(inp.q, inp.blocks, inp.scales, shard, inp.layer_idx, inp.softmax_scale)
        outs.append(out)
        lses.append(lse)
    out, lse = M.merge_parts(torch.stack(outs).contiguous(), torch.stack(lses).contiguous())
    torch.cuda.synchronize()
    assert M.device_status() == 0
    return out, lse


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_small_with_empty_ranges(world):
    cfg = W.DecodeConfig("cp", batch=4, q_len=1, num_q_heads=128, page_size=16, num_layers=2, layer_idx=1,
                         length_kind="list", length_args=(0, 15, 40, 300), pool_kind="permuted", pool_factor=1.5,
                         pool_extra=3, separate_scales=True, scales_pool_extra=4, seed=77)
    inp = W.make_inputs(cfg, device="cuda")
    out, lse = _emulate(inp, world)
    ref_out, ref_lse = oracle_decode(inp)
    check_against(out, lse, ref_out, ref_lse)


def test_context_parallel_moderate_batch():
    inp = W.make_inputs(W.CONFIGS[1], device="cuda")
    out, lse = _emulate(inp, 4)
    rows = [0, 9, 31]
    ref_out, ref_lse = oracle_decode(inp, requests=rows)
    check_against(out, lse, ref_out, ref_lse, rows=rows)


def test_context_parallel_long_context_sampled():
    inp = W.make_inputs(W.CONFIGS[4], device="cuda")
    out, lse = _emulate(inp, 8)
    heads = list(range(0, 128, 17))
    ref_out, ref_lse = oracle_decode(inp, requests=[1], heads=heads)
    check_against(out, lse, ref_out, ref_lse, rows=[1], heads=heads)

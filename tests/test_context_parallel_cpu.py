"""Context parallelism, host side, on the CPU: the page ranges, the local page tables, and the
exchange between two gloo ranks.  Each rank's part is computed by the float64 oracle on its local
tables (the GPU decode of the same tables is checked in tests/test_gpu_context_parallel.py); the
exchanged parts merged by LSE must equal the oracle's decode of the whole request.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import context_parallel as CP
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import to_numpy


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_page_ranges_partition_every_request(world):
    rng = np.random.default_rng(world)
    L = rng.integers(0, 3000, size=40)
    L[:3] = [0, 63, 64]
    P = 64
    parts = CP.page_ranges(L, P, world)
    n = L + 1
    for b in range(len(L)):
        got = []
        for first, count, keys in parts:
            if keys[b]:
                got.append((first[b] * P, first[b] * P + keys[b]))
                assert keys[b] <= count[b] * P
        got.sort()
        assert got[0][0] == 0 and got[-1][1] == n[b]
        assert all(a[1] == c[0] for a, c in zip(got, got[1:]))           # contiguous, disjoint


def _cfg():
    return W.DecodeConfig("cp", batch=4, q_len=1, num_q_heads=8, page_size=16, num_layers=2, layer_idx=1,
                          length_kind="list", length_args=(0, 15, 40, 300), pool_kind="permuted", pool_factor=1.5,
                          pool_extra=3, separate_scales=True, scales_pool_extra=4, seed=77)


def _oracle_part(a, shard):
    lut = shard.lookup_table.numpy().view(np.uint32)
    slut = None if shard.scales_lookup_table is None else shard.scales_lookup_table.numpy().view(np.uint32)
    lens = shard.cache_lengths.numpy().view(np.uint32)
    out, lse = O.decode(a["q"], a["blocks"], a["scales"], lens, lut, slut, 1, a["layer_idx"], a["softmax_scale"])
    lse = np.where(shard.empty.numpy()[:, None, None], -np.inf, lse)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _merge(outs, lses):
    lses = lses.numpy()
    outs = outs.numpy()
    mx = lses.max(axis=0)
    w = np.exp(lses - mx)
    tot = w.sum(axis=0)
    return (w[..., None] * outs).sum(axis=0) / tot[..., None], mx + np.log(tot)


def _rank_main(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = W.make_inputs(_cfg())
        a = to_numpy(inp)
        shard = CP.local_shard(a["lookup_table"], a["cache_lengths"], inp.cfg.page_size, world, rank,
                               scales_lookup_table=a["scales_lookup_table"])
        out, lse = _oracle_part(a, shard)
        outs, lses = CP.exchange_parts(out, lse)
        m_out, m_lse = _merge(outs, lses)
        ref_out, ref_lse = O.decode(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                                    a["scales_lookup_table"], 1, a["layer_idx"], a["softmax_scale"])
        ok = np.allclose(m_out, ref_out, rtol=1e-9, atol=1e-12) and np.allclose(m_lse, ref_lse, rtol=0, atol=1e-9)
        result_q.put((rank, bool(ok), int(shard.empty.sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_exchange_and_merge_to_the_full_decode(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _ in res), res
    assert sum(e for _, _, e in res) >= 1        # the short requests leave some rank without keys


def test_local_shard_tables_and_empty_ranges():
    # lengths 0, 20, 60 at page 16 and q_len 1: 1, 21 and 61 keys = 1, 2 and 4 pages; two ranks
    shard = CP.local_shard(np.arange(12, dtype=np.uint32).reshape(3, 4), [0, 20, 60], 16, 2, 1)
    assert shard.empty.tolist() == [True, False, False]        # request 0's single page is rank 0's
    assert shard.cache_lengths.tolist() == [0, 21 - 16 - 1, 61 - 32 - 1]
    assert shard.lookup_table[1, 0].item() == 5 and shard.lookup_table[2].tolist() == [10, 11]

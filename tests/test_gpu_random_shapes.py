"""Seeded random problem shapes on the GPU, every kernel mode, against the oracle.

The edge-case tests pick shapes by hand; this sweep draws them (batch, query length, heads, page
size, layers, kv_dim, separate scale ids, block-scale granularity, lengths from 0 to a few
thousand, forced split counts) from a fixed seed, so that combinations nobody listed are covered
too.  Each problem is decoded twice and must agree bit for bit with itself, and with the oracle at
the decode's tolerances (the e4m3 P.V mode against its own oracle at the same tolerances).
"""
import random

import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode, to_numpy
from tests.test_gpu_parity import check_against

pytestmark = pytest.mark.gpu

GRANULARITIES = (1, 1, 1, 2, 3, 9, 36)


def draw(i):
    rng = random.Random(9000 + i)
    B = rng.choice((1, 2, 3, 5))
    T = rng.choice((1, 1, 1, 2, 3))
    H = rng.choice((8, 16, 64, 96, 128, 160, 256))
    P = rng.choice((16, 32, 48, 64, 128, 256))
    layers = rng.choice((1, 1, 2, 3))
    kv_dim = rng.choice((1, 1, 2))
    lengths = tuple(rng.choice((0, 1, rng.randrange(0, 200), rng.randrange(0, 3000))) for _ in range(B))
    g = rng.choice(GRANULARITIES)
    mode = rng.choice(("token", "token", "fold", "e4m3"))
    if g > 1:
        mode = "token"                      # the two variants take one scale per token
    nc = rng.choice((0, 0, 1, 5, 150))
    cfg = W.DecodeConfig(f"rand{i}", batch=B, q_len=T, num_q_heads=H, page_size=P, num_layers=layers,
                         layer_idx=rng.randrange(layers), length_kind="list", length_args=lengths,
                         pool_kind="permuted", pool_factor=1.3, pool_extra=2, kv_dim=kv_dim, seed=9100 + i,
                         separate_scales=rng.random() < 0.3, scales_pool_extra=5, scale_blocks=g)
    return cfg, mode, nc


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    yield
    M.set_num_clusters(0)


@pytest.mark.parametrize("i", range(120))
def test_random_problem(i):
    cfg, mode, nc = draw(i)
    inp = W.make_inputs(cfg, device="cuda")
    kw = dict(fold_scales=mode == "fold", e4m3_pv=mode == "e4m3")
    M.set_num_clusters(nc)
    try:
        o1, l1 = M.decode_inputs(inp, **kw)
        o2, l2 = M.decode_inputs(inp, **kw)
        torch.cuda.synchronize()
    finally:
        M.set_num_clusters(0)
    assert M.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    a = to_numpy(inp)
    args = (a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"], a["scales_lookup_table"],
            a["max_prompt_length"], a["layer_idx"], a["softmax_scale"])
    if mode == "fold":
        ref_out, ref_lse = O.decode_scale_folded(*args)
    elif mode == "e4m3":
        ref_out, ref_lse = O.decode_fp8_pv(*args)
    else:
        ref_out, ref_lse = oracle_decode(inp)
    check_against(o1, l1, ref_out, ref_lse)

"""The replica path of bench.py for N > 1, on the CPU with two gloo ranks: every rank gets its own
inputs (different seeds, same shapes), the reported time is the maximum over ranks and the work is
the sum of every rank's bytes."""
import os

import torch.distributed as dist
import torch.multiprocessing as mp


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from paged_fp8_kv_mla_b200 import workloads as W
        cfg = W.CONFIGS[0]
        inp = W.make_inputs(cfg, seed=bench.rank_seed(cfg.seed, rank))
        fp = float(inp.q.float().sum())
        step, kern = bench.max_over_ranks(dist, [10.0 + rank, 5.0 - rank], "cpu")
        total = bench.sum_over_ranks(dist, [float(inp.kv_scale_bytes())], "cpu")[0]
        fps = [None] * world
        dist.all_gather_object(fps, fp)
        sizes = [None] * world
        dist.all_gather_object(sizes, inp.kv_scale_bytes())
        q.put((rank, step, kern, fps, total, sum(sizes)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_timing_and_distinct_inputs():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, step, kern, fps, total, want in res:
        assert step == 11.0 and kern == 5.0          # max over ranks, both ranks agree
        assert fps[0] != fps[1]                       # the replicas decode different batches
        assert total == want                          # the aggregate counts every replica's bytes


def test_single_process_passthrough():
    import bench
    assert bench.max_over_ranks(None, [1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.sum_over_ranks(None, [3.0], "cpu") == [3.0]
    assert bench.rank_seed(1001, 0) == 1001

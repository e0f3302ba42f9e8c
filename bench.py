#!/usr/bin/env python
"""Benchmark of the paged FP8-KV MLA decode on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

One step = one mla_decode_paged_fp8 call over the whole batch of the workload
(plan + decode + split-KV combine kernels).  Inputs are seeded synthetic data
resident in HBM; the L2 is flushed (a write larger than L2) before every timed
step and the flush is outside the timed interval.  Prints one JSON line.

Metric: KV+scale HBM GB/s (each visible key's 576 e4m3 bytes + 4-byte scale,
read once) and decode tokens/s (batch * q_len / step time).  Under torchrun every
rank runs its own batch (weak scaling, no collective on the data path); time is
the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "KV+scale HBM GB/s (% of B200 peak) and decode tokens/s for paged FP8 MLA"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--scale-blocks", type=int, default=1,
                    help="decode with g scales per token (head_dim_granularity), each over 576/g dims")
    ap.add_argument("--fold-scales", action="store_true",
                    help="time the scale-folding decode (per-token scale on score and weight columns)")
    ap.add_argument("--e4m3-pv", action="store_true",
                    help="time the decode whose value product runs on the e4m3 tensor-core path")
    ap.add_argument("--op", choices=["decode", "kv_store"], default="decode",
                    help="decode (the default contract line) or the KV-store step that fills the cache")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=0,
                    help="request groups of the host-buffer call in the e2e measurement (0 = automatic)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0, source="fallback")


def kernel_source_sha():
    """Hash of the CUDA sources' code (comments and whitespace removed), so that a recorded ncu
    capture stays valid across comment edits and becomes invalid with any code change."""
    import re
    h = hashlib.sha256()
    for f in ("ptx.cuh", "mla_kernels.cuh", "mla_api.cu", "mla_kv_store.cuh", "mla_merge.cuh"):
        with open(os.path.join(ROOT, "paged_fp8_kv_mla_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(config_name):
    """DRAM bytes per decode-kernel launch from a committed ncu capture, if it matches this source."""
    p = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_sha") != kernel_source_sha():
        return None
    e = d.get("workloads", {}).get(config_name)
    return None if e is None else e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.idx), "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        rows.append(parts)
            os.unlink(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = sorted(float(r[1]) for r in rows)
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


def rank_seed(base_seed: int, rank: int) -> int:
    """Each replica decodes its own batch (weak scaling): rank r draws its inputs from seed base + 7919 r."""
    return base_seed + 7919 * rank


def max_over_ranks(dist, values, device):
    """Element-wise maximum of per-rank timings (ms) across the process group (one all_reduce)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def sum_over_ranks(dist, values, device):
    """Element-wise sum across the process group (the work all replicas did: their batches differ)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def cpu_oracle_baseline(inp, budget_s, rank_requests=None, fold=False, e4m3_pv=False):
    """The float64 oracle, as it stands, on whole requests of the same workload until ~budget_s."""
    import numpy as np
    from oracle import mla_oracle as O
    from tests.oracle_io import to_numpy
    try:
        from threadpoolctl import threadpool_info
        threads = max([t.get("num_threads", 1) for t in threadpool_info()] or [1])
    except Exception:
        threads = None
    a = to_numpy(inp)
    n = O.num_keys(a["cache_lengths"], a["max_prompt_length"])
    order = rank_requests if rank_requests is not None else list(range(len(n)))
    done, nbytes = [], 0
    t0 = time.perf_counter()
    fn = O.decode_scale_folded if fold else O.decode_fp8_pv if e4m3_pv else O.decode
    for b in order:
        fn(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
           a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"], a["softmax_scale"], requests=[b])
        done.append(b)
        nbytes += int(n[b]) * 580
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": cores, "blas_threads": threads, "kind": "oracle",
            "sample": f"{len(done)} of {len(n)} requests (all {inp.cfg.num_q_heads} heads, "
                      f"{int(sum(n[b] for b in done))} keys), float64 numpy, {dt:.1f} s"}


def run_reference(args):
    """Reference arm: the oracle timed on the host cores on the same workload's requests."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from paged_fp8_kv_mla_b200 import workloads as W
    from oracle import mla_oracle as O
    from tests.oracle_io import to_numpy
    cfg = W.CONFIGS[args.config]
    inp = W.make_inputs(cfg, device="cpu")
    a = to_numpy(inp)
    n = O.num_keys(a["cache_lengths"], a["max_prompt_length"])

    def step(s):
        b = s % len(n)
        O.decode(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                 a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"], a["softmax_scale"], requests=[b])
        return int(n[b]) * 580, a["max_prompt_length"]

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    nbytes = ntok = 0
    for s in range(args.steps):
        bb, tt = step(args.warmup + s)
        nbytes += bb
        ntok += tt
    dt = time.perf_counter() - t0
    v = nbytes / dt / 1e9
    cores = len(os.sched_getaffinity(0))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "decode_tokens_per_s": ntok / dt,
            "config": {"workload": cfg.name, "config_index": args.config, "step": "oracle decode of one request",
                       "l2": "n/a (host)"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"one request per step, rotating over {len(n)} requests"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


STORE_WORKLOAD = dict(batch=64, new_tokens=4096, page_size=64, max_cached=4096, seed=3001)


def run_kv_store(args):
    """KV-store step (quantise + scatter) on a prefill-sized chunk: 64 requests x 4096 new tokens.

    HBM-bound: per token 1152 B of bf16 read, 576 B of e4m3 and a 4 B scale written (454 MB per
    step: the 302 MB of latent alone is larger than L2, so steps run back to back without a flush).
    One GPU.
    """
    import paged_fp8_kv_mla_b200 as M
    from paged_fp8_kv_mla_b200 import workloads as W
    torch.cuda.set_device(0)
    M.load()
    w = STORE_WORKLOAD
    si = W.make_store_inputs(w["batch"], w["new_tokens"], w["page_size"], w["max_cached"], w["seed"], device="cuda")
    nbytes = si.algorithmic_bytes()
    tokens = w["batch"] * w["new_tokens"]
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        M.kv_store(si.latent, si.cache_lengths, si.lookup_table, si.scales_lookup_table, si.layer_idx,
                   si.blocks, si.scales, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if M.device_status() != 0:
        raise RuntimeError("device status error during warm-up")
    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(K):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / K
    if M.device_status() != 0:
        raise RuntimeError("device status error in the timed region")

    e2e = None
    if not args.no_e2e:
        hl = si.latent.cpu().pin_memory()
        dl = torch.empty_like(si.latent)
        Ke = min(K, 50)
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
        for a, b in eev:
            flush.zero_()
            a.record(stream)
            dl.copy_(hl, non_blocking=True)
            M.kv_store(dl, si.cache_lengths, si.lookup_table, si.scales_lookup_table, si.layer_idx,
                       si.blocks, si.scales, stream=stream)
            b.record(stream)
        torch.cuda.synchronize()
        e_ms = sum(a.elapsed_time(b) for a, b in eev) / Ke
        e2e = {"value": nbytes / (e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": hl.numel() * 2,
               "d2h_bytes_per_step": 0, "ms_per_step": e_ms}

    cpu = None
    if not args.no_cpu_baseline:
        import numpy as np
        from oracle import mla_oracle as O
        lat = si.latent[:1].cpu().view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 10.0) and n < lat.shape[1]:
            O.quantize_token(lat[0, n])
            n += 1
        dt = time.perf_counter() - t0
        cpu = {"value": n * (2 * 576 + 576 + 4) / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} tokens of request 0 quantised by the float64 oracle (scatter not timed)"}
    peaks = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "KV-store GB/s (bf16 latent read + e4m3 row and fp32 scale written)", "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, e4m3 + fp32 out", "data": "synthetic",
        "tokens_per_s": tokens / (ms * 1e-3),
        "config": {"workload": "kv_store_prefill_b64_t4096_p64", "batch": w["batch"], "new_tokens": w["new_tokens"],
                   "page_size": w["page_size"], "bytes_per_step": nbytes,
                   "l2": "not flushed: each step's 302 MB of input is larger than L2; steps back to back"},
        "roofline": {"kernel": "mla_kv_store_kernel", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"] + " copy",
                     "traffic": None, "kernel_ms": ms},
        "gpu_launches": K,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "kv_store":
        return run_kv_store(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    import paged_fp8_kv_mla_b200 as M
    from paged_fp8_kv_mla_b200 import workloads as W
    M.load()
    cfg = W.CONFIGS[args.config]
    if args.scale_blocks > 1:
        from dataclasses import replace
        cfg = replace(cfg, name=f"{cfg.name}_g{args.scale_blocks}", scale_blocks=args.scale_blocks)
    fold = bool(args.fold_scales)
    pv = bool(args.e4m3_pv)
    if fold and pv:
        raise SystemExit("--fold-scales and --e4m3-pv select different kernels: pass at most one")
    if fold or pv:
        from dataclasses import replace
        cfg = replace(cfg, name=f"{cfg.name}_{'scale_folded' if fold else 'e4m3_pv'}")
    seed = rank_seed(cfg.seed, rank)
    inp = W.make_inputs(cfg, device="cuda", seed=seed)
    kv_bytes = inp.kv_scale_bytes()
    flops = inp.flops()
    # the bytes every replica reads in one step (each draws its own batch of lengths)
    kv_bytes_all = sum_over_ranks(dist, [kv_bytes], "cuda")[0]
    B, T = cfg.batch, cfg.q_len
    out = torch.empty((B, T, cfg.num_q_heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, T, cfg.num_q_heads), dtype=torch.float32, device="cuda")
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        M.decode_inputs(inp, out=out, lse=lse, stream=stream, fold_scales=fold, e4m3_pv=pv)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if M.device_status() != 0:
        raise RuntimeError("device status error during warm-up")

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in kev:            # torch creates the CUDA event on first record; the library records them later
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    # whole steps (plan -> decode -> combine, launched back to back with programmatic overlap)
    for s in range(K):
        flush.zero_()
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    # the decode kernel alone, for the roofline: events recorded by the library around its launch
    # (a separate pass, because an event between two kernels serialises them)
    for s in range(K):
        flush.zero_()
        M.set_timing_events(*kev[s])
        step()
    M.set_timing_events(None, None)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    step_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    kern_ms = sum(a.elapsed_time(b) for a, b in kev) / K
    if M.device_status() != 0:
        raise RuntimeError("device status error in the timed region")

    # end to end through the public API with host buffers (pinned), copies inside the timed interval
    e2e = None
    if not args.no_e2e:
        hq = inp.q.cpu().pin_memory()
        hl = inp.cache_lengths.cpu().pin_memory()
        hlut = inp.lookup_table.cpu().pin_memory()
        hslut = None if inp.scales_lookup_table is None else inp.scales_lookup_table.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        h2d = hq.numel() * hq.element_size() + hl.numel() * 4 + hlut.numel() * 4 + (0 if hslut is None else hslut.numel() * 4)
        d2h = hout.numel() * 2 + hlse.numel() * 4
        Ke = min(K, 100)
        variant = M.VARIANT_SCALE_FOLDED if fold else M.VARIANT_E4M3_PV if pv else M.VARIANT_DECODE

        def e2e_step():
            # one call of the host-buffer entry point: q, lengths and tables in from pinned host
            # memory, out and lse back, the copies of one request group overlapping another's decode
            M.decode_host(hq, inp.blocks, inp.scales, hl, hlut, hslut, T, inp.max_cache_length, inp.layer_idx,
                          inp.softmax_scale, hout, hlse, variant=variant, num_chunks=args.e2e_chunks, stream=stream)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        for s in range(Ke):
            flush.zero_()
            eev[s][0].record(stream)
            e2e_step()
            eev[s][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = sum(a.elapsed_time(b) for a, b in eev) / Ke
        if dist:
            e2e_ms = max_over_ranks(dist, [e2e_ms], "cuda")[0]
        e2e = {"value": kv_bytes_all / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "api": "mla_decode_paged_fp8_host (pinned host q, lengths, tables in; out, lse back)",
               "num_chunks": args.e2e_chunks if args.e2e_chunks > 0 else "auto"}

    if dist:
        step_ms, kern_ms = max_over_ranks(dist, [step_ms, kern_ms], "cuda")

    peaks = load_peaks()
    gbs = kv_bytes_all / (step_ms * 1e-3) / 1e9
    tflops_k = flops / (kern_ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_baseline(inp, args.cpu_seconds, fold=fold, e4m3_pv=pv)
    if rank == 0:
        line = {
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("e4m3 KV, bf16 Q.K^T MMA, e4m3 P.V MMA (two terms per weight), fp32 accumulate" if pv
                      else "e4m3 KV, bf16 MMA, fp32 accumulate"), "data": "synthetic",
            "decode_tokens_per_s": B * T * world / (step_ms * 1e-3),
            "hbm_frac": gbs / world / peaks["hbm_gbs"],
            "config": {"workload": cfg.name, "config_index": args.config, "batch": B, "q_len": T,
                       "num_q_heads": cfg.num_q_heads, "page_size": cfg.page_size,
                       "kv_scale_bytes_per_step": kv_bytes, "kv_scale_bytes_per_step_all_gpus": kv_bytes_all,
                       "flops_per_step": flops,
                       "l2": "flushed before every timed step (write of %d MB)" % (flush.numel() >> 20),
                       "parallelism": f"replicas x{world}"},
            "roofline": {"kernel": "mla_decode_kernel", "bound": "tensor", "achieved": tflops_k,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": tflops_k / peaks["bf16_tflops"],
                         "peak_source": peaks["source"] + " bf16 burst",
                         "traffic": recorded_traffic(cfg.name), "kernel_ms": kern_ms,
                         "kv_gbs_in_kernel": kv_bytes / (kern_ms * 1e-3) / 1e9,
                         "hbm_frac_in_kernel": kv_bytes / (kern_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "gpu_launches": 3 * K,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

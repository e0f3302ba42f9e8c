"""Per-stage timeline of the decode kernel (diagnostics; not part of the product path).

    python -m paged_fp8_kv_mla_b200.trace --config 1 [--json out.json]

Builds the trace variant of the library (the same kernels with %clock64 stamps compiled in,
libmla_paged_fp8_trace.so), runs one decode of a workload after warm-up, and prints, for cluster 0:
the median duration of each converter / softmax / MMA-issue phase over its tiles and the tile
period, plus the %globaltimer timeline of the launch chain (plan end, decode CTAs, combine).  The
stamps themselves cost time, so absolute numbers run slower than the plain library; the split of
a tile period between the stages is what this is for.  Run it in its own process (the binding
loads one library per process).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import statistics

import torch

from . import _lib, build, workloads as W

TRACE_TILES, TRACE_EVENTS = 64, 32      # the kernel's trace buffer: [2 CTAs][64 tiles][32 events]

# event id -> name (cv = converter warp 0, w7 = converter warp 7, sm = softmax warp 8,
# qk / pv = the MMA issuers, q = the Q loader; cluster 0 only)
EVENTS = {
    1: "cv_kfree", 16: "cv_fetched", 4: "cv_issued", 5: "cv_kdone", 6: "cv_vfree", 2: "cv_vdone", 7: "cv_lutfin",
    26: "w7_kfree", 27: "w7_issued", 28: "w7_kdone", 29: "w7_vfree", 30: "w7_vdone", 31: "w7_lutfin",
    8: "sm_sfull", 9: "sm_ld", 10: "sm_red", 11: "sm_math", 13: "sm_pbuf", 14: "sm_pfull", 15: "sm_epi",
    20: "qk_go", 21: "qk_iss", 22: "pv_go", 23: "pv_iss", 24: "q_free", 25: "q_land",
}

# phases reported: (label, start event, end event), durations in SM clock cycles
PHASES = [
    ("converter K half (warp 0)", "cv_kfree", "cv_kdone"),
    ("converter wait for P.V(g-2) (warp 0)", "cv_kdone", "cv_vfree"),
    ("converter V operand (warp 0)", "cv_vfree", "cv_vdone"),
    ("converter page-table finish (warp 0)", "cv_vdone", "cv_lutfin"),
    ("Q.K^T issue", "qk_go", "qk_iss"),
    ("Q.K^T issue to S in TMEM", "qk_iss", "sm_sfull"),
    ("softmax S to P written", "sm_sfull", "sm_pfull"),
    ("P written to P.V issued", "sm_pfull", "pv_iss"),
]


def run(config: int = 1, seed: int | None = None) -> dict:
    lib = _lib.load(build.build(trace=True))
    lib.mla_debug_set_trace.argtypes = [ctypes.c_void_p]
    lib.mla_debug_marks.argtypes = [ctypes.c_void_p, ctypes.c_int]
    inp = W.make_inputs(W.CONFIGS[config], device="cuda", seed=seed)
    buf = torch.zeros(2 * TRACE_TILES * TRACE_EVENTS + 4 * 4096, dtype=torch.int64, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    marks = (ctypes.c_ulonglong * 8)()
    for _ in range(3):
        _lib.decode_inputs(inp)
    torch.cuda.synchronize()
    flush.zero_()
    buf.zero_()
    torch.cuda.synchronize()
    lib.mla_debug_marks(marks, 1)
    lib.mla_debug_set_trace(ctypes.c_void_p(buf.data_ptr()))
    _lib.decode_inputs(inp)
    torch.cuda.synchronize()
    lib.mla_debug_set_trace(None)
    lib.mla_debug_marks(marks, 0)
    if _lib.device_status() != 0:
        raise RuntimeError("device status error in the traced decode")
    t = buf[:2 * TRACE_TILES * TRACE_EVENTS].view(2, TRACE_TILES, TRACE_EVENTS).cpu()
    rows = []
    for g in range(TRACE_TILES):
        r = {name: int(t[0, g, e]) for e, name in EVENTS.items() if int(t[0, g, e]) > 0}
        if r:
            rows.append(r)
    phases = {}
    for label, a, b in PHASES:
        d = [r[b] - r[a] for r in rows if a in r and b in r]
        if d:
            phases[label] = statistics.median(d)
    starts = [r["cv_kfree"] for r in rows if "cv_kfree" in r]
    period = statistics.median([y - x for x, y in zip(starts, starts[1:])]) if len(starts) > 2 else None
    m = [int(x) for x in marks]
    timeline = {"decode first CTA after plan end (us)": (m[1] - m[0]) / 1e3,
                "decode last CTA exit after plan end (us)": (m[2] - m[0]) / 1e3,
                "combine done after plan end (us)": (m[4] - m[0]) / 1e3 if m[4] else None}
    return {"workload": inp.cfg.name, "tiles_traced": len(rows), "tile_period_cycles": period,
            "phase_median_cycles": phases, "timeline": timeline, "tiles": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--json", default=None, help="also write the full per-tile stamps here")
    a = ap.parse_args()
    res = run(a.config)
    print(f"{res['workload']}: {res['tiles_traced']} tiles of cluster 0, median tile period "
          f"{res['tile_period_cycles']} cycles")
    for k, v in res["phase_median_cycles"].items():
        print(f"  {k:40s} {v:8.0f} cycles")
    for k, v in res["timeline"].items():
        print(f"  {k:40s} {v}")
    if a.json:
        with open(a.json, "w") as fh:
            json.dump(res, fh)


if __name__ == "__main__":
    main()

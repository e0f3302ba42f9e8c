"""Build the C-ABI shared library libmla_paged_fp8.so in place (nvcc, sm_100a only).

    python -m paged_fp8_kv_mla_b200.build [--debug] [--verbose-ptxas] [--trace]

No GPU is needed: nvcc cross-compiles for sm_100a.  The library links the CUDA
runtime statically and reaches the driver's tensor-map encoder through
cudaGetDriverEntryPoint, so it has no link-time dependency on libcuda.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = [os.path.join(PKG, "csrc", "mla_api.cu")]
def _deps():
    """Every source the library is built from (all of csrc/ and the public header)."""
    d = os.path.join(PKG, "csrc")
    return sorted(os.path.join(d, f) for f in os.listdir(d) if f.endswith((".cu", ".cuh"))) + \
        [os.path.join(ROOT, "include", "mla_paged_fp8.h")]
LIB = os.path.join(PKG, "libmla_paged_fp8.so")
# Diagnostic variant with the decode kernel's per-stage timer stamps compiled in (written to a
# device buffer the caller registers); never the library the product path loads.
TRACE_LIB = os.path.join(PKG, "libmla_paged_fp8_trace.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in _deps() + [__file__])


def build(debug: bool = False, verbose_ptxas: bool = False, force: bool = False, out: str = LIB,
          trace: bool = False) -> str:
    if trace and out == LIB:
        out = TRACE_LIB
    if not force and not needs_build(out):
        return out
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"),
        "-o", out + ".tmp",
    ] + SRC
    if debug:
        cmd += ["-DMLA_DEBUG=1"]
    if trace:
        cmd += ["-DMLA_TRACE"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building %s" % out)
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--trace", action="store_true", help="build the diagnostic trace variant")
    a = ap.parse_args()
    print(build(debug=a.debug, verbose_ptxas=a.verbose_ptxas, force=True, trace=a.trace))

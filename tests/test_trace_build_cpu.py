"""The diagnostic trace variant of the library builds (nvcc, no GPU needed) and exports its two
extra entry points; the product library does not export them."""
import ctypes

from paged_fp8_kv_mla_b200 import build, trace


def test_trace_variant_builds_and_exports_its_hooks():
    path = build.build(trace=True)
    assert path == build.TRACE_LIB
    lib = ctypes.CDLL(path)
    assert hasattr(lib, "mla_debug_set_trace") and hasattr(lib, "mla_debug_marks")
    prod = ctypes.CDLL(build.build())
    assert not hasattr(prod, "mla_debug_set_trace")
    assert set(trace.EVENTS.values()) >= {a for _, a, _ in trace.PHASES} | {b for _, _, b in trace.PHASES}

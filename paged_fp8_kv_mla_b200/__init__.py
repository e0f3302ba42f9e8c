"""Paged FP8-KV MLA decode for B200 (sm_100a).

The decode runs in the CUDA kernels of libmla_paged_fp8.so behind the C ABI in
include/mla_paged_fp8.h; this package holds its Python binding (`_lib`), the
build step (`build`), the seeded workload generators (`workloads`) and the host side of context
parallelism (`context_parallel`).
"""
from ._lib import (  # noqa: F401
    MlaError, decode, decode_inputs, gather_dequant, kv_store, set_num_clusters, get_num_clusters, set_wait_limit_ns, withhold_arrival_once, device_status,
    release_workspace, version, set_timing_events, load, LIB_PATH, EXPORTED, merge_parts, decode_noalloc,
    decode_host, VARIANT_DECODE, VARIANT_SCALE_FOLDED, VARIANT_E4M3_PV,
)

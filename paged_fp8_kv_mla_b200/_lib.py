"""ctypes binding of libmla_paged_fp8.so (argument marshalling only).

Every step of the decode runs in the library's CUDA kernels; this module only
turns torch tensors into pointers and shapes.  It raises if the compiled
library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_paged_fp8.so")

MLA_OK = 0
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_CUDA",
                4: "MLA_ERR_WORKSPACE", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_DEVICE_BOUNDS"}

# every symbol include/mla_paged_fp8.h declares
EXPORTED = ["mla_decode_paged_fp8", "mla_gather_dequant_bf16", "mla_set_num_clusters",
            "mla_get_num_clusters", "mla_last_error_string", "mla_get_device_status",
            "mla_release_workspace", "mla_version", "mla_set_timing_events", "mla_decode_paged_fp8_noalloc",
            "mla_kv_store_fp8", "mla_decode_paged_fp8_scale_folded", "mla_merge_lse_parts_bf16",
            "mla_set_wait_limit_ns", "mla_debug_withhold_arrival_once", "mla_decode_paged_fp8_e4m3_pv",
            "mla_decode_paged_fp8_host"]

VARIANT_DECODE, VARIANT_SCALE_FOLDED, VARIANT_E4M3_PV = 0, 1, 2


class MlaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class PagedShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "head_dim", "v_dim", "num_blocks", "kv_dim", "num_layers", "page_size",
        "num_kv_heads", "num_scale_blocks", "head_dim_granularity", "max_pages")]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises FileNotFoundError when it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: build it with `python -m paged_fp8_kv_mla_b200.build`")
    lib = ctypes.CDLL(path)
    vp, u32, f32, i32 = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_float, ctypes.c_int32
    lib.mla_decode_paged_fp8.argtypes = [vp, vp, vp, vp, vp, vp, u32, u32, u32, f32,
                                         ctypes.POINTER(PagedShape), vp, vp, vp]
    lib.mla_decode_paged_fp8.restype = ctypes.c_int
    lib.mla_merge_lse_parts_bf16.argtypes = [vp, vp, ctypes.c_int32, ctypes.c_int64, vp, vp, vp]
    lib.mla_merge_lse_parts_bf16.restype = ctypes.c_int
    lib.mla_decode_paged_fp8_scale_folded.argtypes = lib.mla_decode_paged_fp8.argtypes
    lib.mla_decode_paged_fp8_scale_folded.restype = ctypes.c_int
    lib.mla_decode_paged_fp8_e4m3_pv.argtypes = lib.mla_decode_paged_fp8.argtypes
    lib.mla_decode_paged_fp8_e4m3_pv.restype = ctypes.c_int
    lib.mla_decode_paged_fp8_host.argtypes = [vp, vp, vp, vp, vp, vp, u32, u32, u32, f32,
                                              ctypes.POINTER(PagedShape), vp, vp, i32, i32, vp]
    lib.mla_decode_paged_fp8_host.restype = ctypes.c_int
    lib.mla_decode_paged_fp8_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, u32, u32, u32, f32,
                                                 ctypes.POINTER(PagedShape), vp, vp, vp]
    lib.mla_decode_paged_fp8_noalloc.restype = ctypes.c_int
    lib.mla_gather_dequant_bf16.argtypes = [vp, vp, vp, vp, vp, u32, u32, u32,
                                            ctypes.POINTER(PagedShape), vp, u32, vp]
    lib.mla_gather_dequant_bf16.restype = ctypes.c_int
    lib.mla_kv_store_fp8.argtypes = [vp, vp, vp, vp, u32, u32, ctypes.POINTER(PagedShape), vp, vp, vp]
    lib.mla_kv_store_fp8.restype = ctypes.c_int
    lib.mla_set_num_clusters.argtypes = [i32]
    lib.mla_set_num_clusters.restype = ctypes.c_int
    lib.mla_get_num_clusters.argtypes = []
    lib.mla_get_num_clusters.restype = i32
    lib.mla_last_error_string.argtypes = []
    lib.mla_last_error_string.restype = ctypes.c_char_p
    lib.mla_get_device_status.argtypes = [vp]
    lib.mla_get_device_status.restype = ctypes.c_int
    lib.mla_release_workspace.argtypes = []
    lib.mla_release_workspace.restype = ctypes.c_int
    lib.mla_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.mla_set_wait_limit_ns.restype = ctypes.c_int
    lib.mla_debug_withhold_arrival_once.argtypes = []
    lib.mla_debug_withhold_arrival_once.restype = ctypes.c_int
    lib.mla_set_timing_events.argtypes = [vp, vp]
    lib.mla_set_timing_events.restype = ctypes.c_int
    lib.mla_version.argtypes = []
    lib.mla_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(st: int):
    if st != MLA_OK:
        raise MlaError(st, load().mla_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def paged_shape(batch, num_q_heads, blocks: torch.Tensor, scales: torch.Tensor, lookup_table: torch.Tensor) -> PagedShape:
    """Shape record from the 6-D blocks / scales tensors and the 2-D page table."""
    NB, KVD, NL, P, NKV, D = blocks.shape
    return PagedShape(batch=batch, num_q_heads=num_q_heads, head_dim=D, v_dim=512, num_blocks=NB, kv_dim=KVD,
                      num_layers=NL, page_size=P, num_kv_heads=NKV, num_scale_blocks=scales.shape[0],
                      head_dim_granularity=scales.shape[-1], max_pages=lookup_table.shape[1])


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


_U32 = (torch.int32,) + ((torch.uint32,) if hasattr(torch, "uint32") else ())
_CODES = (torch.uint8,) + ((torch.float8_e4m3fn,) if hasattr(torch, "float8_e4m3fn") else ())


def _expect(name, t, dtypes, ndim=None, last=None, optional=False):
    """The C ABI takes untyped pointers, so the binding checks what it passes: dtype, rank, last dim
    and contiguity (the device is checked last, by _same_device)."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)} (got {t.dtype})")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D (got shape {tuple(t.shape)})")
    if last is not None and t.shape[-1] != last:
        raise ValueError(f"{name} must have last dim {last} (got shape {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(*ts):
    devs = {t.device for t in ts if t is not None}
    if any(d.type != "cuda" for d in devs):
        raise ValueError("all tensors must be CUDA tensors")
    if len(devs) > 1:
        raise ValueError(f"all tensors must be on one CUDA device (got {sorted(str(d) for d in devs)})")


def _check_cache(blocks, scales, cache_lengths, lookup_table, scales_lookup_table, batch):
    _expect("blocks", blocks, _CODES, ndim=6)
    _expect("scales", scales, (torch.float32,), ndim=6)
    _expect("cache_lengths", cache_lengths, _U32, ndim=1)
    _expect("lookup_table", lookup_table, _U32, ndim=2)
    _expect("scales_lookup_table", scales_lookup_table, _U32, ndim=2, optional=True)
    if cache_lengths.shape[0] != batch or lookup_table.shape[0] != batch:
        raise ValueError(f"cache_lengths and lookup_table must have {batch} rows (one per request)")
    if scales_lookup_table is not None and tuple(scales_lookup_table.shape) != tuple(lookup_table.shape):
        raise ValueError("scales_lookup_table must have the shape of lookup_table")


def _check_decode(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, out, lse):
    _expect("q", q, (torch.bfloat16,), ndim=4, last=576)
    B, T, H, _ = q.shape
    _check_cache(blocks, scales, cache_lengths, lookup_table, scales_lookup_table, B)
    _expect("out", out, (torch.bfloat16,), ndim=4, last=512, optional=True)
    _expect("lse", lse, (torch.float32,), ndim=3, optional=True)
    if out is not None and tuple(out.shape) != (B, T, H, 512):
        raise ValueError(f"out must be {(B, T, H, 512)} (got {tuple(out.shape)})")
    if lse is not None and tuple(lse.shape) != (B, T, H):
        raise ValueError(f"lse must be {(B, T, H)} (got {tuple(lse.shape)})")
    _same_device(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, out, lse)


def decode(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length: int,
           max_cache_length: int, layer_idx: int, softmax_scale: float, out=None, lse=None, stream=None,
           want_lse: bool = True, fold_scales: bool = False, e4m3_pv: bool = False):
    """mla_decode_paged_fp8 on torch tensors (all on the current CUDA device).

    q bf16 [B, T, H, 576]; blocks uint8 [NB, kv_dim, L, P, 1, 576]; scales fp32 [NSB, kv_dim, L, P, 1, g];
    cache_lengths / lookup_table / scales_lookup_table int32 tensors holding uint32 values.
    fold_scales=True calls mla_decode_paged_fp8_scale_folded instead, e4m3_pv=True
    mla_decode_paged_fp8_e4m3_pv (g = 1 only, at most one of the two).
    Returns (out bf16 [B, T, H, 512], lse fp32 [B, T, H] or None).
    """
    if fold_scales and e4m3_pv:
        raise ValueError("fold_scales and e4m3_pv select different kernels: pass at most one")
    _check_decode(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, out, lse)
    lib = load()
    B, T, H, D = q.shape
    if out is None:
        out = torch.empty((B, T, H, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=q.device)
    shp = paged_shape(B, H, blocks, scales, lookup_table)
    fn = (lib.mla_decode_paged_fp8_scale_folded if fold_scales else
          lib.mla_decode_paged_fp8_e4m3_pv if e4m3_pv else lib.mla_decode_paged_fp8)
    st = fn(_ptr(q), _ptr(blocks), _ptr(scales), _ptr(cache_lengths), _ptr(lookup_table), _ptr(scales_lookup_table),
            int(max_prompt_length), int(max_cache_length), int(layer_idx), float(softmax_scale), ctypes.byref(shp),
            _ptr(out), _ptr(lse), _stream(stream))
    _check(st)
    return out, lse


def decode_host(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length: int,
                max_cache_length: int, layer_idx: int, softmax_scale: float, out, lse=None, variant: int = 0,
                num_chunks: int = 0, stream=None):
    """mla_decode_paged_fp8_host: q, cache_lengths, the page tables, out and lse are CPU tensors (best
    pinned), blocks and scales CUDA tensors on the current device.  Asynchronous on `stream`: out and
    lse are complete after that stream is synchronised.  variant: VARIANT_DECODE, VARIANT_SCALE_FOLDED
    or VARIANT_E4M3_PV; num_chunks 0 = automatic."""
    _expect("q", q, (torch.bfloat16,), ndim=4, last=576)
    B, T, H, _ = q.shape
    _expect("blocks", blocks, _CODES, ndim=6)
    _expect("scales", scales, (torch.float32,), ndim=6)
    _expect("cache_lengths", cache_lengths, _U32, ndim=1)
    _expect("lookup_table", lookup_table, _U32, ndim=2)
    _expect("scales_lookup_table", scales_lookup_table, _U32, ndim=2, optional=True)
    _expect("out", out, (torch.bfloat16,), ndim=4, last=512)
    _expect("lse", lse, (torch.float32,), ndim=3, optional=True)
    if cache_lengths.shape[0] != B or lookup_table.shape[0] != B:
        raise ValueError(f"cache_lengths and lookup_table must have {B} rows (one per request)")
    if scales_lookup_table is not None and tuple(scales_lookup_table.shape) != tuple(lookup_table.shape):
        raise ValueError("scales_lookup_table must have the shape of lookup_table")
    if tuple(out.shape) != (B, T, H, 512) or (lse is not None and tuple(lse.shape) != (B, T, H)):
        raise ValueError("out / lse shapes do not match q")
    host = [t for t in (q, cache_lengths, lookup_table, scales_lookup_table, out, lse) if t is not None]
    if any(t.device.type != "cpu" for t in host):
        raise ValueError("q, cache_lengths, the page tables, out and lse must be CPU tensors")
    _same_device(blocks, scales)
    lib = load()
    shp = paged_shape(B, H, blocks, scales, lookup_table)
    st = lib.mla_decode_paged_fp8_host(_ptr(q), _ptr(blocks), _ptr(scales), _ptr(cache_lengths), _ptr(lookup_table),
                                       _ptr(scales_lookup_table), int(max_prompt_length), int(max_cache_length),
                                       int(layer_idx), float(softmax_scale), ctypes.byref(shp), _ptr(out), _ptr(lse),
                                       int(variant), int(num_chunks), _stream(stream))
    _check(st)
    return out, lse


def kv_store(latent, cache_lengths, lookup_table, scales_lookup_table, layer_idx: int, blocks, scales,
             stream=None):
    """mla_kv_store_fp8 on torch tensors: quantise latent bf16 [B, T, 576] and write it in place into
    blocks / scales at positions cache_lengths[b] + i (page tables as for decode)."""
    _expect("latent", latent, (torch.bfloat16,), ndim=3, last=576)
    B, T, D = latent.shape
    _check_cache(blocks, scales, cache_lengths, lookup_table, scales_lookup_table, B)
    _same_device(latent, blocks, scales, cache_lengths, lookup_table, scales_lookup_table)
    lib = load()
    shp = paged_shape(B, 0, blocks, scales, lookup_table)
    st = lib.mla_kv_store_fp8(_ptr(latent), _ptr(cache_lengths), _ptr(lookup_table), _ptr(scales_lookup_table),
                              int(T), int(layer_idx), ctypes.byref(shp), _ptr(blocks), _ptr(scales), _stream(stream))
    _check(st)
    return blocks, scales


def decode_noalloc(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length: int,
                   max_cache_length: int, layer_idx: int, softmax_scale: float, out, lse, stream=None):
    """mla_decode_paged_fp8_noalloc: the decode on the library's fixed scratch (no device allocation).

    `out` and `lse` must be preallocated by the caller.
    """
    if out is None or lse is None:
        raise ValueError("decode_noalloc needs preallocated out and lse")
    _check_decode(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, out, lse)
    lib = load()
    B, T, H, D = q.shape
    shp = paged_shape(B, H, blocks, scales, lookup_table)
    st = lib.mla_decode_paged_fp8_noalloc(_ptr(q), _ptr(blocks), _ptr(scales), _ptr(cache_lengths),
                                          _ptr(lookup_table), _ptr(scales_lookup_table), int(max_prompt_length),
                                          int(max_cache_length), int(layer_idx), float(softmax_scale),
                                          ctypes.byref(shp), _ptr(out), _ptr(lse), _stream(stream))
    _check(st)
    return out, lse


def merge_parts(outs, lses, out=None, lse=None, stream=None):
    """mla_merge_lse_parts_bf16: outs bf16 [R, ..., 512] and lses fp32 [R, ...] (the parts' decode
    results over disjoint key ranges) -> (out bf16 [..., 512], lse fp32 [...])."""
    _expect("outs", outs, (torch.bfloat16,), last=512)
    _expect("lses", lses, (torch.float32,))
    if outs.dim() < 2 or outs.shape[:-1] != lses.shape:
        raise ValueError("outs must be [R, ..., 512] and lses [R, ...] with the same leading dims")
    _expect("out", out, (torch.bfloat16,), optional=True)
    _expect("lse", lse, (torch.float32,), optional=True)
    _same_device(outs, lses, out, lse)
    lib = load()
    R = outs.shape[0]
    rows = lses[0].numel()
    if out is None:
        out = torch.empty(outs.shape[1:], dtype=torch.bfloat16, device=outs.device)
    if lse is None:
        lse = torch.empty(lses.shape[1:], dtype=torch.float32, device=lses.device)
    _contig(out, lse)
    st = lib.mla_merge_lse_parts_bf16(_ptr(outs), _ptr(lses), int(R), int(rows), _ptr(out), _ptr(lse), _stream(stream))
    _check(st)
    return out, lse


def decode_inputs(inp, **kw):
    """decode() on a workloads.DecodeInputs bundle."""
    return decode(inp.q, inp.blocks, inp.scales, inp.cache_lengths, inp.lookup_table, inp.scales_lookup_table,
                  inp.max_prompt_length, inp.max_cache_length, inp.layer_idx, inp.softmax_scale, **kw)


def gather_dequant(blocks, scales, cache_lengths, lookup_table, scales_lookup_table, batch: int,
                   max_prompt_length: int, max_cache_length: int, layer_idx: int, max_keys: Optional[int] = None,
                   out_k=None, stream=None):
    """mla_gather_dequant_bf16: bf16 [B, max_keys, 576] of every stored key (rows past n_b untouched)."""
    _check_cache(blocks, scales, cache_lengths, lookup_table, scales_lookup_table, batch)
    if max_keys is None:
        max_keys = max_cache_length + max_prompt_length
    _expect("out_k", out_k, (torch.bfloat16,), ndim=3, last=576, optional=True)
    if out_k is not None and tuple(out_k.shape) != (batch, max_keys, 576):
        raise ValueError(f"out_k must be {(batch, max_keys, 576)} (got {tuple(out_k.shape)})")
    _same_device(blocks, scales, cache_lengths, lookup_table, scales_lookup_table, out_k)
    lib = load()
    if out_k is None:
        out_k = torch.zeros((batch, max_keys, 576), dtype=torch.bfloat16, device=blocks.device)
    shp = paged_shape(batch, 1, blocks, scales, lookup_table)
    st = lib.mla_gather_dequant_bf16(_ptr(blocks), _ptr(scales), _ptr(cache_lengths), _ptr(lookup_table),
                                     _ptr(scales_lookup_table), int(max_prompt_length), int(max_cache_length),
                                     int(layer_idx), ctypes.byref(shp), _ptr(out_k), int(max_keys), _stream(stream))
    _check(st)
    return out_k


def set_num_clusters(n: int):
    _check(load().mla_set_num_clusters(int(n)))


def set_wait_limit_ns(ns: int):
    """Bound of every wait inside the decode kernel (default 2 s)."""
    _check(load().mla_set_wait_limit_ns(int(ns)))


def withhold_arrival_once():
    """Test hook: the next decode call withholds one barrier arrival, so a bounded wait runs out."""
    _check(load().mla_debug_withhold_arrival_once())


def get_num_clusters() -> int:
    return int(load().mla_get_num_clusters())


def device_status(stream=None) -> int:
    """Synchronise, then return and clear the sticky device status (0 = OK)."""
    return int(load().mla_get_device_status(_stream(stream)))


def release_workspace():
    _check(load().mla_release_workspace())


def set_timing_events(before=None, after=None):
    """Record torch.cuda.Event `before`/`after` around every later decode-kernel launch (None, None stops)."""
    if before is not None and (before.cuda_event == 0 or after.cuda_event == 0):
        raise ValueError("record each event once before handing it to the library (torch creates it lazily)")
    b = None if before is None else ctypes.c_void_p(before.cuda_event)
    a = None if after is None else ctypes.c_void_p(after.cuda_event)
    _check(load().mla_set_timing_events(b, a))


def version() -> str:
    return load().mla_version().decode()

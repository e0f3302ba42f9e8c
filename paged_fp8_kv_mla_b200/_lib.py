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
            "mla_kv_store_fp8", "mla_decode_paged_fp8_scale_folded", "mla_merge_lse_parts_bf16"]


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


def decode(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, max_prompt_length: int,
           max_cache_length: int, layer_idx: int, softmax_scale: float, out=None, lse=None, stream=None,
           want_lse: bool = True, fold_scales: bool = False):
    """mla_decode_paged_fp8 on torch tensors (all on the current CUDA device).

    q bf16 [B, T, H, 576]; blocks uint8 [NB, kv_dim, L, P, 1, 576]; scales fp32 [NSB, kv_dim, L, P, 1, g];
    cache_lengths / lookup_table / scales_lookup_table int32 tensors holding uint32 values.
    fold_scales=True calls mla_decode_paged_fp8_scale_folded instead (g = 1 only).
    Returns (out bf16 [B, T, H, 512], lse fp32 [B, T, H] or None).
    """
    lib = load()
    B, T, H, D = q.shape
    _contig(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table)
    if out is None:
        out = torch.empty((B, T, H, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=q.device)
    shp = paged_shape(B, H, blocks, scales, lookup_table)
    fn = lib.mla_decode_paged_fp8_scale_folded if fold_scales else lib.mla_decode_paged_fp8
    st = fn(_ptr(q), _ptr(blocks), _ptr(scales), _ptr(cache_lengths), _ptr(lookup_table), _ptr(scales_lookup_table),
            int(max_prompt_length), int(max_cache_length), int(layer_idx), float(softmax_scale), ctypes.byref(shp),
            _ptr(out), _ptr(lse), _stream(stream))
    _check(st)
    return out, lse


def kv_store(latent, cache_lengths, lookup_table, scales_lookup_table, layer_idx: int, blocks, scales,
             stream=None):
    """mla_kv_store_fp8 on torch tensors: quantise latent bf16 [B, T, 576] and write it in place into
    blocks / scales at positions cache_lengths[b] + i (page tables as for decode)."""
    lib = load()
    B, T, D = latent.shape
    _contig(latent, blocks, scales, cache_lengths, lookup_table, scales_lookup_table)
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
    lib = load()
    B, T, H, D = q.shape
    _contig(q, blocks, scales, cache_lengths, lookup_table, scales_lookup_table, out, lse)
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
    lib = load()
    _contig(outs, lses)
    R = outs.shape[0]
    rows = lses[0].numel()
    if outs.shape[:-1] != lses.shape or outs.shape[-1] != 512:
        raise ValueError("outs must be [R, ..., 512] and lses [R, ...] with the same leading dims")
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
    lib = load()
    _contig(blocks, scales, cache_lengths, lookup_table, scales_lookup_table)
    if max_keys is None:
        max_keys = max_cache_length + max_prompt_length
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

"""CPU-side checks of the C-ABI library: it loads, exports every declared symbol, and rejects bad
arguments on the host before any CUDA work is enqueued."""
import ctypes
import os
import re

import pytest

import paged_fp8_kv_mla_b200 as M
from paged_fp8_kv_mla_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declarations_match_exports(lib):
    hdr = open(os.path.join(ROOT, "include", "mla_paged_fp8.h")).read()
    declared = set(re.findall(r"^\s*(?:mla_status_t|const char\*|int32_t)\s+(mla_\w+)\s*\(", hdr, re.M))
    assert declared == set(_lib.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_version(lib):
    assert re.match(r"\d+\.\d+\.\d+", M.version())


def _shape(**kw):
    base = dict(batch=2, num_q_heads=16, head_dim=576, v_dim=512, num_blocks=16, kv_dim=1, num_layers=1,
                page_size=16, num_kv_heads=1, num_scale_blocks=16, head_dim_granularity=1, max_pages=8)
    base.update(kw)
    return _lib.PagedShape(**base)


FAKE = ctypes.c_void_p(0x10000)     # 16-byte aligned, never dereferenced: validation fails first


def _call(lib, shape, q=FAKE, blocks=FAKE, scales=FAKE, lens=FAKE, lut=FAKE, slut=None, T=1, maxc=64, layer=0,
          out=FAKE):
    return lib.mla_decode_paged_fp8(q, blocks, scales, lens, lut, slut, T, maxc, layer, 0.07,
                                    ctypes.byref(shape) if shape is not None else None, out, None, None)


@pytest.mark.parametrize("kw,want", [
    (dict(head_dim=512), 2), (dict(v_dim=256), 2), (dict(num_kv_heads=2), 2),
    (dict(head_dim_granularity=72), 2), (dict(head_dim_granularity=5), 2), (dict(page_size=24), 2),
    (dict(num_layers=0), 1),
    (dict(max_pages=2), 1),
])
def test_host_validation_rejects_bad_shapes(lib, kw, want):
    assert _call(lib, _shape(**kw)) == want
    assert lib.mla_last_error_string().decode()


def test_host_validation_rejects_null_and_misaligned(lib):
    assert _call(lib, None) == 1
    assert _call(lib, _shape(), blocks=None) == 1
    assert _call(lib, _shape(), q=ctypes.c_void_p(0x10004)) == 1
    assert _call(lib, _shape(), layer=1) == 1
    assert _call(lib, _shape(), T=0) == 1


def test_scale_folded_host_validation(lib):
    """The scale-folding entry shares the decode's checks and takes only one scale per token; all of
    these fail on the host before anything is launched."""
    def fold(shape, **kw):
        a = dict(q=FAKE, blocks=FAKE, scales=FAKE, lens=FAKE, lut=FAKE, T=1, maxc=64, layer=0, out=FAKE)
        a.update(kw)
        return lib.mla_decode_paged_fp8_scale_folded(a["q"], a["blocks"], a["scales"], a["lens"], a["lut"], None,
                                                     a["T"], a["maxc"], a["layer"], 0.07,
                                                     ctypes.byref(shape) if shape is not None else None,
                                                     a["out"], None, None)
    assert fold(None) == 1
    assert fold(_shape(), blocks=None) == 1
    assert fold(_shape(head_dim=512)) == 2
    assert fold(_shape(head_dim_granularity=9)) == 2
    assert "one scale per token" in lib.mla_last_error_string().decode()


def test_merge_host_validation(lib):
    """Argument checks of the LSE merge; none of these launches anything (rows = 0 is a no-op)."""
    f = lib.mla_merge_lse_parts_bf16
    assert f(FAKE, FAKE, 2, 0, FAKE, None, None) == 0
    assert f(FAKE, FAKE, 0, 10, FAKE, None, None) == 1
    assert f(None, FAKE, 2, 10, FAKE, None, None) == 1
    assert f(FAKE, FAKE, 2, 10, ctypes.c_void_p(0x10004), None, None) == 1


def test_empty_batch_is_a_no_op_on_every_entry(lib):
    """batch = 0 (or no new tokens) returns MLA_OK after the host checks, before any CUDA call."""
    shp = _shape(batch=0)
    assert _call(lib, shp) == 0
    assert lib.mla_decode_paged_fp8_scale_folded(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 64, 0, 0.07,
                                                 ctypes.byref(shp), FAKE, None, None) == 0
    assert lib.mla_decode_paged_fp8_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 64, 0, 0.07,
                                            ctypes.byref(shp), FAKE, None, None) == 0
    assert lib.mla_gather_dequant_bf16(FAKE, FAKE, FAKE, FAKE, None, 1, 64, 0, ctypes.byref(shp), FAKE, 65,
                                       None) == 0
    assert _store(lib, _shape(batch=0)) == 0
    assert _store(lib, _shape(), T=0) == 0


def _store(lib, shape, latent=FAKE, lens=FAKE, lut=FAKE, slut=None, T=1, layer=0, blocks=FAKE, scales=FAKE):
    return lib.mla_kv_store_fp8(latent, lens, lut, slut, T, layer,
                                ctypes.byref(shape) if shape is not None else None, blocks, scales, None)


def test_kv_store_host_validation(lib):
    assert _store(lib, None) == 1
    assert _store(lib, _shape(), latent=None) == 1
    assert _store(lib, _shape(), blocks=None) == 1
    assert _store(lib, _shape(), latent=ctypes.c_void_p(0x10008)) == 1
    assert _store(lib, _shape(), layer=1) == 1
    assert _store(lib, _shape(head_dim=512)) == 2
    assert _store(lib, _shape(head_dim_granularity=9)) == 2
    assert _store(lib, _shape(num_kv_heads=2)) == 2
    # no new tokens: nothing to launch, nothing dereferenced
    assert _store(lib, _shape(), T=0) == 0
    assert _store(lib, _shape(batch=0)) == 0


def test_set_num_clusters_range(lib):
    assert lib.mla_set_num_clusters(-1) == 1
    assert lib.mla_set_num_clusters(0) == 0


def test_product_path_fails_loudly_without_library(tmp_path):
    saved = _lib._lib
    try:
        _lib._lib = None
        with pytest.raises(FileNotFoundError):
            _lib.load(str(tmp_path / "missing.so"))
    finally:
        _lib._lib = saved


def test_noalloc_rejects_more_items_than_its_fixed_scratch(lib):
    """The no-allocation entry holds its plan in a fixed array sized for 65 536 (request, query token,
    head group) items; one more is refused on the host with the reason, before any CUDA call."""
    heads = 128
    too_many = _shape(batch=65537, num_q_heads=heads, max_pages=8)

    def noalloc(shape, T=1):
        return lib.mla_decode_paged_fp8_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, T, 64, 0, 0.07,
                                                ctypes.byref(shape), FAKE, None, None)
    assert noalloc(too_many) == 2
    msg = lib.mla_last_error_string().decode()
    assert "65537" in msg and "65536" in msg
    # the same count reached through query tokens and head groups: 32769 * 2 tokens * 1 group
    assert noalloc(_shape(batch=32769, num_q_heads=heads, max_pages=8), T=2) == 2
    assert "65538" in lib.mla_last_error_string().decode()


def test_wait_limit_range(lib):
    """The decode kernel's wait bound is settable within [1 ms, 60 s] (host check only)."""
    assert lib.mla_set_wait_limit_ns(999_999) == 1
    assert lib.mla_set_wait_limit_ns(60_000_000_001) == 1
    assert lib.mla_set_wait_limit_ns(1_000_000) == 0
    assert lib.mla_set_wait_limit_ns(2_000_000_000) == 0


def test_host_buffer_entry_validation(lib):
    """mla_decode_paged_fp8_host checks everything on the host before any CUDA call: NULL host
    pointers, an unknown variant, a chunk count outside [0, 16], the shared shape checks, and the
    one-scale-per-token rule of its two variants; batch = 0 is a no-op."""
    def host(shape, variant=0, chunks=0, **kw):
        a = dict(q=FAKE, blocks=FAKE, scales=FAKE, lens=FAKE, lut=FAKE, out=FAKE, T=1, maxc=64, layer=0)
        a.update(kw)
        return lib.mla_decode_paged_fp8_host(a["q"], a["blocks"], a["scales"], a["lens"], a["lut"], None, a["T"],
                                             a["maxc"], a["layer"], 0.07,
                                             ctypes.byref(shape) if shape is not None else None, a["out"], None,
                                             variant, chunks, None)
    assert host(None) == 1
    assert host(_shape(), q=None) == 1
    assert host(_shape(), out=None) == 1
    assert host(_shape(), variant=3) == 1
    assert host(_shape(), variant=-1) == 1
    assert host(_shape(), chunks=17) == 1
    assert host(_shape(), chunks=-1) == 1
    assert host(_shape(), layer=1) == 1
    assert host(_shape(head_dim=512)) == 2
    assert host(_shape(head_dim_granularity=9), variant=2) == 2
    assert "one scale per token" in lib.mla_last_error_string().decode()
    assert host(_shape(batch=0)) == 0
    assert host(_shape(batch=0), variant=2, chunks=16) == 0


def test_binding_rejects_two_variants_at_once():
    """fold_scales and e4m3_pv select different kernels; asking for both is an argument error that
    the binding raises before touching any tensor."""
    import paged_fp8_kv_mla_b200 as M
    with pytest.raises(ValueError, match="at most one"):
        M.decode(None, None, None, None, None, None, 1, 64, 0, 0.07, fold_scales=True, e4m3_pv=True)

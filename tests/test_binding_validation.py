"""The Python binding checks what it hands to the untyped C ABI (dtype, rank, shape, contiguity,
device) and raises before any library call.  CPU tensors suffice: every check here fires before
the device check, except the last test, which is about the device check itself."""
import pytest
import torch

import paged_fp8_kv_mla_b200 as M


def _args(B=2, T=1, H=16, NB=8, P=16, pages=4, **over):
    a = dict(q=torch.zeros((B, T, H, 576), dtype=torch.bfloat16),
             blocks=torch.zeros((NB, 1, 1, P, 1, 576), dtype=torch.uint8),
             scales=torch.ones((NB, 1, 1, P, 1, 1), dtype=torch.float32),
             cache_lengths=torch.zeros(B, dtype=torch.int32),
             lookup_table=torch.zeros((B, pages), dtype=torch.int32),
             scales_lookup_table=None)
    a.update(over)
    return a


def _decode(a, **kw):
    return M.decode(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                    a["scales_lookup_table"], 1, 0, 0, 0.07, **kw)


@pytest.mark.parametrize("over,msg", [
    (dict(q=torch.zeros((2, 1, 16, 576), dtype=torch.float32)), "q must have dtype"),
    (dict(q=torch.zeros((2, 1, 16, 512), dtype=torch.bfloat16)), "last dim 576"),
    (dict(q=torch.zeros((2, 16, 576), dtype=torch.bfloat16)), "4-D"),
    (dict(blocks=torch.zeros((8, 1, 1, 16, 1, 576), dtype=torch.int8)), "blocks must have dtype"),
    (dict(scales=torch.ones((8, 1, 1, 16, 1, 1), dtype=torch.float16)), "scales must have dtype"),
    (dict(cache_lengths=torch.zeros(2, dtype=torch.int64)), "cache_lengths must have dtype"),
    (dict(cache_lengths=torch.zeros(3, dtype=torch.int32)), "rows"),
    (dict(lookup_table=torch.zeros((2, 4), dtype=torch.int64)), "lookup_table must have dtype"),
    (dict(scales_lookup_table=torch.zeros((2, 5), dtype=torch.int32)), "shape of lookup_table"),
    (dict(q=torch.zeros((2, 576, 16, 1), dtype=torch.bfloat16).transpose(1, 3)), "contiguous"),
])
def test_decode_rejects_bad_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        _decode(_args(**over))


def test_decode_rejects_bad_out_and_lse():
    a = _args()
    with pytest.raises(ValueError, match="out must be"):
        _decode(a, out=torch.zeros((2, 1, 8, 512), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="lse must have dtype"):
        _decode(a, lse=torch.zeros((2, 1, 16), dtype=torch.float64))


def test_kv_store_and_merge_and_gather_reject_bad_tensors():
    a = _args()
    with pytest.raises(ValueError, match="latent must have dtype"):
        M.kv_store(torch.zeros((2, 1, 576), dtype=torch.float32), a["cache_lengths"], a["lookup_table"], None, 0,
                   a["blocks"], a["scales"])
    with pytest.raises(ValueError, match="same leading dims"):
        M.merge_parts(torch.zeros((2, 4, 512), dtype=torch.bfloat16), torch.zeros((2, 5), dtype=torch.float32))
    with pytest.raises(ValueError, match="out_k must be"):
        M.gather_dequant(a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"], None, 2, 1, 10, 0,
                         out_k=torch.zeros((2, 5, 576), dtype=torch.bfloat16))


def test_host_tensors_are_rejected_before_the_library_is_called():
    with pytest.raises(ValueError, match="CUDA tensors"):
        _decode(_args())

"""Property-based checks (hypothesis) of the oracle's number formats and of the context-parallel
page split, over inputs the fixed-sample tests do not enumerate."""
import math

import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import context_parallel as CP

finite_f32 = st.floats(min_value=-1e4, max_value=1e4, allow_nan=False, allow_infinity=False, width=32)


@settings(max_examples=300, deadline=None)
@given(finite_f32)
def test_e4m3_encode_is_nearest_and_decodes_back(y):
    code = int(O.e4m3_encode_rn_sat(np.float32(y)))
    v = float(O.e4m3_decode(np.uint8(code)))
    a = min(abs(y), 448.0)
    # nearest: no finite code is strictly closer to the saturated value
    allv = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    allv = allv[np.isfinite(allv)]
    best = np.min(np.abs(np.abs(allv) - a))
    assert abs(abs(v) - a) <= best + 1e-12
    # sign kept (also for zero), and re-encoding the decoded value is the identity
    assert (code >> 7) == (1 if math.copysign(1.0, y) < 0 else 0)
    assert int(O.e4m3_encode_rn_sat(np.float32(v))) == code


@settings(max_examples=200, deadline=None)
@given(st.lists(st.integers(min_value=0, max_value=20000), min_size=1, max_size=12),
       st.sampled_from([16, 32, 48, 64, 128]), st.integers(min_value=1, max_value=9))
def test_context_parallel_ranges_cover_each_request_once(lengths, page, world):
    parts = CP.page_ranges(lengths, page, world)
    for b, L in enumerate(lengths):
        n = L + 1
        covered = 0
        prev_end = 0
        for first, count, keys in parts:
            if keys[b] == 0:
                continue
            start = first[b] * page
            assert start == prev_end                       # contiguous, in rank order
            assert start % page == 0                       # page aligned
            assert keys[b] <= count[b] * page
            prev_end = start + keys[b]
            covered += keys[b]
        assert covered == n and prev_end == n

"""Float64 CPU oracle for paged FP8-KV MLA decode (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg import
this package.  The product path never does.
"""
from .mla_oracle import (  # noqa: F401
    HEAD_DIM, V_DIM, INVALID_PAGE, e4m3_decode, bf16_round_f32, bf16_bits_to_f64,
    dequant_rows, num_keys, gather_request, dequant_request, attend, decode,
    attend_partial, combine,
)

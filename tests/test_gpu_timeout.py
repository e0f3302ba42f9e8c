"""The decode kernel's bounded waits, exercised on the GPU without a fault.

Every mbarrier wait inside the decode kernel gives up after the wait limit; the role that gives up
marks its CTA pair as aborted, every role drains its own copies and MMAs and returns, and the
status word reports a timeout.  A test hook makes one arrival go missing (the Q loader of one CTA
withholds its Q-ready arrival), with a short limit, so that the wait runs out; the device must stay
usable and the next ordinary call must match the oracle.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_mla_b200 as M
from oracle import mla_oracle as O
from paged_fp8_kv_mla_b200 import workloads as W
from tests.oracle_io import oracle_decode

pytestmark = pytest.mark.gpu

MLA_ERR_TIMEOUT = 5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_fp8_kv_mla_b200 import build
    build.build()
    M.load()
    M.set_num_clusters(0)
    yield
    M.set_wait_limit_ns(2_000_000_000)


def _parity(inp, out, lse):
    ref_out, ref_lse = oracle_decode(inp)
    o = O.bf16_bits_to_f64(out.cpu().view(torch.int16).numpy().view(np.uint16))
    assert np.abs(o - ref_out).max() <= 2e-2 * np.abs(ref_out).max() + 1e-2
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() <= 1e-3


@pytest.mark.parametrize("cfg_i", [0, 1])
def test_withheld_arrival_times_out_then_device_is_usable(cfg_i):
    inp = W.make_inputs(W.CONFIGS[cfg_i], device="cuda")
    assert M.device_status() == 0
    M.set_wait_limit_ns(20_000_000)          # 20 ms
    try:
        M.withhold_arrival_once()
        M.decode_inputs(inp)
        torch.cuda.synchronize()
        assert M.device_status() == MLA_ERR_TIMEOUT
    finally:
        M.set_wait_limit_ns(2_000_000_000)
    # the hook is one-shot: the next call is an ordinary decode on the same context
    out, lse = M.decode_inputs(inp)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    _parity(inp, out, lse)

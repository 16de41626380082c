"""Failure detection on the GPU without a fault: a kernel waits on an on-chip
barrier that nothing ever arrives on, with a 20 ms limit.  The wait must give
up, leave its location code (0x900) in the device error word and return, so
that sq_device_status reports SQ_ERR_TIMEOUT, the word is cleared by reading
it, and the context keeps working (a GEMM afterwards is still bit-exact).
"""
import time

import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import assert_bits_equal, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_int8_gemm_channel_b200 import _build

    _build.build()
    yield


def test_bounded_wait_times_out_and_context_survives(oracle):
    st, code = sq.sq_device_status()
    assert st == sq.SQ_OK, f"stale device error word {code:#x}"
    t0 = time.perf_counter()
    sq.sq_selftest_wait_timeout(20000)
    st, code = sq.sq_device_status()
    waited = time.perf_counter() - t0
    assert st == sq.SQ_ERR_TIMEOUT and code == 0x900, (st, hex(code))
    assert 0.015 < waited < 5.0, waited
    st, code = sq.sq_device_status()  # reading the word cleared it
    assert st == sq.SQ_OK and code == 0
    # the context is still usable
    M, N, K = 40, 272, 1040
    xq = wls.random_int8((M, K), seed=5)
    wq = wls.random_int8((N, K), seed=6)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq.cuda(), wq.cuda(), acc)
    assert_bits_equal(to_np(acc), oracle.gemm_i32(to_np(xq), to_np(wq)), "acc after the timeout")
    st, code = sq.sq_device_status()
    assert st == sq.SQ_OK, hex(code)

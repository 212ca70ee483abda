"""GPU test of failure detection without a GPU fault.

Every wait inside the library's kernels is bounded; when a bound runs out
the kernel records a timeout in the library's error word and returns, and
fp8bl_check() reports FP8BL_ERR_TIMEOUT.  fp8bl_selftest_wait_timeout runs
the same bounded waits (suspending and polling) on an mbarrier that nothing
ever arrives on, with a limit of about a millisecond: the test checks that
the status comes back, is cleared by the check, and that the device then
still runs the real kernels correctly.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import to_dev, u8, f32

pytestmark = pytest.mark.gpu

TIMEOUT = 6


@pytest.fixture(scope="module")
def fp8():
    import fine_grained_block_token_b200 as m
    return m


def _c(fp8):
    lib = ctypes.CDLL(fp8.lib_path)
    lib.fp8bl_selftest_wait_timeout.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
    lib.fp8bl_selftest_wait_timeout.restype = ctypes.c_int
    lib.fp8bl_check.argtypes = [ctypes.c_void_p]
    lib.fp8bl_check.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("kind", [0, 1])
def test_bounded_wait_reports_timeout_and_device_stays_usable(fp8, kind):
    lib = _c(fp8)
    st = torch.cuda.current_stream().cuda_stream
    assert lib.fp8bl_check(st) == 0                 # nothing pending
    assert lib.fp8bl_selftest_wait_timeout(1 << 21, kind, st) == 0
    assert lib.fp8bl_check(st) == TIMEOUT           # the wait ran out and said so
    assert lib.fp8bl_check(st) == 0                 # the check cleared it
    # the context is intact: a real quantization still matches the oracle
    bits = wl.normal((64, 1024), 1.0, 0, 7)
    q, s = fp8.quant_act(to_dev(bits))
    torch.cuda.synchronize()
    qo, so = oracle.quant_act(bits, nthreads=4)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(f32(s).view(np.uint32), so.view(np.uint32))
    assert lib.fp8bl_check(st) == 0

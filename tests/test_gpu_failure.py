"""Device-side failure detection without a GPU fault: a bounded wait that runs
out sets the library's error flag, the host reads FP8BS_ERR_TIMEOUT, and the
CUDA context stays usable (a GEMM right after is still correct)."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_11_b200 import build, inputs, ops

pytestmark = pytest.mark.gpu

TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    ops.lib()
    oracle.lib()


def selftest(limit_ns):
    fn = ops.lib().fp8bs_selftest_wait_timeout
    fn.argtypes = [ctypes.c_uint64, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(limit_ns, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_bounded_wait_reports_timeout_and_context_survives():
    assert ops.fp8bs_check_device_error() == 0          # flag starts clear
    t = time.time()
    assert selftest(50_000_000) == 0                    # 50 ms limit
    assert ops.fp8bs_check_device_error() == TIMEOUT
    assert time.time() - t < 5.0
    assert ops.fp8bs_check_device_error() == 0          # reading clears it
    # the context still works: a small GEMM against the oracle
    A = inputs.random_e4m3_bytes(128, 256, seed=1)
    B = inputs.random_e4m3_bytes(256, 256, seed=2)
    sa = torch.tensor([0.5], dtype=torch.float32)
    sb = torch.tensor([0.25], dtype=torch.float32)
    D = ops.fp8_scaled_gemm(A.cuda(), B.cuda(), sa.cuda(), sb.cuda(), ops.SCALE_TENSOR, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ops.fp8bs_check_device_error() == 0
    ref = oracle.gemm(A.numpy(), B.numpy(), sa.numpy(), sb.numpy(), oracle.SCALE_TENSOR)
    assert np.linalg.norm(D.cpu().numpy() - ref) <= 1e-5 * np.linalg.norm(ref)


def test_selftest_rejects_bad_limits():
    assert selftest(0) == 1
    assert selftest(20_000_000_000) == 1

"""fp8_quant_tensor_noalloc: per-tensor quantization for callers that cannot
allocate device memory where they call it (e.g. a plugin whose host framework
gives it no workspace).  It uses a fixed scratch array inside the library
instead of a caller-provided workspace; its results must equal the oracle's
per-tensor quantization and those of fp8_quant_tensor (bit for bit, the
tolerance every quantization test here uses) on consecutive calls, whatever
the previous call left in the scratch.

This file is collected last so that a failure here cannot hide any other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_11_b200 import build, inputs, ops
from parity import assert_bytes_equal, assert_scales_equal, bits

pytestmark = pytest.mark.gpu

WORKSPACE_ERR = 4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    ops.lib()
    oracle.lib()


def call_noalloc(x, q, s):
    """Straight through the C ABI: pointers, sizes and the current stream."""
    fn = ops.lib().fp8_quant_tensor_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    xt = 0 if x.dtype == torch.bfloat16 else 1
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(x.data_ptr(), xt, x.numel(), q.data_ptr(), s.data_ptr(), stream)


def _inputs(dtype):
    # first a tensor with a large amax spread over many CTAs' partials, then a
    # smaller tensor with a small amax: stale partials from call 1 would show up
    # as a wrong scale in call 2
    big = (inputs.random_matrix(4096, 4096, seed=21, dtype=torch.float32) * 50.0).to(dtype)
    small = (inputs.random_matrix(300, 1024, seed=22, dtype=torch.float32) * 0.01).to(dtype)
    return big, small


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_oracle_and_workspace_entry_point_on_consecutive_calls(dtype):
    for x in _inputs(dtype):
        xd = x.cuda()
        q = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
        s = torch.empty((1,), dtype=torch.float32, device="cuda")
        assert call_noalloc(xd, q, s) == 0
        q_ref, s_ref = ops.fp8_quant_tensor(xd)
        torch.cuda.synchronize()
        assert ops.fp8bs_check_device_error() == 0
        qo, so = oracle.quant_tensor(bits(x))
        assert_bytes_equal(q, qo, "noalloc bytes vs oracle")
        assert_scales_equal(s.cpu().numpy(), so, "noalloc scale vs oracle")
        assert torch.equal(q, q_ref)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("prealloc", [False, True])
def test_noalloc_python_wrapper(dtype, prealloc):
    """The binding's wrapper, with and without preallocated outputs, bit-exact
    against fp8_quant_tensor and the oracle on two calls in a row."""
    for x in _inputs(dtype):
        xd = x.cuda()
        if prealloc:
            q = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
            s = torch.empty((1,), dtype=torch.float32, device="cuda")
            q2, s2 = ops.fp8_quant_tensor_noalloc(xd, q=q, scale_inv=s)
            assert q2 is q and s2 is s
        else:
            q, s = ops.fp8_quant_tensor_noalloc(xd)
        q_ref, s_ref = ops.fp8_quant_tensor(xd)
        torch.cuda.synchronize()
        assert ops.fp8bs_check_device_error() == 0
        assert torch.equal(q, q_ref)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.cpu().numpy().view(np.uint32))
        qo, so = oracle.quant_tensor(bits(x))
        assert_bytes_equal(q, qo, "wrapper bytes vs oracle")


def test_noalloc_wrapper_rejects_what_it_cannot_copy():
    """No copy is possible without allocating: a non-contiguous view, a wrong
    output dtype or size, and outputs on the host are refused up front."""
    x = torch.randn(256, 512, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.fp8_quant_tensor_noalloc(x[:, :256])            # column slice of a wider matrix
    with pytest.raises(ValueError):
        ops.fp8_quant_tensor_noalloc(x.t())                  # transposed view
    with pytest.raises(ValueError):
        ops.fp8_quant_tensor_noalloc(x, q=torch.empty(x.shape, dtype=torch.int8, device="cuda"))
    with pytest.raises(ValueError):
        ops.fp8_quant_tensor_noalloc(x, q=torch.empty((100,), dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        ops.fp8_quant_tensor_noalloc(x, scale_inv=torch.empty((1,), dtype=torch.float32))
    with pytest.raises(ValueError):
        ops.fp8_quant_tensor_noalloc(x, scale_inv=torch.empty((1,), dtype=torch.float16, device="cuda"))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # validation happens before anything is read or launched: a 16-byte aligned
    # dummy pointer with an oversized element count is refused
    dummy = torch.empty((16,), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((16,), dtype=torch.uint8, device="cuda")
    s = torch.empty((1,), dtype=torch.float32, device="cuda")
    fn = ops.lib().fp8_quant_tensor_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    assert fn(dummy.data_ptr(), 0, (1 << 28) + 16, q.data_ptr(), s.data_ptr(), None) == WORKSPACE_ERR
    assert ops.fp8bs_status_string(WORKSPACE_ERR) == "FP8BS_ERR_WORKSPACE"

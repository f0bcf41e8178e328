"""GPU parity for the tcgen05 scaled GEMM against the CPU oracle.

fp32 output: relative Frobenius error <= 1e-5; bf16 output: per element
<= 2 bf16 ulp + 1e-6 * ||row||.  Operands are either random e4m3 codes with
random scales (the GEMM alone) or the workloads' seeded inputs quantized by
the GPU kernels and, independently, by the oracle (bit-exact, checked)."""
import math

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_11_b200 import build, inputs, ops
from fp8_block_scaled_11_b200.linear import Fp8LinearStep
from parity import assert_bf16_close, assert_bytes_equal, assert_f32_close, assert_scales_equal, bits, grid_np

pytestmark = pytest.mark.gpu

MODES = [ops.SCALE_TENSOR, ops.SCALE_ROWWISE, ops.SCALE_BLOCK_1x128_128x128, ops.SCALE_BLOCK_1x128_1x128]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    ops.lib()
    oracle.lib()


def no_device_error():
    st = ops.fp8bs_check_device_error()
    assert st == 0, ops.fp8bs_status_string(st)


def rand_scales(rng, shape):
    return (2.0 ** rng.uniform(-8, 0, size=shape)).astype(np.float32)


def make_scales(rng, mode, M, N, K):
    Kb = (K + 127) // 128
    if mode == ops.SCALE_TENSOR:
        return rand_scales(rng, (1,)), rand_scales(rng, (1,))
    if mode == ops.SCALE_ROWWISE:
        return rand_scales(rng, (M,)), rand_scales(rng, (N,))
    if mode == ops.SCALE_BLOCK_1x128_128x128:
        return rand_scales(rng, (M, Kb)), rand_scales(rng, ((N + 127) // 128, Kb))
    return rand_scales(rng, (M, Kb)), rand_scales(rng, (N, Kb))


def to_gpu_scales(s, mode):
    if mode in (ops.SCALE_TENSOR, ops.SCALE_ROWWISE):
        return torch.from_numpy(s).cuda()
    g = ops.colmajor_grid(s.shape[0], s.shape[1], "cuda")
    g.copy_(torch.from_numpy(s))
    return g


def run_random(M, N, K, mode, out_dtype, seed, rows=None, guard=False):
    rng = np.random.default_rng(seed)
    A = inputs.random_e4m3_bytes(M, K, seed=seed)
    B = inputs.random_e4m3_bytes(N, K, seed=seed + 1)
    sa, sb = make_scales(rng, mode, M, N, K)
    Ad, Bd = A.cuda(), B.cuda()
    sad, sbd = to_gpu_scales(sa, mode), to_gpu_scales(sb, mode)
    if guard:
        ldd = (N + 15) // 8 * 8 + 8
        buf = torch.full((M + 2, ldd), float("nan"), dtype=out_dtype, device="cuda")
        out = buf[:M, :N]
        D = ops.fp8_scaled_gemm(Ad, Bd, sad, sbd, mode, out=out)
    else:
        D = ops.fp8_scaled_gemm(Ad, Bd, sad, sbd, mode, out_dtype=out_dtype)
    torch.cuda.synchronize()
    no_device_error()
    if guard:
        g = buf.clone()
        g[:M, :N] = 0
        assert torch.isnan(g[M:]).all() and torch.isnan(g[:M, N:]).all(), "write outside the output view"
    ref = oracle.gemm(A.numpy(), B.numpy(), sa, sb, mode, rows=rows)
    got = D if rows is None else D[torch.as_tensor(rows, device="cuda")]
    if out_dtype == torch.float32:
        assert_f32_close(got, ref, f"M{M} N{N} K{K} mode{mode}")
    else:
        assert_bf16_close(got, ref, f"M{M} N{N} K{K} mode{mode}")
    return D


def test_gemm_single_tile_smoke():
    run_random(128, 256, 128, ops.SCALE_TENSOR, torch.float32, seed=1)
    run_random(128, 256, 128, ops.SCALE_BLOCK_1x128_128x128, torch.float32, seed=2)


SHAPES = [(128, 256, 256), (1, 1, 16), (16, 32, 32), (127, 129, 256), (129, 255, 384), (256, 512, 640),
          (300, 260, 1008), (64, 1000, 160), (513, 384, 2048)]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_shapes_fp32(M, N, K, mode):
    run_random(M, N, K, mode, torch.float32, seed=M * 7 + N * 3 + K + mode)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,N,K", [(129, 255, 384), (256, 512, 1024), (300, 264, 1008)])
def test_gemm_shapes_bf16_with_guard(M, N, K, mode):
    run_random(M, N, K, mode, torch.bfloat16, seed=M + N + K + mode, guard=True)


@pytest.mark.parametrize("mode", [ops.SCALE_BLOCK_1x128_128x128, ops.SCALE_BLOCK_1x128_1x128])
@pytest.mark.parametrize("kb", [1, 2, 3, 4, 5, 7, 64])
def test_gemm_k_blocks_small(kb, mode):
    run_random(256, 512, 128 * kb, mode, torch.float32, seed=kb + 10 * mode)


@pytest.mark.parametrize("mode", [ops.SCALE_BLOCK_1x128_128x128, ops.SCALE_BLOCK_1x128_1x128])
@pytest.mark.parametrize("kb", [1000, 1001, 1002, 1003])
def test_gemm_k_blocks_long(kb, mode):
    """Every k_blocks residue mod 4 at the long-K sizes (split-K path); sampled rows."""
    run_random(256, 512, 128 * kb, mode, torch.float32, seed=kb + mode, rows=[0, 1, 77, 128, 200, 255])


def test_gemm_deterministic_split_k():
    rng = np.random.default_rng(0)
    M, N, K = 256, 512, 128 * 1001
    A = inputs.random_e4m3_bytes(M, K, seed=3).cuda()
    B = inputs.random_e4m3_bytes(N, K, seed=4).cuda()
    sa, sb = make_scales(rng, 2, M, N, K)
    sad, sbd = to_gpu_scales(sa, 2), to_gpu_scales(sb, 2)
    D1 = ops.fp8_scaled_gemm(A, B, sad, sbd, 2, out_dtype=torch.float32)
    D2 = ops.fp8_scaled_gemm(A, B, sad, sbd, 2, out_dtype=torch.float32)
    D3 = ops.fp8_scaled_gemm(A, B, sad, sbd, 2, out_dtype=torch.float32, split_k=False)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.equal(D1, D2)
    rel = (D1 - D3).norm() / D3.norm()
    assert rel < 1e-6


# ------------------------------------------------------------------ workloads
def test_tiny_blockwise_workload():
    """A fp32 256x1024 (1x128), B fp32 1024x512 (128x128, as B^T), bf16 out."""
    A, Bt = inputs.tiny_blockwise()
    qa, sa = ops.fp8_quant_1x128(A.cuda())
    qb, sb, _, _ = ops.fp8_quant_128x128(Bt.cuda())
    D = ops.fp8_scaled_gemm(qa, qb, sa, sb, ops.SCALE_BLOCK_1x128_128x128)
    torch.cuda.synchronize()
    no_device_error()
    qao, sao = oracle.quant_1x128(bits(A))
    qbo, sbo = oracle.quant_128x128(bits(Bt))
    assert_bytes_equal(qa, qao)
    assert_scales_equal(grid_np(sa), sao)
    assert_bytes_equal(qb, qbo)
    assert_scales_equal(grid_np(sb), sbo)
    ref = oracle.gemm(qao, qbo, sao, sbo, oracle.SCALE_BLOCK_1x128_128x128)
    assert_bf16_close(D, ref, "tiny blockwise")
    fp32 = oracle.matmul_ref(bits(A), bits(Bt))
    assert oracle.sqnr(fp32, D.float().cpu().numpy()) >= 28.0


@pytest.mark.parametrize("rowwise", [False, True])
def test_per_tensor_workload(rowwise):
    """x bf16 256x1024, W bf16 4096x1024, out = x_q . W_q^T in bf16."""
    x, W = inputs.per_tensor()
    if rowwise:
        qx, sx = ops.fp8_quant_rowwise(x.cuda())
        qw, sw = ops.fp8_quant_rowwise(W.cuda())
        mode, omode = ops.SCALE_ROWWISE, oracle.SCALE_ROWWISE
        qxo, sxo = oracle.quant_rowwise(bits(x))
        qwo, swo = oracle.quant_rowwise(bits(W))
    else:
        qx, sx = ops.fp8_quant_tensor(x.cuda())
        qw, sw = ops.fp8_quant_tensor(W.cuda())
        mode, omode = ops.SCALE_TENSOR, oracle.SCALE_TENSOR
        qxo, sxo = oracle.quant_tensor(bits(x))
        qwo, swo = oracle.quant_tensor(bits(W))
    D = ops.fp8_scaled_gemm(qx, qw, sx, sw, mode)
    torch.cuda.synchronize()
    no_device_error()
    assert_bytes_equal(qx, qxo)
    assert_bytes_equal(qw, qwo)
    ref = oracle.gemm(qxo, qwo, sxo, swo, omode)
    assert_bf16_close(D, ref, "per-tensor" if not rowwise else "rowwise")
    # the page's own comparison: dequantized reference rounded to bf16, allclose at 1e-2
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16)
    assert torch.allclose(D.cpu(), ref_bf16, rtol=1e-2, atol=1e-2)


def test_tiny_tensorwise_fp32():
    """16x32x32 tensorwise, fp32 out (the shape an Inductor template got wrong)."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(16, 32, generator=g)
    w = torch.randn(32, 32, generator=g)
    qx, sx = ops.fp8_quant_tensor(x.cuda())
    qw, sw = ops.fp8_quant_tensor(w.cuda())
    D = ops.fp8_scaled_gemm(qx, qw, sx, sw, ops.SCALE_TENSOR, out_dtype=torch.float32)
    torch.cuda.synchronize()
    no_device_error()
    qxo, sxo = oracle.quant_tensor(bits(x))
    qwo, swo = oracle.quant_tensor(bits(w))
    ref = oracle.gemm(qxo, qwo, sxo, swo, oracle.SCALE_TENSOR)
    assert_f32_close(D, ref)
    assert torch.allclose(D.cpu().double(), torch.from_numpy(ref), atol=0.05, rtol=0.01)


@pytest.mark.parametrize("K", inputs.LONG_K_VALUES)
@pytest.mark.parametrize("recipe", ["1x128_128x128", "1x128_1x128"])
def test_long_k_workload(K, recipe):
    """grad_out^T (256 x K) . x (K x 512) at k_blocks 1000/1001/1002, bf16 out,
    sampled rows vs the oracle, SQNR >= 28 dB vs the unquantized fp64 matmul."""
    goT, x = inputs.long_k(K)
    goTd, xd = goT.cuda(), x.cuda()
    qa, sa = ops.fp8_quant_1x128(goTd)
    if recipe == "1x128_128x128":
        _, _, qb, sb = ops.fp8_quant_128x128(xd, want_q=False, want_qt=True)
        mode = ops.SCALE_BLOCK_1x128_128x128
    else:
        qb, sb = ops.fp8_quant_1x128(xd, transpose_out=True)
        mode = ops.SCALE_BLOCK_1x128_1x128
    D = ops.fp8_scaled_gemm(qa, qb, sa, sb, mode)
    D2 = ops.fp8_scaled_gemm(qa, qb, sa, sb, mode)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.equal(D, D2)
    rows = [0, 5, 64, 127, 128, 191, 255]
    qao, sao = oracle.quant_1x128(bits(goT), rows=rows)
    if recipe == "1x128_128x128":
        qbo, sbo = oracle.quant_128x128(bits(x), transpose=True)
    else:
        qbo, sbo = oracle.quant_1x128(bits(x), transpose=True)
    assert_bytes_equal(qb, qbo, "B^T bytes")
    assert_scales_equal(grid_np(sb), sbo, "B^T scales")
    assert_bytes_equal(qa[torch.as_tensor(rows, device="cuda")], qao, "A bytes")
    ref = oracle.gemm(qao, qbo, sao, sbo, mode)
    got = D[torch.as_tensor(rows, device="cuda")]
    assert_bf16_close(got, ref, f"long K={K} {recipe}")
    fp32 = oracle.matmul_ref(bits(goT[rows]), bits(x.t().contiguous()))
    assert oracle.sqnr(fp32, got.float().cpu().numpy()) >= 28.0


@pytest.mark.parametrize("wt_copy", [True, False])
@pytest.mark.parametrize("N,K", inputs.LLAMA4_SHAPES)
def test_llama4_fwd_bwd_workload(N, K, wt_copy):
    """The Llama4-shape linear fwd + bwd (M = 16640) at full size, in the
    launch configuration the benchmark times (wt_copy=False: dgrad reads W_q
    MN-major) and with dgrad reading the 128x128 kernel's transposed copy
    instead; sampled output rows of all three GEMMs and sampled quantized rows
    against the oracle."""
    M = inputs.LLAMA4_M
    x, W, dy = inputs.llama4(N, K)
    step = Fp8LinearStep(M, N, K, dgrad_wt_copy=wt_copy)
    xd, Wd, dyd = x.cuda(), W.cuda(), dy.cuda()
    y, dx, dW = step.run(xd, Wd, dyd)
    torch.cuda.synchronize()
    no_device_error()
    xb, Wb, dyb = bits(x), bits(W), bits(dy)
    rows_m = [0, 1, 2047, 8320, M - 1]
    rows_n = [0, 129, N // 2, N - 1]
    # forward: y = x W^T
    qxo, sxo = oracle.quant_1x128(xb, rows=rows_m)
    qwo, swo = oracle.quant_128x128(Wb)
    assert_bytes_equal(step.wq, qwo, "W_q")
    assert_scales_equal(grid_np(step.ws), swo, "W scales")
    assert_bytes_equal(step.xq[torch.as_tensor(rows_m, device="cuda")], qxo, "x_q rows")
    ref = oracle.gemm(qxo, qwo, sxo, swo, oracle.SCALE_BLOCK_1x128_128x128)
    assert_bf16_close(y[torch.as_tensor(rows_m, device="cuda")], ref, "fwd")
    # dgrad: dx = dy W  (B^T = W^T, the same 128x128 tiles; without the copy
    # the GPU reads W_q in its stored orientation)
    qdyo, sdyo = oracle.quant_1x128(dyb, rows=rows_m)
    qwto, swto = oracle.quant_128x128(Wb, transpose=True)
    if wt_copy:
        assert_bytes_equal(step.wtq, qwto, "W^T_q")
    else:
        assert step.wtq is None, "dgrad reads W_q without a transposed copy"
    ref = oracle.gemm(qdyo, qwto, sdyo, swto, oracle.SCALE_BLOCK_1x128_128x128)
    assert_bf16_close(dx[torch.as_tensor(rows_m, device="cuda")], ref, "dgrad")
    # wgrad: dW = dy^T x  (both quantized along tokens)
    qdyto, sdyto = oracle.quant_1x128(dyb, transpose=True, rows=rows_n)
    qxto, sxto = oracle.quant_1x128(xb, transpose=True)
    assert_bytes_equal(step.xtq, qxto, "x^T_q")
    assert_scales_equal(grid_np(step.xts), sxto, "x^T scales")
    assert_bytes_equal(step.dytq[torch.as_tensor(rows_n, device="cuda")], qdyto, "dy^T_q rows")
    ref = oracle.gemm(qdyto, qxto, sdyto, sxto, oracle.SCALE_BLOCK_1x128_1x128)
    assert_bf16_close(dW[torch.as_tensor(rows_n, device="cuda")], ref, "wgrad")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [129, 256, 257, 384, 512])
def test_gemm_several_tile_rows(M, mode):
    """Row counts above 128: several 128-row tiles, the last one partly past
    the last row."""
    run_random(M, 512, 384, mode, torch.float32, seed=M + 3 * mode)
    run_random(M, 264, 1024, mode, torch.bfloat16, seed=M + 5 * mode, guard=True)



@pytest.mark.parametrize("mode", [ops.SCALE_BLOCK_1x128_128x128, ops.SCALE_BLOCK_1x128_1x128])
@pytest.mark.parametrize("M,N,K", [(1280, 2056, 256), (200, 520, 64 * 128)])
def test_gemm_unaligned_output_pitch(M, N, K, mode):
    """bf16 output into a view whose row pitch (N + 3 elements) is not a
    multiple of 16 bytes, so every row is written element by element: by the
    GEMM's epilogue (first shape: 90 tiles, no split) and by the split-K
    reduction (second shape: 6 tiles, 64 K-blocks split 8 ways).  Parity on
    all rows; nothing written outside the view."""
    rng = np.random.default_rng(M + N)
    A = inputs.random_e4m3_bytes(M, K, seed=M)
    B = inputs.random_e4m3_bytes(N, K, seed=N)
    sa, sb = make_scales(rng, mode, M, N, K)
    buf = torch.full((M + 1, N + 3), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[:M, :N]
    ops.fp8_scaled_gemm(A.cuda(), B.cuda(), to_gpu_scales(sa, mode), to_gpu_scales(sb, mode), mode, out=out)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.isnan(buf[M:]).all() and torch.isnan(buf[:M, N:]).all(), "write outside the output view"
    assert_bf16_close(out, oracle.gemm(A.numpy(), B.numpy(), sa, sb, mode), f"pitch N+3 M{M} N{N} K{K}")


def test_llama4_forward_fp32_output_sampled():
    """The forward GEMM at full size (16640 x 5120 x 8192, 1x128 x 128x128) with
    fp32 output, in the benchmark's launch configuration: sampled rows from
    the first, middle and last tile rows against the oracle (relative
    Frobenius error <= 1e-5)."""
    M = inputs.LLAMA4_M
    x, W, _ = inputs.llama4(5120, 8192)
    xd, Wd = x.cuda(), W.cuda()
    qx, sx = ops.fp8_quant_1x128(xd)
    qw, sw, _, _ = ops.fp8_quant_128x128(Wd)
    D = ops.fp8_scaled_gemm(qx, qw, sx, sw, ops.SCALE_BLOCK_1x128_128x128, out_dtype=torch.float32)
    torch.cuda.synchronize()
    no_device_error()
    rows = [0, 77, 128, 8191, 8320, M - 129, M - 1]
    qxo, sxo = oracle.quant_1x128(bits(x), rows=rows)
    qwo, swo = oracle.quant_128x128(bits(W))
    ref = oracle.gemm(qxo, qwo, sxo, swo, oracle.SCALE_BLOCK_1x128_128x128)
    assert_f32_close(D[torch.as_tensor(rows, device="cuda")], ref, "fwd fp32 out")


@pytest.mark.parametrize("recipe", ["1x128_128x128", "1x128_1x128"])
def test_long_k_fp32_output(recipe):
    """The long-K case at k_blocks 1001 with fp32 output (split-K reduction
    writing fp32): sampled rows of both 128-row tiles against the oracle."""
    K = 128128
    goT, x = inputs.long_k(K)
    goTd, xd = goT.cuda(), x.cuda()
    qa, sa = ops.fp8_quant_1x128(goTd)
    if recipe == "1x128_128x128":
        _, _, qb, sb = ops.fp8_quant_128x128(xd, want_q=False, want_qt=True)
        mode = ops.SCALE_BLOCK_1x128_128x128
        qbo, sbo = oracle.quant_128x128(bits(x), transpose=True)
    else:
        qb, sb = ops.fp8_quant_1x128(xd, transpose_out=True)
        mode = ops.SCALE_BLOCK_1x128_1x128
        qbo, sbo = oracle.quant_1x128(bits(x), transpose=True)
    D = ops.fp8_scaled_gemm(qa, qb, sa, sb, mode, out_dtype=torch.float32)
    torch.cuda.synchronize()
    no_device_error()
    rows = [0, 5, 64, 127, 128, 191, 255]
    qao, sao = oracle.quant_1x128(bits(goT), rows=rows)
    assert_f32_close(D[torch.as_tensor(rows, device="cuda")], oracle.gemm(qao, qbo, sao, sbo, mode),
                     f"long K fp32 out {recipe}")


@pytest.mark.parametrize("mode", [ops.SCALE_TENSOR, ops.SCALE_ROWWISE, ops.SCALE_BLOCK_1x128_128x128])
@pytest.mark.parametrize("M,N,K", [(300, 264, 1024), (256, 1008, 640), (1280, 2056, 512)])
def test_gemm_quant_output(M, N, K, mode):
    """The GEMM with its bf16 output quantized 1x128 along N in the epilogue:
    D within the bf16 tolerance of the oracle, and the quantized bytes and
    scales bit-exact against the oracle's 1x128 quantization of the GPU's own D
    (N not a multiple of 128: a ragged last group; more tiles than SMs).  The
    same call without storing D gives the same bytes and scales."""
    rng = np.random.default_rng(M + N + K)
    A = inputs.random_e4m3_bytes(M, K, seed=M)
    B = inputs.random_e4m3_bytes(N, K, seed=N)
    sa, sb = make_scales(rng, mode, M, N, K)
    Ad, Bd, sad, sbd = A.cuda(), B.cuda(), to_gpu_scales(sa, mode), to_gpu_scales(sb, mode)
    D, q, s = ops.fp8_scaled_gemm_quant(Ad, Bd, sad, sbd, mode)
    D2, q2, s2 = ops.fp8_scaled_gemm_quant(Ad, Bd, sad, sbd, mode, store_out=False)
    torch.cuda.synchronize()
    no_device_error()
    assert D2 is None
    assert_bf16_close(D, oracle.gemm(A.numpy(), B.numpy(), sa, sb, mode), f"D M{M} N{N} K{K}")
    qo, so = oracle.quant_1x128(bits(D.cpu()))
    assert_bytes_equal(q, qo, "quantized output")
    assert_scales_equal(grid_np(s), so, "output scales")
    assert torch.equal(q, q2)
    assert_scales_equal(grid_np(s2), so, "output scales without D")
    if N % 16 == 0:
        # and equal to the separate quantization launch on D (which needs N % 16 == 0)
        q3, s3 = ops.fp8_quant_1x128(D)
        torch.cuda.synchronize()
        assert torch.equal(q, q3)
        assert_scales_equal(grid_np(s), grid_np(s3), "vs fp8_quant_1x128(D)")


# ------------------------------------------------------------------ B given MN-major (stored K x N)
def run_random_mn(M, N, K, mode, out_dtype, seed, rows=None):
    """D = A . B with B stored K x N (row pitch rounded up to 16 bytes) through
    fp8_scaled_gemm_ex(MAJOR_MN); the oracle gets B^T and the scale grid in
    its (n-block, k-block) order.  The GPU's 128x128 grid for B is the one of
    B's storage order, (k-block, n-block)."""
    rng = np.random.default_rng(seed)
    A = inputs.random_e4m3_bytes(M, K, seed=seed)
    B = inputs.random_e4m3_bytes(K, N, seed=seed + 1)
    sa, sb = make_scales(rng, mode, M, N, K)
    ldb = (N + 15) // 16 * 16
    Bbuf = torch.zeros((K, ldb), dtype=torch.uint8, device="cuda")
    Bbuf[:, :N] = B.cuda()
    Bd = Bbuf[:, :N]
    if mode == ops.SCALE_BLOCK_1x128_128x128:
        sbd = to_gpu_scales(np.ascontiguousarray(sb.T), mode)      # (Kb, Nb) grid
    else:
        sbd = to_gpu_scales(sb, mode)
    D = ops.fp8_scaled_gemm_ex(A.cuda(), Bd, ops.MAJOR_MN, to_gpu_scales(sa, mode), sbd, mode, out_dtype=out_dtype)
    torch.cuda.synchronize()
    no_device_error()
    ref = oracle.gemm(A.numpy(), np.ascontiguousarray(B.numpy().T), sa, sb, mode, rows=rows)
    got = D if rows is None else D[torch.as_tensor(rows, device="cuda")]
    if out_dtype == torch.float32:
        assert_f32_close(got, ref, f"MN-major B: M{M} N{N} K{K} mode{mode}")
    else:
        assert_bf16_close(got, ref, f"MN-major B: M{M} N{N} K{K} mode{mode}")


MN_MODES = [ops.SCALE_TENSOR, ops.SCALE_ROWWISE, ops.SCALE_BLOCK_1x128_128x128]


@pytest.mark.parametrize("mode", MN_MODES)
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 1, 16), (16, 32, 32), (127, 129, 256), (129, 255, 384),
                                   (300, 260, 1008), (64, 1000, 160), (513, 384, 2048)])
def test_gemm_b_mn_major_shapes(M, N, K, mode):
    """Ragged M, N and K (last K-block partial), several tiles, every recipe
    the MN-major form supports."""
    run_random_mn(M, N, K, mode, torch.float32, seed=3 * M + N + K + mode)
    run_random_mn(M, N, K, mode, torch.bfloat16, seed=5 * M + N + K + mode)


@pytest.mark.parametrize("mode", MN_MODES)
def test_gemm_b_mn_major_single_cta_split_k(mode):
    """60 output tiles, 16 K-blocks: the CTA-pair plan does not split K (too
    many pair tiles), the single-CTA plan splits it in two, so B is read
    MN-major by the single-CTA kernel with split-K partials and the reduction."""
    run_random_mn(1280, 1536, 2048, mode, torch.float32, seed=17 + mode, rows=list(range(0, 1280, 37)))


@pytest.mark.parametrize("kb", [1, 3, 64, 1001])
def test_gemm_b_mn_major_k_blocks(kb):
    """K-block counts up to the long-K case (split-K path at 1001)."""
    rows = [0, 1, 77, 128, 200, 255] if kb > 64 else None
    run_random_mn(256, 512, 128 * kb, ops.SCALE_BLOCK_1x128_128x128, torch.float32, seed=kb, rows=rows)


def test_gemm_b_mn_major_unsupported_recipe():
    A = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    B = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    s = ops.colmajor_grid(128, 2, "cuda").fill_(1.0)
    with pytest.raises(ops.Fp8bsError):
        ops.fp8_scaled_gemm_ex(A, B, ops.MAJOR_MN, s, s, ops.SCALE_BLOCK_1x128_1x128)


def test_dgrad_mn_major_equals_transposed_copy():
    """Llama4 dgrad (16640 x 8192 x 5120): reading W_q MN-major gives exactly
    the output of reading the 128x128 kernel's transposed copy K-major."""
    M = inputs.LLAMA4_M
    _, W, dy = inputs.llama4(5120, 8192)
    qdy, sdy = ops.fp8_quant_1x128(dy.cuda())
    qw, sw, qwt, swt = ops.fp8_quant_128x128(W.cuda(), want_q=True, want_qt=True)
    D_mn = ops.fp8_scaled_gemm_ex(qdy, qw, ops.MAJOR_MN, sdy, sw, ops.SCALE_BLOCK_1x128_128x128)
    D_k = ops.fp8_scaled_gemm(qdy, qwt, sdy, swt, ops.SCALE_BLOCK_1x128_128x128)
    torch.cuda.synchronize()
    no_device_error()
    assert D_mn.shape == (M, 8192)
    assert torch.equal(D_mn, D_k)

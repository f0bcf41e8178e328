"""GPU parity for the dynamic-quantization kernels: bytes and fp32 reciprocal
scales bit-exact against the CPU oracle, on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_11_b200 import build, inputs, ops
from parity import assert_bytes_equal, assert_scales_equal, bits, grid_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    ops.lib()
    oracle.lib()


def dev(x):
    return x.to("cuda")


def check_1x128(x_cpu, transpose=False, rows=None):
    q, s = ops.fp8_quant_1x128(dev(x_cpu), transpose_out=transpose)
    torch.cuda.synchronize()
    qo, so = oracle.quant_1x128(bits(x_cpu), transpose=transpose, rows=rows)
    if rows is None:
        assert_bytes_equal(q, qo, "q")
        assert_scales_equal(grid_np(s), so, "scale_inv")
    else:
        assert_bytes_equal(q[torch.as_tensor(rows, device="cuda")], qo, "q (sampled rows)")
        assert_scales_equal(grid_np(s)[rows], so, "scale_inv (sampled rows)")
    return q, s


SHAPES = [(256, 1024, torch.float32), (300, 400, torch.bfloat16), (1, 16, torch.bfloat16),
          (17, 2048, torch.float32), (1024, 1024, torch.bfloat16), (33, 144, torch.bfloat16)]


@pytest.mark.parametrize("R,C,dt", SHAPES)
def test_quant_1x128_rows(R, C, dt):
    check_1x128(inputs.random_matrix(R, C, seed=R + C, dtype=dt))


@pytest.mark.parametrize("R,C,dt", [(304, 400, torch.bfloat16), (256, 1024, torch.float32), (16, 16, torch.bfloat16),
                                    (1040, 272, torch.bfloat16), (128, 130 * 16, torch.float32)])
def test_quant_1x128_transposed(R, C, dt):
    check_1x128(inputs.random_matrix(R, C, seed=R * 3 + C, dtype=dt), transpose=True)


def check_dual(x_cpu):
    """fp8_quant_1x128_dual against the oracle's two 1x128 directions, and
    against the two single-direction launches, byte for byte."""
    xd = dev(x_cpu)
    q, s, qt, st = ops.fp8_quant_1x128_dual(xd)
    q1, s1 = ops.fp8_quant_1x128(xd)
    qt1, st1 = ops.fp8_quant_1x128(xd, transpose_out=True)
    torch.cuda.synchronize()
    xb = bits(x_cpu)
    qo, so = oracle.quant_1x128(xb)
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(grid_np(s), so, "scale_inv")
    qto, sto = oracle.quant_1x128(xb, transpose=True)
    assert_bytes_equal(qt, qto, "q_t")
    assert_scales_equal(grid_np(st), sto, "scale_inv_t")
    assert torch.equal(q, q1) and torch.equal(qt, qt1)
    assert_scales_equal(grid_np(s), grid_np(s1), "scale_inv vs single-direction launch")
    assert_scales_equal(grid_np(st), grid_np(st1), "scale_inv_t vs single-direction launch")


@pytest.mark.parametrize("R,C,dt", [(304, 400, torch.bfloat16), (256, 1024, torch.float32), (16, 16, torch.bfloat16),
                                    (1040, 272, torch.bfloat16), (128, 130 * 16, torch.float32),
                                    (400, 144, torch.float32), (2048, 1024, torch.bfloat16)])
def test_quant_1x128_dual(R, C, dt):
    """Both directions from one read: several tiles, ragged last tile row and
    column (sizes multiples of 16, not of 128), both input dtypes."""
    check_dual(inputs.random_matrix(R, C, seed=R * 5 + C, dtype=dt))


def test_quant_1x128_dual_special_values():
    """Groups whose row and column maxima differ by orders of magnitude inside
    one tile (zeros, +-0, 448 exactly, near-fp32-max, subnormal-range values),
    so that a row scale used for a column group (or the reverse) shows."""
    x = inputs.random_matrix(256, 384, seed=9, dtype=torch.float32)
    x[0, :128] = 0.0
    x[1, :128] = -0.0
    x[:, 5] = 0.0
    x[2, :] = 448.0
    x[:, 200] = 3.0e38
    x[3, 130:250] = 1e-30
    x[130:140, 300:310] = -2.0 ** -9
    check_dual(x)


def test_quant_1x128_dual_full_size_sampled():
    """The Llama4 activation (16640 x 8192 bf16) in the launch the linear
    step uses; sampled rows of the row direction and sampled rows of the
    transposed direction against the oracle."""
    x = inputs.llama4(5120, 8192)[0]
    xd = dev(x)
    q, s, qt, st = ops.fp8_quant_1x128_dual(xd)
    torch.cuda.synchronize()
    xb = bits(x)
    M, K = x.shape
    rows = [0, 1, 127, 128, M // 2 + 3, M - 1]
    qo, so = oracle.quant_1x128(xb, rows=rows)
    assert_bytes_equal(q[torch.as_tensor(rows, device="cuda")], qo, "q (sampled rows)")
    assert_scales_equal(grid_np(s)[rows], so, "scale_inv (sampled rows)")
    cols = [0, 5, 128, K // 2 + 1, K - 1]
    qto, sto = oracle.quant_1x128(xb, transpose=True, rows=cols)
    assert_bytes_equal(qt[torch.as_tensor(cols, device="cuda")], qto, "q_t (sampled rows)")
    assert_scales_equal(grid_np(st)[cols], sto, "scale_inv_t (sampled rows)")


@pytest.mark.parametrize("R,C,dt", [(304, 400, torch.bfloat16), (1024, 512, torch.float32), (16, 16, torch.bfloat16),
                                    (128, 128, torch.float32), (384, 1040, torch.bfloat16)])
def test_quant_128x128_with_transpose(R, C, dt):
    x = inputs.random_matrix(R, C, seed=R + 7 * C, dtype=dt)
    q, s, qt, st = ops.fp8_quant_128x128(dev(x), want_q=True, want_qt=True)
    torch.cuda.synchronize()
    qo, so = oracle.quant_128x128(bits(x))
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(grid_np(s), so, "scale_inv")
    qto, sto = oracle.quant_128x128(bits(x), transpose=True)
    assert_bytes_equal(qt, qto, "q_t")
    assert_scales_equal(grid_np(st), sto, "scale_inv_t")
    # the transposed output is the same tile bytes transposed, with the same scales
    assert torch.equal(qt.t(), q)
    assert np.array_equal(grid_np(st).T, grid_np(s))
    # only-transposed call gives the same bytes
    _, _, qt2, st2 = ops.fp8_quant_128x128(dev(x), want_q=False, want_qt=True)
    assert torch.equal(qt2, qt) and torch.equal(st2.cpu(), st.cpu())


@pytest.mark.parametrize("shape,dt", [((256, 1024), torch.bfloat16), ((4096, 1024), torch.bfloat16),
                                      ((1000, 16), torch.float32), ((1, 16), torch.bfloat16)])
def test_quant_tensor(shape, dt):
    x = inputs.random_matrix(*shape, seed=11, dtype=dt)
    q, s = ops.fp8_quant_tensor(dev(x))
    torch.cuda.synchronize()
    qo, so = oracle.quant_tensor(bits(x))
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(s.cpu().numpy(), so, "scale_inv")


@pytest.mark.parametrize("shape,dt", [((256, 1024), torch.bfloat16), ((4096, 1024), torch.bfloat16),
                                      ((37, 4112), torch.float32), ((1, 16), torch.bfloat16)])
def test_quant_rowwise(shape, dt):
    x = inputs.random_matrix(*shape, seed=12, dtype=dt)
    q, s = ops.fp8_quant_rowwise(dev(x))
    torch.cuda.synchronize()
    qo, so = oracle.quant_rowwise(bits(x))
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(s.cpu().numpy(), so, "scale_inv")


def test_per_tensor_workload():
    """Inputs of the per-tensor GEMM workload (256x1024 x, 4096x1024 W)."""
    x, W = inputs.per_tensor()
    for t in (x, W):
        q, s = ops.fp8_quant_tensor(dev(t))
        qr, sr = ops.fp8_quant_rowwise(dev(t))
        torch.cuda.synchronize()
        qo, so = oracle.quant_tensor(bits(t))
        assert_bytes_equal(q, qo)
        assert_scales_equal(s.cpu().numpy(), so)
        qro, sro = oracle.quant_rowwise(bits(t))
        assert_bytes_equal(qr, qro)
        assert_scales_equal(sr.cpu().numpy(), sro)


@pytest.mark.parametrize("n", inputs.QUANT_SWEEP_SIZES)
def test_quant_sweep_full_size(n):
    """The quantization sweep workload at its full sizes, in the launch
    configuration the benchmark times; full comparison up to 2048, sampled
    rows / row blocks above."""
    x = inputs.quant_sweep(n)
    xd = dev(x)
    xb = bits(x)
    q, s = ops.fp8_quant_1x128(xd)
    q2, s2, _, _ = ops.fp8_quant_128x128(xd)
    torch.cuda.synchronize()
    if n <= 2048:
        qo, so = oracle.quant_1x128(xb)
        assert_bytes_equal(q, qo)
        assert_scales_equal(grid_np(s), so)
        qo2, so2 = oracle.quant_128x128(xb)
        assert_bytes_equal(q2, qo2)
        assert_scales_equal(grid_np(s2), so2)
        return
    rows = sorted(set([0, 1, 127, 128, n // 2 + 5, n - 1] + list(range(37, n, n // 16))))
    qo, so = oracle.quant_1x128(xb, rows=rows)
    assert_bytes_equal(q[torch.as_tensor(rows, device="cuda")], qo)
    assert_scales_equal(grid_np(s)[rows], so)
    rbs = [0, n // 256, n // 128 - 1]
    qo2, so2 = oracle.quant_128x128(xb, rblocks=rbs)
    for i, rb in enumerate(rbs):
        assert_bytes_equal(q2[128 * rb:128 * rb + 128], qo2[128 * i:128 * i + 128])
    assert_scales_equal(grid_np(s2)[rbs], so2)


def test_special_values():
    """amax exactly 448 (s = 1), negative underflow to -0 (0x80), all-zero
    groups, subnormal-producing values, and huge dynamic range in one group."""
    C = 512
    x = inputs.random_matrix(16, C, seed=5, dtype=torch.float32)
    x[0, :128] = 0.0
    x[0, 128:256] = -0.0
    x[1, :] = torch.linspace(-448, 448, C)
    x[2, :128] = 1e-30
    x[2, 0] = 1.0
    x[2, 1:64] = -1e-6
    x[3, 128:256] = 3.0e38 * torch.sign(torch.randn(128))
    x[3, 130] = 1e-38
    x[4, :] = 448.0
    x[5, 256:384] = torch.arange(128, dtype=torch.float32) * 2.0 ** -12
    for tr in (False, True):
        check_1x128(x, transpose=tr)
    q, s, qt, st = ops.fp8_quant_128x128(dev(x[:, :256].contiguous().repeat(16, 1)), want_qt=True)
    torch.cuda.synchronize()
    qo, so = oracle.quant_128x128(bits(x[:, :256].contiguous().repeat(16, 1)))
    assert_bytes_equal(q, qo)
    assert_scales_equal(grid_np(s), so)


def test_cvt_exhaustive_unit_scale():
    """Every fp32 bit pattern of magnitude <= 448 goes through the 1x128 kernel
    in a group whose amax is 448 (so s = 1 and q = e4m3(x)), signs alternating
    by row; compared with the oracle's encoder byte for byte."""
    top = 0x43E00000                      # bits of 448.0
    per_row = 127
    chunk_rows = 1 << 19
    start = 0
    while start <= top:
        n = min(chunk_rows * per_row, top + 1 - start)
        pats = np.arange(start, start + n, dtype=np.uint64).astype(np.uint32)
        rows = (n + per_row - 1) // per_row
        body = np.zeros(rows * per_row, dtype=np.uint32)
        body[:n] = pats
        body = body.reshape(rows, per_row)
        body[1::2] |= np.uint32(0x80000000)              # negative on odd rows
        vals = body.view(np.float32)
        x = np.empty((rows, 128), dtype=np.float32)
        x[:, 0] = 448.0
        x[:, 1:] = vals
        q, s = ops.fp8_quant_1x128(torch.from_numpy(x).cuda())
        want = oracle.e4m3_encode(x)
        got = q.cpu().numpy()
        assert np.all(grid_np(s) == 1.0)
        if not np.array_equal(got, want):
            i = tuple(np.argwhere(got != want)[0])
            raise AssertionError(f"pattern {x.view(np.uint32)[i]:#010x}: gpu {got[i]:#04x} oracle {want[i]:#04x}")
        start += n

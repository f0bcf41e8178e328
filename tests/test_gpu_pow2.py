"""GPU parity for the power-of-two scale rule and the block-scaled MMA GEMM
(the fast-accumulation variant of pytorch/pytorch issue #159940, Describe the
bug: USE_FAST_ACCUM, in its B200 form).

* quantization with SCALE_RULE_POW2: bytes and scales bit-exact against the
  oracle under oracle.scale_rule(SCALE_RULE_POW2);
* GEMM recipes SCALE_BLOCK_*_POW2: the oracle's GEMM of the same recipe (the
  sum is the same; only the scales are restricted), within the method's
  tolerances (fp32 out: relative Frobenius <= 1e-5; bf16 out: 2 bf16 ulp +
  1e-6 * ||row||), and SQNR >= 28 dB against the unquantized matmul at
  k_blocks 1000 / 1001 / 1002;
* a scale that is not a power of two is reported (FP8BS_ERR_SCALE)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_11_b200 import build, inputs, ops
from parity import assert_bf16_close, assert_bytes_equal, assert_f32_close, assert_scales_equal, bits, grid_np

pytestmark = pytest.mark.gpu

POW2_MODES = [ops.SCALE_BLOCK_1x128_128x128_POW2, ops.SCALE_BLOCK_1x128_1x128_POW2]
BASE_MODE = {ops.SCALE_BLOCK_1x128_128x128_POW2: ops.SCALE_BLOCK_1x128_128x128,
             ops.SCALE_BLOCK_1x128_1x128_POW2: ops.SCALE_BLOCK_1x128_1x128}
FP8BS_ERR_SCALE = 8


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


# ------------------------------------------------------------------ quantization
@pytest.mark.parametrize("R,C,dt,transpose", [(300, 400, torch.bfloat16, False), (256, 1024, torch.float32, False),
                                              (33, 144, torch.bfloat16, False), (1040, 272, torch.bfloat16, True),
                                              (128, 130 * 16, torch.float32, True)])
def test_quant_1x128_pow2(R, C, dt, transpose):
    x = inputs.random_matrix(R, C, seed=R + 5 * C, dtype=dt)
    q, s = ops.fp8_quant_1x128(x.cuda(), transpose_out=transpose, rule=ops.SCALE_RULE_POW2)
    torch.cuda.synchronize()
    with oracle.scale_rule(oracle.SCALE_RULE_POW2):
        qo, so = oracle.quant_1x128(bits(x), transpose=transpose)
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(grid_np(s), so, "scale_inv")


@pytest.mark.parametrize("R,C,dt", [(304, 400, torch.bfloat16), (256, 1024, torch.float32)])
def test_quant_dual_pow2(R, C, dt):
    x = inputs.random_matrix(R, C, seed=3 * R + C, dtype=dt)
    q, s, qt, st = ops.fp8_quant_1x128_dual(x.cuda(), rule=ops.SCALE_RULE_POW2)
    torch.cuda.synchronize()
    with oracle.scale_rule(oracle.SCALE_RULE_POW2):
        qo, so = oracle.quant_1x128(bits(x))
        qto, sto = oracle.quant_1x128(bits(x), transpose=True)
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(grid_np(s), so, "scale_inv")
    assert_bytes_equal(qt, qto, "q_t")
    assert_scales_equal(grid_np(st), sto, "scale_inv_t")


@pytest.mark.parametrize("R,C,dt", [(300, 400, torch.bfloat16), (512, 256, torch.float32), (16, 144, torch.bfloat16)])
def test_quant_128x128_pow2(R, C, dt):
    R16 = (R + 15) // 16 * 16
    x = inputs.random_matrix(R16, C, seed=R + C, dtype=dt)
    q, s, qt, st = ops.fp8_quant_128x128(x.cuda(), want_q=True, want_qt=True, rule=ops.SCALE_RULE_POW2)
    torch.cuda.synchronize()
    with oracle.scale_rule(oracle.SCALE_RULE_POW2):
        qo, so = oracle.quant_128x128(bits(x))
        qto, sto = oracle.quant_128x128(bits(x), transpose=True)
    assert_bytes_equal(q, qo, "q")
    assert_scales_equal(grid_np(s), so, "scale_inv")
    assert_bytes_equal(qt, qto, "q_t")
    assert_scales_equal(grid_np(st), sto, "scale_inv_t")


def test_pow2_scales_bound_the_fp32_scales():
    """r_pow2 is a power of two with r_fp32 <= r_pow2 < 2 r_fp32 (the scale is
    rounded down to a power of two, its reciprocal up), group by group."""
    x = inputs.random_matrix(512, 1024, seed=11, dtype=torch.bfloat16).cuda()
    _, s32 = ops.fp8_quant_1x128(x)
    _, s2 = ops.fp8_quant_1x128(x, rule=ops.SCALE_RULE_POW2)
    torch.cuda.synchronize()
    a, b = grid_np(s32).astype(np.float64), grid_np(s2).astype(np.float64)
    m, _ = np.frexp(b)
    assert np.all(m == 0.5)
    assert np.all(b >= a) and np.all(b < 2 * a)


# ------------------------------------------------------------------ GEMM
def pow2_scales(rng, shape):
    return (2.0 ** rng.integers(-9, 1, size=shape)).astype(np.float32)


def to_grid(s):
    g = ops.colmajor_grid(s.shape[0], s.shape[1], "cuda")
    g.copy_(torch.from_numpy(s))
    return g


def run_random_pow2(M, N, K, mode, out_dtype, seed, rows=None, guard=False, split_k=True):
    rng = np.random.default_rng(seed)
    Kb = (K + 127) // 128
    A = inputs.random_e4m3_bytes(M, K, seed=seed)
    B = inputs.random_e4m3_bytes(N, K, seed=seed + 1)
    sa = pow2_scales(rng, (M, Kb))
    sb = pow2_scales(rng, (((N + 127) // 128) if mode == ops.SCALE_BLOCK_1x128_128x128_POW2 else N, Kb))
    Ad, Bd, sad, sbd = A.cuda(), B.cuda(), to_grid(sa), to_grid(sb)
    if guard:
        ldd = (N + 15) // 8 * 8 + 8
        buf = torch.full((M + 2, ldd), float("nan"), dtype=out_dtype, device="cuda")
        out = buf[:M, :N]
        D = ops.fp8_scaled_gemm(Ad, Bd, sad, sbd, mode, out=out, split_k=split_k)
    else:
        D = ops.fp8_scaled_gemm(Ad, Bd, sad, sbd, mode, out_dtype=out_dtype, split_k=split_k)
    torch.cuda.synchronize()
    no_device_error()
    if guard:
        g = buf.clone()
        g[:M, :N] = 0
        assert torch.isnan(g[M:]).all() and torch.isnan(g[:M, N:]).all(), "write outside the output view"
    ref = oracle.gemm(A.numpy(), B.numpy(), sa, sb, BASE_MODE[mode], rows=rows)
    got = D if rows is None else D[torch.as_tensor(rows, device="cuda")]
    if out_dtype == torch.float32:
        assert_f32_close(got, ref, f"M{M} N{N} K{K} mode{mode}")
    else:
        assert_bf16_close(got, ref, f"M{M} N{N} K{K} mode{mode}")
    return D


def test_gemm_pow2_single_tile_smoke():
    run_random_pow2(128, 256, 128, ops.SCALE_BLOCK_1x128_128x128_POW2, torch.float32, seed=1)
    run_random_pow2(128, 256, 128, ops.SCALE_BLOCK_1x128_1x128_POW2, torch.float32, seed=2)


SHAPES = [(128, 256, 256), (1, 1, 16), (16, 32, 32), (127, 129, 256), (129, 255, 384), (256, 512, 640),
          (300, 260, 1008), (64, 1000, 160), (513, 384, 2048)]


@pytest.mark.parametrize("mode", POW2_MODES)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_pow2_shapes_fp32(M, N, K, mode):
    run_random_pow2(M, N, K, mode, torch.float32, seed=M * 7 + N * 3 + K + mode)


@pytest.mark.parametrize("mode", POW2_MODES)
@pytest.mark.parametrize("M,N,K", [(129, 255, 384), (256, 512, 1024), (300, 264, 1008)])
def test_gemm_pow2_shapes_bf16_with_guard(M, N, K, mode):
    run_random_pow2(M, N, K, mode, torch.bfloat16, seed=M + N + K + mode, guard=True)


@pytest.mark.parametrize("mode", POW2_MODES)
@pytest.mark.parametrize("kb", [1, 2, 3, 4, 5, 7, 8, 9, 64])
def test_gemm_pow2_k_blocks_small(kb, mode):
    """K-block counts around the four-K-block scale-factor stages, with and
    without split-K."""
    run_random_pow2(256, 512, 128 * kb, mode, torch.float32, seed=kb + 10 * mode)
    run_random_pow2(256, 512, 128 * kb, mode, torch.float32, seed=kb + 10 * mode + 1, split_k=False)


@pytest.mark.parametrize("mode", POW2_MODES)
@pytest.mark.parametrize("kb", [1000, 1001, 1002, 1003])
def test_gemm_pow2_k_blocks_long(kb, mode):
    """Every k_blocks residue mod 4 at the long-K sizes (split-K); sampled rows."""
    run_random_pow2(256, 512, 128 * kb, mode, torch.float32, seed=kb + mode, rows=[0, 1, 77, 128, 200, 255])


def test_gemm_pow2_full_tile_grid():
    """Several waves of persistent tiles (more tiles than SMs), bf16 out."""
    run_random_pow2(2048, 4096, 512, ops.SCALE_BLOCK_1x128_128x128_POW2, torch.bfloat16, seed=7,
                    rows=list(range(0, 2048, 97)))


@pytest.mark.parametrize("K", [128000, 128128, 128256])
@pytest.mark.parametrize("recipe", ["1x128_128x128", "1x128_1x128"])
def test_long_k_workload_pow2(K, recipe):
    """The long-K workload quantized with the power-of-two rule: quantized
    operands against the oracle, the GEMM against the oracle's GEMM on them,
    SQNR >= 28 dB against the unquantized fp64 matmul (sampled rows)."""
    goT, x = inputs.long_k(K)
    goTd, xd = goT.cuda(), x.cuda()
    P = ops.SCALE_RULE_POW2
    qa, sa = ops.fp8_quant_1x128(goTd, rule=P)
    if recipe == "1x128_128x128":
        _, _, qb, sb = ops.fp8_quant_128x128(xd, want_q=False, want_qt=True, rule=P)
        mode = ops.SCALE_BLOCK_1x128_128x128_POW2
    else:
        qb, sb = ops.fp8_quant_1x128(xd, transpose_out=True, rule=P)
        mode = ops.SCALE_BLOCK_1x128_1x128_POW2
    D = ops.fp8_scaled_gemm(qa, qb, sa, sb, mode)
    D2 = ops.fp8_scaled_gemm(qa, qb, sa, sb, mode)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.equal(D, D2)
    rows = [0, 5, 64, 127, 128, 191, 255]
    with oracle.scale_rule(oracle.SCALE_RULE_POW2):
        qao, sao = oracle.quant_1x128(bits(goT), rows=rows)
        if recipe == "1x128_128x128":
            qbo, sbo = oracle.quant_128x128(bits(x), transpose=True)
        else:
            qbo, sbo = oracle.quant_1x128(bits(x), transpose=True)
    assert_bytes_equal(qb, qbo, "B^T bytes")
    assert_scales_equal(grid_np(sb), sbo, "B^T scales")
    assert_bytes_equal(qa[torch.as_tensor(rows, device="cuda")], qao, "A bytes")
    ref = oracle.gemm(qao, qbo, sao, sbo, BASE_MODE[mode])
    got = D[torch.as_tensor(rows, device="cuda")]
    assert_bf16_close(got, ref, f"long K={K} {recipe}")
    fp32 = oracle.matmul_ref(bits(goT[rows]), bits(x.t().contiguous()))
    assert oracle.sqnr(fp32, got.float().cpu().numpy()) >= 28.0


def test_llama4_forward_pow2():
    """The Llama4 forward GEMM 16640 x 5120 x 8192 with power-of-two scales at
    full size (the launch configuration the ablation times): sampled rows of
    the quantized activations and of the output against the oracle."""
    M, (N, K) = inputs.LLAMA4_M, inputs.LLAMA4_SHAPES[0]
    x = inputs.random_matrix(M, K, seed=41, dtype=torch.bfloat16)
    W = inputs.random_matrix(N, K, seed=42, dtype=torch.bfloat16)
    P = ops.SCALE_RULE_POW2
    xq, xs = ops.fp8_quant_1x128(x.cuda(), rule=P)
    wq, ws, _, _ = ops.fp8_quant_128x128(W.cuda(), rule=P)
    D = ops.fp8_scaled_gemm(xq, wq, xs, ws, ops.SCALE_BLOCK_1x128_128x128_POW2)
    torch.cuda.synchronize()
    no_device_error()
    rows = [0, 1, 127, 128, 5000, 9999, 16511, 16639]
    with oracle.scale_rule(oracle.SCALE_RULE_POW2):
        qxo, sxo = oracle.quant_1x128(bits(x), rows=rows)
        qwo, swo = oracle.quant_128x128(bits(W))
    r = torch.as_tensor(rows, device="cuda")
    assert_bytes_equal(xq[r], qxo, "x bytes")
    assert_scales_equal(grid_np(xs)[rows], sxo, "x scales")
    assert_bytes_equal(wq, qwo, "W bytes")
    assert_scales_equal(grid_np(ws), swo, "W scales")
    ref = oracle.gemm(qxo, qwo, sxo, swo, ops.SCALE_BLOCK_1x128_128x128)
    assert_bf16_close(D[r], ref, "Llama4 forward, power-of-two scales")


# ------------------------------------------------------------------ errors
@pytest.mark.parametrize("bad", [0.3, 0.0, -0.5, float("inf")])
def test_gemm_pow2_reports_non_power_of_two_scales(bad):
    """A scale that is not a positive normal power of two sets the device error
    flag, read back as FP8BS_ERR_SCALE; the flag is cleared by the read."""
    rng = np.random.default_rng(5)
    M, N, K = 256, 512, 512
    A = inputs.random_e4m3_bytes(M, K, seed=8).cuda()
    B = inputs.random_e4m3_bytes(N, K, seed=9).cuda()
    sa = pow2_scales(rng, (M, 4))
    sb = pow2_scales(rng, (4, 4))
    sa[17, 2] = bad
    ops.fp8_scaled_gemm(A, B, to_grid(sa), to_grid(sb), ops.SCALE_BLOCK_1x128_128x128_POW2)
    assert ops.fp8bs_check_device_error() == FP8BS_ERR_SCALE
    no_device_error()


def test_gemm_pow2_unsupported_forms():
    A = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
    s = ops.colmajor_grid(256, 2, "cuda").fill_(1.0)
    sb = ops.colmajor_grid(2, 2, "cuda").fill_(1.0)
    with pytest.raises(ops.Fp8bsError):
        ops.fp8_scaled_gemm_ex(A, A, ops.MAJOR_MN, s, sb, ops.SCALE_BLOCK_1x128_128x128_POW2)
    with pytest.raises(ops.Fp8bsError):
        ops.fp8_scaled_gemm_quant(A, A, s, sb, ops.SCALE_BLOCK_1x128_128x128_POW2)


@pytest.mark.parametrize("K", [8192, 32768, 128128])
def test_whole_k_accumulation_error_bound(K):
    """The accuracy cost of the fast-accumulation variant: one unit's whole K
    range accumulated in TMEM (split-K off) loses at most about one fp32 unit
    roundoff per 32-wide MMA step, relative Frobenius error <= (K/32) * 2^-23
    against the oracle, while the promoted recipe on the same power-of-two
    operands stays within the method's 1e-5."""
    rng = np.random.default_rng(K)
    M, N = 256, 512
    Kb = (K + 127) // 128
    A = inputs.random_e4m3_bytes(M, K, seed=1)
    B = inputs.random_e4m3_bytes(N, K, seed=2)
    sa, sb = pow2_scales(rng, (M, Kb)), pow2_scales(rng, ((N + 127) // 128, Kb))
    rows = [0, 1, 100, 255]
    ref = oracle.gemm(A.numpy(), B.numpy(), sa, sb, ops.SCALE_BLOCK_1x128_128x128, rows=rows)
    r = torch.as_tensor(rows, device="cuda")
    Ad, Bd = A.cuda(), B.cuda()
    fast = ops.fp8_scaled_gemm(Ad, Bd, to_grid(sa), to_grid(sb), ops.SCALE_BLOCK_1x128_128x128_POW2,
                               out_dtype=torch.float32, split_k=False)
    prom = ops.fp8_scaled_gemm(Ad, Bd, to_grid(sa), to_grid(sb), ops.SCALE_BLOCK_1x128_128x128,
                               out_dtype=torch.float32, split_k=False)
    torch.cuda.synchronize()
    no_device_error()
    rel = lambda D: np.linalg.norm(D[r].double().cpu().numpy() - ref) / np.linalg.norm(ref)
    assert rel(fast) <= (K / 32) * 2.0 ** -23, rel(fast)
    assert rel(prom) <= 1e-5, rel(prom)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M,N,K", [(1200, 1500, 512), (256, 600, 8192)])
def test_gemm_pow2_unaligned_output_pitch(M, N, K, dtype):
    """Output into a view whose row pitch (N + 3 elements) is not a multiple
    of 16 bytes, so every row is written element by element: by the block-
    scaled kernel's epilogue (first shape: 60 tiles, no split) and by the
    split-K reduction (second shape: 6 tiles, 64 K-blocks split).  Parity on
    all rows; nothing written outside the view."""
    rng = np.random.default_rng(M + N + K)
    Kb = (K + 127) // 128
    A = inputs.random_e4m3_bytes(M, K, seed=M)
    B = inputs.random_e4m3_bytes(N, K, seed=N)
    sa, sb = pow2_scales(rng, (M, Kb)), pow2_scales(rng, ((N + 127) // 128, Kb))
    buf = torch.full((M + 1, N + 3), float("nan"), dtype=dtype, device="cuda")
    out = buf[:M, :N]
    ops.fp8_scaled_gemm(A.cuda(), B.cuda(), to_grid(sa), to_grid(sb), ops.SCALE_BLOCK_1x128_128x128_POW2, out=out)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.isnan(buf[M:]).all() and torch.isnan(buf[:M, N:]).all(), "write outside the output view"
    ref = oracle.gemm(A.numpy(), B.numpy(), sa, sb, ops.SCALE_BLOCK_1x128_128x128)
    if dtype == torch.float32:
        assert_f32_close(out, ref, f"pitch N+3 M{M} N{N} K{K}")
    else:
        assert_bf16_close(out, ref, f"pitch N+3 M{M} N{N} K{K}")

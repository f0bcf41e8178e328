"""GPU parity of the grouped (mixture-of-experts) blockwise GEMM: every
group's rows of D against the oracle's GEMM of that group's A rows and B_g
(each group is an ordinary 1x128 x 128x128 scaled GEMM), with ragged and
empty groups, ragged N and K, and the Llama4 layer shape split over eight
groups (equal and ragged token counts)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_11_b200 import build, inputs, ops
from parity import assert_bf16_close, assert_bytes_equal, assert_f32_close, assert_scales_equal, bits, grid_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    ops.lib()
    oracle.lib()


def rand_scales(rng, shape):
    return (2.0 ** rng.uniform(-8, 0, size=shape)).astype(np.float32)


def run_grouped(rows, N, K, seed, out_dtype, sample=None):
    rng = np.random.default_rng(seed)
    G, Mt, Kb, Nb = len(rows), sum(rows), (K + 127) // 128, (N + 127) // 128
    A = inputs.random_e4m3_bytes(max(Mt, 1), K, seed=seed)[:Mt]
    Bt = inputs.random_e4m3_bytes(G * N, K, seed=seed + 1)
    sa = rand_scales(rng, (Mt, Kb))
    sb = rand_scales(rng, (G, Nb, Kb))
    sad = ops.colmajor_grid(max(Mt, 1), Kb, "cuda")
    sad[:Mt].copy_(torch.from_numpy(sa))
    sbd = ops.grouped_scale_grids(G, N, K, "cuda")
    for g in range(G):
        ops.grouped_grid_view(sbd, g, N).copy_(torch.from_numpy(sb[g]))
    D = ops.fp8_scaled_gemm_grouped(A.cuda(), Bt.cuda(), rows, sad, sbd, N, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ops.fp8bs_check_device_error() == 0
    r0 = 0
    for g, mg in enumerate(rows):
        if mg:
            sel = None if sample is None else sorted({0, mg // 2, mg - 1} | {i for i in sample if i < mg})
            ref = oracle.gemm(A[r0:r0 + mg].numpy(), Bt[g * N:(g + 1) * N].numpy(), sa[r0:r0 + mg], sb[g],
                              oracle.SCALE_BLOCK_1x128_128x128, rows=sel)
            got = D[r0:r0 + mg] if sel is None else D[r0:r0 + mg][torch.as_tensor(sel, device="cuda")]
            what = f"group {g} ({mg} rows) of {rows}, N{N} K{K}"
            if out_dtype == torch.float32:
                assert_f32_close(got, ref, what)
            else:
                assert_bf16_close(got, ref, what)
        r0 += mg
    return D


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,N,K", [([300, 17, 0, 513, 1], 384, 1008), ([128], 256, 128), ([0, 0, 5], 520, 512),
                                      ([129, 255, 1000, 64], 1000, 2048)])
def test_grouped_ragged(rows, N, K, out_dtype):
    run_grouped(rows, N, K, seed=sum(rows) + N + K, out_dtype=out_dtype)


def test_grouped_all_empty():
    """Every group empty: nothing to compute, nothing written, status OK."""
    A = torch.zeros((0, 256), dtype=torch.uint8, device="cuda")
    Bt = torch.zeros((2 * 256, 256), dtype=torch.uint8, device="cuda")
    sa = ops.colmajor_grid(1, 2, "cuda")
    sb = ops.grouped_scale_grids(2, 256, 256, "cuda")
    D = ops.fp8_scaled_gemm_grouped(A, Bt, [0, 0], sa, sb, 256)
    torch.cuda.synchronize()
    assert D.shape == (0, 256)


@pytest.mark.parametrize("rows", [[2080] * 8, [4000, 1, 127, 129, 3000, 0, 5000, 4383]])
def test_grouped_llama4_shape(rows):
    """Sixteen thousand six hundred forty tokens over eight groups at the Llama4
    layer shape (N, K) = (5120, 8192), sampled rows of every group."""
    run_grouped(rows, 5120, 8192, seed=len(rows) + rows[0], out_dtype=torch.bfloat16, sample=[1, 127, 128, 1999])


def test_grouped_workload_from_quantized_inputs():
    """Four experts' kaiming-uniform weights quantized 128x128 into the stacked
    grids, token rows quantized 1x128, all on the GPU and bit-exact against
    the oracle's quantization; each group's output against the oracle GEMM."""
    rows, N, K = [200, 0, 333, 96], 512, 1024
    g_ = torch.Generator().manual_seed(7)
    x = torch.randn(sum(rows), K, generator=g_).to(torch.bfloat16)
    W = ((torch.rand(len(rows) * N, K, generator=g_) * 2 - 1) / K ** 0.5).to(torch.bfloat16)
    qx, sx = ops.fp8_quant_1x128(x.cuda())
    qw = torch.empty((len(rows) * N, K), dtype=torch.uint8, device="cuda")
    sw = ops.grouped_scale_grids(len(rows), N, K, "cuda")
    Wd = W.cuda()
    for g in range(len(rows)):
        ops.fp8_quant_128x128(Wd[g * N:(g + 1) * N], out=(qw[g * N:(g + 1) * N], ops.grouped_grid_view(sw, g, N),
                                                           None, None))
    D = ops.fp8_scaled_gemm_grouped(qx, qw, rows, sx, sw, N)
    torch.cuda.synchronize()
    assert ops.fp8bs_check_device_error() == 0
    qxo, sxo = oracle.quant_1x128(bits(x))
    assert_bytes_equal(qx, qxo, "token rows")
    assert_scales_equal(grid_np(sx), sxo, "token scales")
    r0 = 0
    for g, mg in enumerate(rows):
        qwo, swo = oracle.quant_128x128(bits(W[g * N:(g + 1) * N]))
        assert_bytes_equal(qw[g * N:(g + 1) * N], qwo, f"W_{g} bytes")
        assert_scales_equal(grid_np(ops.grouped_grid_view(sw, g, N)), swo, f"W_{g} scales")
        if mg:
            ref = oracle.gemm(qxo[r0:r0 + mg], qwo, sxo[r0:r0 + mg], swo, oracle.SCALE_BLOCK_1x128_128x128)
            assert_bf16_close(D[r0:r0 + mg], ref, f"expert {g}")
        r0 += mg


def test_grouped_rejects_other_recipes_and_too_many_groups():
    A = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    Bt = torch.zeros((65 * 128, 128), dtype=torch.uint8, device="cuda")
    sa = ops.colmajor_grid(128, 1, "cuda").fill_(1.0)
    sb = ops.grouped_scale_grids(65, 128, 128, "cuda").fill_(1.0)
    with pytest.raises(ops.Fp8bsError):
        ops.fp8_scaled_gemm_grouped(A, Bt, [2] * 64 + [0], sa, sb, 128)

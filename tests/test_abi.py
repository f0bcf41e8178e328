"""The C-ABI library loads, exports every entry point include/fp8bs.h declares,
and rejects bad arguments with the documented status codes before touching the
GPU (every call below fails validation, so nothing is launched; these run on
a machine without a GPU)."""
import ctypes
import os
import re

import pytest

from fp8_block_scaled_11_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bs.h")

OK, INVALID, UNSUPPORTED, ALIGN, WORKSPACE = 0, 1, 2, 3, 4
GOOD = 0x10000          # fake 16-byte-aligned address: only used in calls that fail validation
BAD = 0x10001           # misaligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:fp8|fp8bs)_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def test_header_declares_the_path(L):
    names = declared_functions()
    for want in ("fp8_quant_1x128", "fp8_quant_1x128_dual", "fp8_quant_128x128", "fp8_quant_tensor",
                 "fp8_quant_rowwise", "fp8_scaled_gemm", "fp8_scaled_gemm_quant", "fp8_scaled_gemm_workspace_size",
                 "fp8bs_status_string",
                 "fp8bs_check_device_error", "fp8_quant_tensor_workspace_size"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in ops.STATUS_NAMES.items():
        assert ops.fp8bs_status_string(code) == name


def q1x128(L, x=GOOD, xt=0, rows=256, cols=256, ldx=256, q=GOOD, ldq=256, s=GOOD, lds=256, t=0):
    return L.fp8_quant_1x128(x, xt, rows, cols, ldx, q, ldq, s, lds, t, None)


def test_quant_1x128_validation(L):
    assert q1x128(L, x=0) == INVALID
    assert q1x128(L, rows=0) == INVALID
    assert q1x128(L, xt=7) == UNSUPPORTED
    assert q1x128(L, ldx=128) == INVALID            # ldx < cols
    assert q1x128(L, lds=100) == INVALID            # ld_scale < rows
    assert q1x128(L, t=2) == INVALID
    assert q1x128(L, x=BAD) == ALIGN
    assert q1x128(L, cols=200, ldx=200, ldq=208) == ALIGN     # cols % 16
    assert q1x128(L, ldq=260) == ALIGN
    assert q1x128(L, lds=258) == ALIGN
    assert q1x128(L, rows=200, lds=256, t=1) == ALIGN         # transposed needs rows % 16


def qdual(L, x=GOOD, xt=0, rows=256, cols=384, ldx=384, q=GOOD, ldq=384, s=GOOD, lds=256, qt=GOOD, ldqt=256,
          st=GOOD, ldst=384):
    return L.fp8_quant_1x128_dual(x, xt, rows, cols, ldx, q, ldq, s, lds, qt, ldqt, st, ldst, None)


def test_quant_1x128_dual_validation(L):
    for kw in ({"x": 0}, {"q": 0}, {"s": 0}, {"qt": 0}, {"st": 0}, {"rows": 0}, {"cols": 0}):
        assert qdual(L, **kw) == INVALID, kw
    assert qdual(L, ldx=256) == INVALID              # ldx < cols
    assert qdual(L, ldq=368) == INVALID              # ldq < cols
    assert qdual(L, lds=240) == INVALID              # ld_scale < rows
    assert qdual(L, ldqt=240) == INVALID             # ldq_t < rows
    assert qdual(L, ldst=368) == INVALID             # ld_scale_t < cols
    assert qdual(L, xt=5) == UNSUPPORTED
    for kw in ({"x": BAD}, {"q": BAD}, {"s": BAD}, {"qt": BAD}, {"st": BAD}):
        assert qdual(L, **kw) == ALIGN, kw
    assert qdual(L, rows=200, lds=200, ldqt=208) == ALIGN       # rows % 16
    assert qdual(L, cols=200, ldx=200, ldq=208, ldst=200) == ALIGN   # cols % 16
    assert qdual(L, ldq=392) == ALIGN                # ldq % 16
    assert qdual(L, ldqt=264) == ALIGN               # ldq_t % 16
    assert qdual(L, lds=258) == ALIGN                # ld_scale % 4
    assert qdual(L, ldx=388) == ALIGN                # bf16 rows of 776 bytes: not a multiple of 16


def test_quant_128x128_validation(L):
    f = L.fp8_quant_128x128
    assert f(GOOD, 0, 256, 256, 256, 0, 0, 0, 0, 0, 0, 0, 0, None) == INVALID        # no output
    assert f(GOOD, 0, 256, 256, 256, GOOD, 256, 0, 4, 0, 0, 0, 0, None) == INVALID   # q without scales
    assert f(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 1, 0, 0, 0, 0, None) == INVALID  # ld_scale < 2
    assert f(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 2, 0, 0, 0, 0, None) == ALIGN    # ld_scale % 4
    assert f(GOOD, 0, 256, 256, 256, 0, 0, 0, 0, GOOD, 256, 0, 4, None) == INVALID     # q_t without scales
    assert f(GOOD, 0, 250, 256, 256, GOOD, 256, GOOD, 4, 0, 0, 0, 0, None) == ALIGN    # rows % 16
    assert f(GOOD, 3, 256, 256, 256, GOOD, 256, GOOD, 4, 0, 0, 0, 0, None) == UNSUPPORTED


def test_quant_tensor_and_rowwise_validation(L):
    assert L.fp8_quant_tensor_workspace_size(1 << 20) >= 4
    assert L.fp8_quant_tensor(GOOD, 0, 1024, GOOD, GOOD, 0, 0, None) == WORKSPACE
    assert L.fp8_quant_tensor(GOOD, 0, 1000, GOOD, GOOD, GOOD, 1 << 16, None) == ALIGN
    assert L.fp8_quant_tensor(0, 0, 1024, GOOD, GOOD, GOOD, 1 << 16, None) == INVALID
    assert L.fp8_quant_rowwise(GOOD, 0, 16, 24, 24, GOOD, 32, GOOD, None) == ALIGN
    assert L.fp8_quant_rowwise(GOOD, 0, 16, 32, 16, GOOD, 32, GOOD, None) == INVALID


def gemm(L, M=256, N=256, K=256, A=GOOD, lda=256, B=GOOD, ldb=256, sa=GOOD, ldsa=256, sb=GOOD, ldsb=256,
         mode=3, layout=0, D=GOOD, ldd=256, od=0, ws=0, wsb=0):
    return L.fp8_scaled_gemm(M, N, K, A, lda, B, ldb, sa, ldsa, sb, ldsb, mode, layout, D, ldd, od, ws, wsb, None)


def test_gemm_validation(L):
    assert gemm(L, mode=9) == UNSUPPORTED
    assert gemm(L, layout=1) == UNSUPPORTED
    assert gemm(L, od=5) == UNSUPPORTED
    assert gemm(L, A=0) == INVALID
    assert gemm(L, K=8) == INVALID                       # K < 16
    assert gemm(L, K=200, lda=256, ldb=256) == ALIGN     # K % 16
    assert gemm(L, lda=128) == INVALID                   # lda < K
    assert gemm(L, ldsa=128) == INVALID                  # ld_sa < M (block modes)
    assert gemm(L, mode=2, ldsb=1) == INVALID            # ld_sb < ceil(N/128)
    assert gemm(L, ldsa=258) == ALIGN
    assert gemm(L, lda=264) == ALIGN
    assert gemm(L, D=BAD) == ALIGN                       # not element-aligned
    assert gemm(L, D=GOOD + 2, od=1) == ALIGN            # fp32 output needs 4-byte alignment
    assert gemm(L, sa=GOOD + 4) == ALIGN


def test_workspace_size_is_zero_for_large_problems(L):
    # with >= 74 output tiles the GEMM never splits K (sizes only; no GPU needed
    # beyond the SM count query, which falls back to 148 without a device)
    assert L.fp8_scaled_gemm_workspace_size(16640, 5120, 8192, 2) == 0
    small = L.fp8_scaled_gemm_workspace_size(256, 512, 128000, 2)
    assert small > 0 and small % 16 == 0


def gq(L, M=256, N=384, K=256, A=GOOD, lda=256, B=GOOD, ldb=256, sa=GOOD, lsa=256, sb=GOOD, lsb=4, mode=2, lay=0,
       D=GOOD, ldd=384, q=GOOD, ldq=384, s=GOOD, lds=256):
    return L.fp8_scaled_gemm_quant(M, N, K, A, lda, B, ldb, sa, lsa, sb, lsb, mode, lay, D, ldd, q, ldq, s, lds, None)


def test_gemm_quant_validation(L):
    assert gq(L, q=0) == INVALID                    # no quantized output
    assert gq(L, s=0) == INVALID                    # no scales
    assert gq(L, ldq=256) == INVALID                # ldq_out < N
    assert gq(L, lds=128) == INVALID                # ld_scale_out < M
    assert gq(L, q=BAD) == ALIGN
    assert gq(L, s=GOOD + 8) == ALIGN
    assert gq(L, ldq=392) == ALIGN                  # ldq_out % 16
    assert gq(L, lds=258) == ALIGN                  # ld_scale_out % 4
    assert gq(L, mode=3, lsb=384) == UNSUPPORTED    # 1x128 x 1x128: 64 columns per promotion thread
    assert gq(L, mode=7) == UNSUPPORTED
    assert gq(L, A=0) == INVALID
    assert gq(L, D=GOOD, ldd=100) == INVALID        # stored output with ldd < N



def test_quant_ex_validation(L):
    """The scale-rule entry points: an unknown rule is refused; with a known
    rule they validate exactly as the plain entry points."""
    f = L.fp8_quant_1x128_ex
    assert f(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 256, 0, 2, None) == UNSUPPORTED
    for rule in (0, 1):
        assert f(0, 0, 256, 256, 256, GOOD, 256, GOOD, 256, 0, rule, None) == INVALID
        assert f(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 258, 0, rule, None) == ALIGN
        assert f(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 100, 0, rule, None) == INVALID
    d = L.fp8_quant_1x128_dual_ex
    assert d(GOOD, 0, 256, 384, 384, GOOD, 384, GOOD, 256, GOOD, 256, GOOD, 384, 5, None) == UNSUPPORTED
    assert d(GOOD, 0, 256, 384, 384, GOOD, 384, GOOD, 256, 0, 256, GOOD, 384, 1, None) == INVALID
    assert d(GOOD, 0, 256, 384, 384, GOOD, 392, GOOD, 256, GOOD, 256, GOOD, 384, 1, None) == ALIGN
    t = L.fp8_quant_128x128_ex
    assert t(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 4, 0, 0, 0, 0, -1, None) == UNSUPPORTED
    assert t(GOOD, 0, 256, 256, 256, 0, 0, 0, 0, 0, 0, 0, 0, 1, None) == INVALID
    assert t(GOOD, 0, 256, 256, 256, GOOD, 256, GOOD, 2, 0, 0, 0, 0, 1, None) == ALIGN


def test_gemm_pow2_validation(L):
    """The power-of-two recipes take the block recipes' scale grids and their
    checks; they have no MN-major, fused-quantization or grouped form."""
    assert gemm(L, mode=4, ldsb=1) == INVALID            # 128x128 grid: ld_sb < ceil(N/128)
    assert gemm(L, mode=5, ldsb=128) == INVALID          # 1x128 grid: ld_sb < N
    assert gemm(L, mode=4, ldsa=128) == INVALID          # ld_sa < M
    assert gemm(L, mode=5, ldsb=258) == ALIGN
    assert gemm(L, mode=6) == UNSUPPORTED
    ex = L.fp8_scaled_gemm_ex
    assert ex(256, 256, 256, GOOD, 256, GOOD, 256, 1, GOOD, 256, GOOD, 4, 4, 0, GOOD, 256, 0, 0, 0, None) == UNSUPPORTED
    assert gq(L, mode=4) == UNSUPPORTED
    assert gq(L, mode=5, lsb=384) == UNSUPPORTED
    # split-K workspace: the power-of-two recipes plan 128 x 256 single-CTA tiles
    assert L.fp8_scaled_gemm_workspace_size(16640, 5120, 8192, 4) == 0
    ws = L.fp8_scaled_gemm_workspace_size(256, 512, 128128, 4)
    assert ws > 0 and ws % 16 == 0

"""CPU oracle for the FP8 (e4m3) dynamic-quantization + scaled-GEMM path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``fp8_block_scaled_11_b200``) never imports it, and the two share
no code: the arithmetic lives in ``oracle/fp8_oracle.c`` (plain C, fp64 where
the method does not fix fp32), wrapped here with numpy arrays through ctypes.

Passages each function follows are cited in ``fp8_oracle.c``.  Every function
here is pinned by ``tests/test_oracle_pins.py`` (closed forms, a library e4m3
cast, printed values from the pages, exact-rational brute force).
"""
from __future__ import annotations

import ctypes
import os
import numpy as np

from .build import build as _build, LIB_PATH

_lib = None

BF16 = 0
F32 = 1

SCALE_TENSOR = 0
SCALE_ROWWISE = 1
SCALE_BLOCK_1x128_128x128 = 2
SCALE_BLOCK_1x128_1x128 = 3

SCALE_RULE_FP32 = 0
SCALE_RULE_POW2 = 1

_p = ctypes.c_void_p
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            _build()
        L = ctypes.CDLL(LIB_PATH)
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode_array.argtypes = [_p, _i64, _p]
        L.oracle_e4m3_decode_array.argtypes = [_p, _i64, _p]
        L.oracle_quant_1x128.argtypes = [_p, ctypes.c_int, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64, _p, _i64]
        L.oracle_quant_128x128.argtypes = [_p, ctypes.c_int, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64, _p, _i64]
        L.oracle_quant_rowwise.argtypes = [_p, ctypes.c_int, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64, _p]
        L.oracle_quant_tensor.argtypes = [_p, ctypes.c_int, _i64, _p, _p]
        gemm_args = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, _i64, _p, _i64, ctypes.c_int, _p, _i64, _p]
        L.oracle_gemm.argtypes = gemm_args
        L.oracle_gemm_blocksum.argtypes = gemm_args
        L.oracle_matmul_ref.argtypes = [_i64, _i64, _p, ctypes.c_int, _i64, _i64, _p, ctypes.c_int, _i64, _i64, _p, _i64, _p]
        L.oracle_sqnr.restype = ctypes.c_double
        L.oracle_sqnr.argtypes = [_p, _p, _i64]
        L.oracle_to_bf16.argtypes = [_p, _i64, _p]
        L.oracle_set_scale_rule.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _as_input(x: np.ndarray):
    """Accept float32 arrays or bf16 given as uint16 bit patterns."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), BF16
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), F32
    raise TypeError(f"oracle input must be float32 or bf16 bits (uint16), got {x.dtype}")


def _rows_arg(rows):
    if rows is None:
        return None, ctypes.c_void_p(0), 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, _ptr(r), r.size


# --------------------------------------------------------------------------- #
# e4m3 codec
# --------------------------------------------------------------------------- #
def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, dtype=np.float64)
    lib().oracle_e4m3_decode_array(_ptr(b), b.size, _ptr(out))
    return out


# --------------------------------------------------------------------------- #
# Quantization.  x is a 2-D row-major array (float32, or bf16 bits as uint16).
# --------------------------------------------------------------------------- #
class scale_rule:
    """Context manager selecting the quantization functions' scale rule:
    SCALE_RULE_FP32 (the method's s = 448/amax, the default) or
    SCALE_RULE_POW2 (the largest power of two not above it: the UE8M0 block
    scales of hardware block scaling).  Not thread-safe (test infrastructure)."""

    def __init__(self, rule: int):
        self.rule = rule

    def __enter__(self):
        lib().oracle_set_scale_rule(self.rule)
        return self

    def __exit__(self, *exc):
        lib().oracle_set_scale_rule(SCALE_RULE_FP32)
        return False


def quant_1x128(x: np.ndarray, transpose: bool = False, rows=None):
    """1x128 groups along the contiguous dim of x (or, with transpose=True,
    along the rows of x, producing the quantized transpose).

    Returns (q, scale_inv) with q of shape (n_out, C') and scale_inv of shape
    (n_out, ceil(C'/128)) holding the column-major grid as a numpy array
    indexed [row, group]."""
    x, xt = _as_input(x)
    R, C = x.shape
    if transpose:
        nview, cols, s0, s1 = C, R, 1, C
    else:
        nview, cols, s0, s1 = R, C, C, 1
    r, rp, nr = _rows_arg(rows)
    n_out = nr if r is not None else nview
    G = (cols + 127) // 128
    q = np.zeros((n_out, cols), dtype=np.uint8)
    sinv = np.zeros((G, max(n_out, 1)), dtype=np.float32)   # column-major grid
    lib().oracle_quant_1x128(_ptr(x), xt, nview, cols, s0, s1, rp, nr,
                             _ptr(q), cols, _ptr(sinv), max(n_out, 1))
    return q, sinv.T[:n_out].copy()


def quant_128x128(x: np.ndarray, transpose: bool = False, rblocks=None):
    """128x128 tiles.  Returns (q, scale_inv[row_block, col_block])."""
    x, xt = _as_input(x)
    R, C = x.shape
    if transpose:
        nview, cols, s0, s1 = C, R, 1, C
    else:
        nview, cols, s0, s1 = R, C, C, 1
    RB = (nview + 127) // 128
    CB = (cols + 127) // 128
    r, rp, nr = _rows_arg(rblocks)
    n_rb = nr if r is not None else RB
    n_rows_out = n_rb * 128 if r is not None else nview
    q = np.zeros((max(n_rb * 128, n_rows_out), cols), dtype=np.uint8)
    sinv = np.zeros((CB, n_rb), dtype=np.float32)
    lib().oracle_quant_128x128(_ptr(x), xt, nview, cols, s0, s1, rp, nr,
                               _ptr(q), cols, _ptr(sinv), n_rb)
    return q[:n_rows_out], sinv.T.copy()


def quant_rowwise(x: np.ndarray, rows=None):
    x, xt = _as_input(x)
    R, C = x.shape
    r, rp, nr = _rows_arg(rows)
    n_out = nr if r is not None else R
    q = np.zeros((n_out, C), dtype=np.uint8)
    sinv = np.zeros((n_out,), dtype=np.float32)
    lib().oracle_quant_rowwise(_ptr(x), xt, R, C, C, 1, rp, nr, _ptr(q), C, _ptr(sinv))
    return q, sinv


def quant_tensor(x: np.ndarray):
    x, xt = _as_input(x)
    q = np.zeros(x.shape, dtype=np.uint8)
    sinv = np.zeros((1,), dtype=np.float32)
    lib().oracle_quant_tensor(_ptr(x), xt, x.size, _ptr(q), _ptr(sinv))
    return q, sinv


# --------------------------------------------------------------------------- #
# GEMM
# --------------------------------------------------------------------------- #
def _scale_arg(s, mode, what):
    """Scales are passed as numpy arrays indexed like the method's grids:
    tensor -> shape (1,), rowwise -> (M,) / (N,), block -> [row, kb] (A, and B
    for 1x128) or [nb, kb] (B for 128x128).  Returns (flat column-major
    buffer, leading dimension)."""
    s = np.asarray(s, dtype=np.float32)
    if mode in (SCALE_TENSOR, SCALE_ROWWISE):
        return np.ascontiguousarray(s.reshape(-1)), 1
    colmajor = np.ascontiguousarray(s.T)      # [kb][row] -> leading dim = rows
    return colmajor.reshape(-1), s.shape[0]


def gemm(A, Bt, sa, sb, mode, rows=None, exact_blocks=False):
    """C = A . Bt^T with scales, returned in fp64 (n_out x N)."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    Bt = np.ascontiguousarray(Bt, dtype=np.uint8)
    M, K = A.shape
    N, K2 = Bt.shape
    assert K == K2
    sa_buf, ld_sa = _scale_arg(sa, mode, "a")
    sb_buf, ld_sb = _scale_arg(sb, mode, "b")
    r, rp, nr = _rows_arg(rows)
    n_out = nr if r is not None else M
    C = np.zeros((n_out, N), dtype=np.float64)
    fn = lib().oracle_gemm_blocksum if exact_blocks else lib().oracle_gemm
    fn(M, N, K, _ptr(A), K, _ptr(Bt), K, _ptr(sa_buf), ld_sa, _ptr(sb_buf), ld_sb,
       int(mode), rp, nr, _ptr(C))
    return C


def matmul_ref(X, Y, rows=None):
    """Unquantized fp64 reference C = X . Y^T on the original inputs."""
    X, xt = _as_input(X)
    Y, yt = _as_input(Y)
    M, K = X.shape
    N, _ = Y.shape
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    r, rp, nr = _rows_arg(rows)
    C = np.zeros((nr, N), dtype=np.float64)
    lib().oracle_matmul_ref(N, K, _ptr(X), xt, K, 1, _ptr(Y), yt, K, 1, rp, nr, _ptr(C))
    return C


def sqnr(ref, out) -> float:
    ref = np.ascontiguousarray(ref, dtype=np.float64)
    out = np.ascontiguousarray(out, dtype=np.float64)
    assert ref.size == out.size
    return float(lib().oracle_sqnr(_ptr(ref), _ptr(out), ref.size))


def to_bf16_bits(c):
    c = np.ascontiguousarray(c, dtype=np.float64)
    out = np.empty(c.shape, dtype=np.uint16)
    lib().oracle_to_bf16(_ptr(c), c.size, _ptr(out))
    return out

"""Python binding of libfp8bs (the C ABI in include/fp8bs.h).

Argument marshalling only: every function here checks the tensors' device,
allocates outputs with torch when they are not given, and calls the C entry
point of the same name with raw pointers and torch's current CUDA stream.  All
arithmetic happens in the CUDA library; if the library is missing or was not
built, the first call raises -- there is no fallback path.

Scale grids are column-major fp32, as the library writes and reads them.  In
torch they are returned as (rows, groups) views with strides (1, ld): element
[i, j] is the scale of row i, group j, stored at i + j*ld.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

FP8BS_OK = 0
STATUS_NAMES = {
    0: "FP8BS_OK", 1: "FP8BS_ERR_INVALID_ARG", 2: "FP8BS_ERR_UNSUPPORTED", 3: "FP8BS_ERR_ALIGNMENT",
    4: "FP8BS_ERR_WORKSPACE", 5: "FP8BS_ERR_CUDA", 6: "FP8BS_ERR_TIMEOUT", 7: "FP8BS_ERR_NO_SM100",
    8: "FP8BS_ERR_SCALE",
}

BF16, F32 = 0, 1
SCALE_TENSOR, SCALE_ROWWISE, SCALE_BLOCK_1x128_128x128, SCALE_BLOCK_1x128_1x128 = 0, 1, 2, 3
# the block recipes with power-of-two scales on the block-scaled MMA
SCALE_BLOCK_1x128_128x128_POW2, SCALE_BLOCK_1x128_1x128_POW2 = 4, 5
BLOCK_MODES = (SCALE_BLOCK_1x128_128x128, SCALE_BLOCK_1x128_1x128,
               SCALE_BLOCK_1x128_128x128_POW2, SCALE_BLOCK_1x128_1x128_POW2)
SCALE_RULE_FP32, SCALE_RULE_POW2 = 0, 1
SCALE_COL_MAJOR = 0
MAJOR_K, MAJOR_MN = 0, 1

_lib = None


class Fp8bsError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib():
    """Load libfp8bs.so (built in-tree).  Raises if it is absent."""
    global _lib
    if _lib is None:
        path = _build.LIB_PATH
        if not os.path.exists(path):
            raise ImportError(f"libfp8bs.so not built ({path}); run fp8_block_scaled_11_b200/build.py")
        L = ctypes.CDLL(path)
        p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.fp8_quant_1x128.argtypes = [p, i32, i64, i64, i64, p, i64, p, i64, i32, p]
        L.fp8_quant_1x128_dual.argtypes = [p, i32, i64, i64, i64, p, i64, p, i64, p, i64, p, i64, p]
        L.fp8_quant_128x128.argtypes = [p, i32, i64, i64, i64, p, i64, p, i64, p, i64, p, i64, p]
        L.fp8_quant_1x128_ex.argtypes = [p, i32, i64, i64, i64, p, i64, p, i64, i32, i32, p]
        L.fp8_quant_1x128_dual_ex.argtypes = [p, i32, i64, i64, i64, p, i64, p, i64, p, i64, p, i64, i32, p]
        L.fp8_quant_128x128_ex.argtypes = [p, i32, i64, i64, i64, p, i64, p, i64, p, i64, p, i64, i32, p]
        L.fp8_quant_tensor_workspace_size.argtypes = [i64]
        L.fp8_quant_tensor_workspace_size.restype = sz
        L.fp8_quant_tensor.argtypes = [p, i32, i64, p, p, p, sz, p]
        L.fp8_quant_rowwise.argtypes = [p, i32, i64, i64, i64, p, i64, p, p]
        L.fp8_scaled_gemm_workspace_size.argtypes = [i64, i64, i64, i32]
        L.fp8_scaled_gemm_workspace_size.restype = sz
        L.fp8_scaled_gemm.argtypes = [i64, i64, i64, p, i64, p, i64, p, i64, p, i64, i32, i32, p, i64, i32, p, sz, p]
        L.fp8_scaled_gemm_ex.argtypes = [i64, i64, i64, p, i64, p, i64, i32, p, i64, p, i64, i32, i32, p, i64, i32,
                                         p, sz, p]
        L.fp8_scaled_gemm_grouped.argtypes = [i64, p, i64, i64, p, i64, p, i64, p, i64, p, i64, i64, i32, i32, p,
                                              i64, i32, p]
        L.fp8_scaled_gemm_quant.argtypes = [i64, i64, i64, p, i64, p, i64, p, i64, p, i64, i32, i32, p, i64,
                                            p, i64, p, i64, p]
        L.fp8bs_status_string.argtypes = [i32]
        L.fp8bs_status_string.restype = ctypes.c_char_p
        L.fp8bs_check_device_error.argtypes = [p]
        L.fp8_quant_tensor_noalloc.argtypes = [p, i32, i64, p, p, p]
        for fn in ("fp8_quant_1x128", "fp8_quant_1x128_dual", "fp8_quant_128x128", "fp8_quant_1x128_ex",
                   "fp8_quant_1x128_dual_ex", "fp8_quant_128x128_ex", "fp8_quant_tensor",
                   "fp8_quant_rowwise", "fp8_scaled_gemm", "fp8_scaled_gemm_ex", "fp8_scaled_gemm_quant", "fp8_scaled_gemm_grouped",
                   "fp8bs_check_device_error", "fp8_quant_tensor_noalloc"):
            getattr(L, fn).restype = i32
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != FP8BS_OK:
        raise Fp8bsError(fn, status)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported input dtype {t.dtype} (bf16 or fp32)")


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D row-major tensor (unit column stride)")
    return t.stride(0)


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def colmajor_grid(rows: int, groups: int, device) -> torch.Tensor:
    """Allocate a column-major fp32 scale grid (rows x groups), ld = rows rounded up to 4."""
    ld = _round_up(max(rows, 1), 4)
    return torch.empty((groups, ld), dtype=torch.float32, device=device)[:, :rows].t()


def _grid_ld(s: torch.Tensor, rows: int) -> int:
    if s.dim() != 2 or s.dtype != torch.float32:
        raise ValueError("scale grid must be a 2-D fp32 tensor")
    if s.shape[1] == 1:
        return s.stride(1) if s.stride(0) == 1 and s.stride(1) >= rows else _round_up(rows, 4)
    if s.stride(0) != 1:
        raise ValueError("scale grid must be column-major (stride (1, ld))")
    return s.stride(1)


# ---------------------------------------------------------------------------- quantization
def fp8_quant_1x128(x: torch.Tensor, transpose_out: bool = False, q: Optional[torch.Tensor] = None,
                    scale_inv: Optional[torch.Tensor] = None, rule: int = SCALE_RULE_FP32):
    """Returns (q uint8, scale_inv grid).  transpose_out=False: q is rows x cols,
    grid rows x ceil(cols/128).  transpose_out=True: groups run along rows and
    q is the quantized transpose (cols x rows), grid cols x ceil(rows/128).
    Preallocated outputs may be passed as q / scale_inv.  rule =
    SCALE_RULE_POW2 rounds every scale down to a power of two (fp8_quant_1x128_ex)."""
    rows, cols = x.shape
    xt = _dtype_code(x)
    out_rows, out_cols = (cols, rows) if transpose_out else (rows, cols)
    if q is None:
        q = torch.empty((out_rows, out_cols), dtype=torch.uint8, device=x.device)
    s = scale_inv if scale_inv is not None else colmajor_grid(out_rows, (out_cols + 127) // 128, x.device)
    ld_s = _grid_ld(s, out_rows)
    if rule == SCALE_RULE_FP32:
        _check("fp8_quant_1x128", lib().fp8_quant_1x128(x.data_ptr(), xt, rows, cols, _ld(x), q.data_ptr(),
                                                        q.stride(0), s.data_ptr(), ld_s, int(transpose_out),
                                                        _stream(x)))
    else:
        _check("fp8_quant_1x128_ex", lib().fp8_quant_1x128_ex(x.data_ptr(), xt, rows, cols, _ld(x), q.data_ptr(),
                                                              q.stride(0), s.data_ptr(), ld_s, int(transpose_out),
                                                              int(rule), _stream(x)))
    return q, s


def fp8_quant_1x128_dual(x: torch.Tensor, out=None, rule: int = SCALE_RULE_FP32):
    """Both 1x128 quantizations from one read of x: returns (q, scale_inv,
    q_t, scale_inv_t), equal to fp8_quant_1x128(x) followed by
    fp8_quant_1x128(x, transpose_out=True).  Preallocated outputs may be
    passed as out=(q, scale_inv, q_t, scale_inv_t).  rule as fp8_quant_1x128."""
    rows, cols = x.shape
    xt = _dtype_code(x)
    if out is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
        s = colmajor_grid(rows, (cols + 127) // 128, x.device)
        qt = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
        st = colmajor_grid(cols, (rows + 127) // 128, x.device)
    else:
        q, s, qt, st = out
    args = (x.data_ptr(), xt, rows, cols, _ld(x), q.data_ptr(), q.stride(0), s.data_ptr(), _grid_ld(s, rows),
            qt.data_ptr(), qt.stride(0), st.data_ptr(), _grid_ld(st, cols))
    if rule == SCALE_RULE_FP32:
        _check("fp8_quant_1x128_dual", lib().fp8_quant_1x128_dual(*args, _stream(x)))
    else:
        _check("fp8_quant_1x128_dual_ex", lib().fp8_quant_1x128_dual_ex(*args, int(rule), _stream(x)))
    return q, s, qt, st


def fp8_quant_128x128(x: torch.Tensor, want_q: bool = True, want_qt: bool = False, out=None,
                      rule: int = SCALE_RULE_FP32):
    """Returns (q, scale_inv, q_t, scale_inv_t); the unrequested pair is None.
    q: rows x cols, grid ceil(rows/128) x ceil(cols/128).  q_t: cols x rows
    (the same quantized tiles transposed), grid ceil(cols/128) x ceil(rows/128).
    Preallocated outputs may be passed as out=(q, s, q_t, s_t).  rule as
    fp8_quant_1x128."""
    rows, cols = x.shape
    xt = _dtype_code(x)
    rb, cb = (rows + 127) // 128, (cols + 127) // 128
    q = s = qt = st = None
    if out is not None:
        q, s, qt, st = out
    qp = sp = qtp = stp = 0
    ldq = lds = ldqt = ldst = 0
    if want_q:
        if q is None:
            q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
            s = colmajor_grid(rb, cb, x.device)
        qp, sp, ldq, lds = q.data_ptr(), s.data_ptr(), q.stride(0), _grid_ld(s, rb)
    if want_qt:
        if qt is None:
            qt = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
            st = colmajor_grid(cb, rb, x.device)
        qtp, stp, ldqt, ldst = qt.data_ptr(), st.data_ptr(), qt.stride(0), _grid_ld(st, cb)
    args = (x.data_ptr(), xt, rows, cols, _ld(x), qp, ldq, sp, lds, qtp, ldqt, stp, ldst)
    if rule == SCALE_RULE_FP32:
        _check("fp8_quant_128x128", lib().fp8_quant_128x128(*args, _stream(x)))
    else:
        _check("fp8_quant_128x128_ex", lib().fp8_quant_128x128_ex(*args, int(rule), _stream(x)))
    return q, s, qt, st


def fp8_quant_tensor(x: torch.Tensor, workspace: Optional[torch.Tensor] = None):
    """Returns (q, scale_inv[1])."""
    n = x.numel()
    xc = x.contiguous()
    xt = _dtype_code(x)
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    s = torch.empty((1,), dtype=torch.float32, device=x.device)
    wsb = lib().fp8_quant_tensor_workspace_size(n)
    if workspace is None:
        workspace = torch.empty((wsb,), dtype=torch.uint8, device=x.device)
    _check("fp8_quant_tensor", lib().fp8_quant_tensor(xc.data_ptr(), xt, n, q.data_ptr(), s.data_ptr(),
                                                      workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                                      _stream(x)))
    return q, s


def fp8_quant_rowwise(x: torch.Tensor):
    """Returns (q, scale_inv[rows])."""
    rows, cols = x.shape
    xt = _dtype_code(x)
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    s = torch.empty((rows,), dtype=torch.float32, device=x.device)
    _check("fp8_quant_rowwise", lib().fp8_quant_rowwise(x.data_ptr(), xt, rows, cols, _ld(x), q.data_ptr(),
                                                        q.stride(0), s.data_ptr(), _stream(x)))
    return q, s


# ---------------------------------------------------------------------------- GEMM
def fp8_scaled_gemm_workspace_size(M: int, N: int, K: int, mode: int) -> int:
    return int(lib().fp8_scaled_gemm_workspace_size(M, N, K, mode))


def fp8_scaled_gemm(A: torch.Tensor, Bt: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor, mode: int,
                    out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, split_k: bool = True) -> torch.Tensor:
    """D = scaled(A . Bt^T).  A: M x K uint8 (e4m3), Bt: N x K uint8 (e4m3).
    Scales as returned by the quantization functions (TENSOR: 1 element;
    ROWWISE: M / N elements; BLOCK: column-major grids)."""
    M, K = A.shape
    N, K2 = Bt.shape
    if K2 != K:
        raise ValueError("A and Bt must share K")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    oc = F32 if out.dtype == torch.float32 else BF16
    if mode in BLOCK_MODES:
        ld_sa = _grid_ld(scale_a, M)
        ld_sb = _grid_ld(scale_b, scale_b.shape[0])
    else:
        ld_sa = ld_sb = 0
    wsb = fp8_scaled_gemm_workspace_size(M, N, K, mode) if split_k else 0
    if wsb > 0 and workspace is None:
        workspace = torch.empty((wsb,), dtype=torch.uint8, device=A.device)
    wp = workspace.data_ptr() if (workspace is not None and wsb > 0) else 0
    wn = workspace.numel() * workspace.element_size() if (workspace is not None and wsb > 0) else 0
    _check("fp8_scaled_gemm", lib().fp8_scaled_gemm(M, N, K, A.data_ptr(), _ld(A), Bt.data_ptr(), _ld(Bt),
                                                    scale_a.data_ptr(), ld_sa, scale_b.data_ptr(), ld_sb, mode,
                                                    SCALE_COL_MAJOR, out.data_ptr(), _ld(out), oc, wp, wn,
                                                    _stream(A)))
    return out


def fp8_scaled_gemm_ex(A: torch.Tensor, B: torch.Tensor, b_major: int, scale_a: torch.Tensor,
                       scale_b: torch.Tensor, mode: int, out_dtype: torch.dtype = torch.bfloat16,
                       out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       split_k: bool = True) -> torch.Tensor:
    """D = scaled(A . B).  A: M x K uint8 (e4m3).  b_major = MAJOR_MN: B is the
    K x N uint8 matrix itself (N contiguous), with a TENSOR / ROWWISE scale or
    the ceil(K/128) x ceil(N/128) grid fp8_quant_128x128 writes for it;
    b_major = MAJOR_K: B is B^T (N x K), exactly fp8_scaled_gemm."""
    if b_major == MAJOR_K:
        return fp8_scaled_gemm(A, B, scale_a, scale_b, mode, out_dtype=out_dtype, out=out, workspace=workspace,
                               split_k=split_k)
    M, K = A.shape
    K2, N = B.shape
    if K2 != K:
        raise ValueError("A (M x K) and B (K x N) must share K")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    oc = F32 if out.dtype == torch.float32 else BF16
    if mode in BLOCK_MODES:
        ld_sa = _grid_ld(scale_a, M)
        ld_sb = _grid_ld(scale_b, scale_b.shape[0])
    else:
        ld_sa = ld_sb = 0
    wsb = fp8_scaled_gemm_workspace_size(M, N, K, mode) if split_k else 0
    if wsb > 0 and workspace is None:
        workspace = torch.empty((wsb,), dtype=torch.uint8, device=A.device)
    wp = workspace.data_ptr() if (workspace is not None and wsb > 0) else 0
    wn = workspace.numel() * workspace.element_size() if (workspace is not None and wsb > 0) else 0
    _check("fp8_scaled_gemm_ex", lib().fp8_scaled_gemm_ex(M, N, K, A.data_ptr(), _ld(A), B.data_ptr(), _ld(B),
                                                          b_major, scale_a.data_ptr(), ld_sa, scale_b.data_ptr(),
                                                          ld_sb, mode, SCALE_COL_MAJOR, out.data_ptr(), _ld(out),
                                                          oc, wp, wn, _stream(A)))
    return out


def grouped_scale_grids(groups: int, N: int, K: int, device) -> torch.Tensor:
    """Allocate the stacked 128x128 scale grids of a grouped GEMM's B: a
    (groups, ceil(K/128), ld) fp32 tensor, ld = ceil(N/128) rounded up to 4.
    grouped_grid_view(t, g, N) is group g's (ceil(N/128) x ceil(K/128))
    column-major grid, the form fp8_quant_128x128 fills (out=...)."""
    nb, kb = (N + 127) // 128, (K + 127) // 128
    return torch.empty((groups, kb, _round_up(nb, 4)), dtype=torch.float32, device=device)


def grouped_grid_view(t: torch.Tensor, g: int, N: int) -> torch.Tensor:
    """Group g's grid of a grouped_scale_grids tensor: ceil(N/128) x ceil(K/128),
    column-major (strides (1, ld))."""
    return t[g][:, :(N + 127) // 128].t()


def fp8_scaled_gemm_grouped(A: torch.Tensor, Bt: torch.Tensor, group_rows, scale_a: torch.Tensor,
                            scale_b: torch.Tensor, N: int, out_dtype: torch.dtype = torch.bfloat16,
                            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Grouped 1x128 x 128x128 GEMM: for each group g, rows of A from
    sum(group_rows[:g]) on (group_rows[g] of them) times B_g^T = rows
    g*N .. g*N+N-1 of Bt.  A: (sum rows) x K uint8; Bt: (G*N) x K uint8;
    scale_a: the 1x128 grid over A's rows; scale_b: grouped_scale_grids(G, N, K).
    Returns D (sum rows) x N."""
    rows = [int(r) for r in group_rows]
    G = len(rows)
    Mt, K = A.shape
    if Mt != sum(rows) or Bt.shape != (G * N, K):
        raise ValueError("A must hold sum(group_rows) rows and Bt G*N rows of K bytes")
    if scale_b.dim() != 3 or scale_b.dtype != torch.float32 or not scale_b.is_contiguous() or scale_b.shape[0] != G:
        raise ValueError("scale_b must be grouped_scale_grids(G, N, K)")
    if out is None:
        out = torch.empty((Mt, N), dtype=out_dtype, device=A.device)
    oc = F32 if out.dtype == torch.float32 else BF16
    gr = (ctypes.c_int64 * G)(*rows)
    ld_sa = _grid_ld(scale_a, max(Mt, 1))
    _check("fp8_scaled_gemm_grouped",
           lib().fp8_scaled_gemm_grouped(G, ctypes.cast(gr, ctypes.c_void_p), N, K, A.data_ptr(), _ld(A), Bt.data_ptr(),
                                         _ld(Bt), scale_a.data_ptr(), ld_sa, scale_b.data_ptr(), scale_b.shape[2],
                                         scale_b.shape[1] * scale_b.shape[2], SCALE_BLOCK_1x128_128x128,
                                         SCALE_COL_MAJOR, out.data_ptr(), _ld(out), oc, _stream(A)))
    return out


def fp8_scaled_gemm_quant(A: torch.Tensor, Bt: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor, mode: int,
                          out: Optional[torch.Tensor] = None, store_out: bool = True,
                          q_out: Optional[torch.Tensor] = None, scale_out: Optional[torch.Tensor] = None):
    """D = scaled(A . Bt^T) in bf16, quantized 1x128 along N in the GEMM's
    epilogue: returns (D or None, q uint8 M x N, scale_inv grid M x ceil(N/128)),
    byte-identical to fp8_quant_1x128(D).  store_out=False skips writing D."""
    M, K = A.shape
    N, K2 = Bt.shape
    if K2 != K:
        raise ValueError("A and Bt must share K")
    if store_out and out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    if not store_out:
        out = None
    if q_out is None:
        # the byte rows start 16-byte aligned (pitch rounded up to 16)
        q_out = torch.empty((M, (N + 15) // 16 * 16), dtype=torch.uint8, device=A.device)[:, :N]
    if scale_out is None:
        scale_out = colmajor_grid(M, (N + 127) // 128, A.device)
    if mode == SCALE_BLOCK_1x128_128x128:
        ld_sa = _grid_ld(scale_a, M)
        ld_sb = _grid_ld(scale_b, scale_b.shape[0])
    else:
        ld_sa = ld_sb = 0
    dp, ldd = (out.data_ptr(), _ld(out)) if out is not None else (0, 0)
    _check("fp8_scaled_gemm_quant",
           lib().fp8_scaled_gemm_quant(M, N, K, A.data_ptr(), _ld(A), Bt.data_ptr(), _ld(Bt), scale_a.data_ptr(),
                                       ld_sa, scale_b.data_ptr(), ld_sb, mode, SCALE_COL_MAJOR, dp, ldd,
                                       q_out.data_ptr(), q_out.stride(0), scale_out.data_ptr(),
                                       _grid_ld(scale_out, M), _stream(A)))
    return out, q_out, scale_out


def fp8bs_status_string(status: int) -> str:
    return lib().fp8bs_status_string(status).decode()


def fp8bs_check_device_error(stream: Optional[torch.cuda.Stream] = None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(lib().fp8bs_check_device_error(ctypes.c_void_p(s.cuda_stream)))


def fp8_quant_tensor_noalloc(x: torch.Tensor, q: Optional[torch.Tensor] = None,
                             scale_inv: Optional[torch.Tensor] = None):
    """Per-tensor quantization through fp8_quant_tensor_noalloc (no workspace:
    the library uses its built-in 16 KB scratch).  Returns (q, scale_inv[1]);
    pass preallocated q / scale_inv to keep the call itself allocation-free.

    The call cannot copy (a copy would allocate), so x must already be a
    contiguous bf16 / fp32 tensor on the current CUDA device; q must be a
    contiguous uint8 tensor with as many elements as x and scale_inv a
    contiguous fp32 tensor with at least one element, on the same device.
    Anything else raises ValueError before the library is called."""
    dev = torch.device("cuda", torch.cuda.current_device())
    if x.device != dev or not x.is_contiguous():
        raise ValueError("fp8_quant_tensor_noalloc: x must be contiguous and on the current CUDA device")
    xt = _dtype_code(x)
    if q is None:
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale_inv is None:
        scale_inv = torch.empty((1,), dtype=torch.float32, device=x.device)
    if q.dtype != torch.uint8 or q.numel() != x.numel() or not q.is_contiguous() or q.device != dev:
        raise ValueError("fp8_quant_tensor_noalloc: q must be a contiguous uint8 tensor of x.numel() elements "
                         "on the current CUDA device")
    if (scale_inv.dtype != torch.float32 or scale_inv.numel() < 1 or not scale_inv.is_contiguous()
            or scale_inv.device != dev):
        raise ValueError("fp8_quant_tensor_noalloc: scale_inv must be a contiguous fp32 tensor with at least "
                         "one element on the current CUDA device")
    _check("fp8_quant_tensor_noalloc", lib().fp8_quant_tensor_noalloc(x.data_ptr(), xt, x.numel(), q.data_ptr(),
                                                                      scale_inv.data_ptr(), _stream(x)))
    return q, scale_inv

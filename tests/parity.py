"""Comparison helpers for the GPU-vs-oracle parity tests (test code only).

Tolerances (from the method's contract):
  * quantized bytes and fp32 scales: bit-exact;
  * GEMM, fp32 output: relative Frobenius error <= 1e-5 against the oracle's fp64 result;
  * GEMM, bf16 output: per element |C - C_ref| <= 2 ulp_bf16(C_ref) + 1e-6 * ||C_ref[m, :]||_2.
"""
import numpy as np
import torch

FP32_REL_FROB = 1e-5
BF16_ULPS = 2.0
BF16_ROW_REL = 1e-6


def to_np_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def grid_np(s: torch.Tensor) -> np.ndarray:
    """A (rows, groups) column-major grid view -> dense numpy [row, group]."""
    return s.detach().cpu().contiguous().numpy()


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_close(out: torch.Tensor, ref: np.ndarray, what: str = ""):
    got = out.detach().float().cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rown = np.linalg.norm(ref, axis=1, keepdims=True)
    tol = BF16_ULPS * bf16_ulp(ref) + BF16_ROW_REL * rown
    err = np.abs(got - ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements outside 2 bf16 ulp + 1e-6|row|; "
                             f"first at {tuple(i)}: got {got[tuple(i)]!r} ref {ref[tuple(i)]!r} tol {tol[tuple(i)]!r}")


def assert_f32_close(out: torch.Tensor, ref: np.ndarray, what: str = ""):
    got = out.detach().cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape
    num = np.linalg.norm(got - ref)
    den = np.linalg.norm(ref)
    assert num <= FP32_REL_FROB * den, f"{what}: relative Frobenius error {num / max(den, 1e-300):.3e}"


def assert_bytes_equal(got: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = to_np_bits(got)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    if not np.array_equal(g, ref):
        bad = np.argwhere(g != ref)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} bytes differ; first at {i}: gpu {g[i]:#04x} oracle {ref[i]:#04x}")


def assert_scales_equal(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    gb = got.astype(np.float32).view(np.uint32)
    rb = ref.astype(np.float32).view(np.uint32)
    if not np.array_equal(gb, rb):
        bad = np.argwhere(gb != rb)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} scales differ; first at {i}: gpu {got[i]!r} oracle {ref[i]!r}")


def bits(x: torch.Tensor) -> np.ndarray:
    """Oracle input form of a CPU tensor: bf16 -> uint16 bit patterns, fp32 as is."""
    x = x.contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.uint16).numpy()
    return x.numpy()

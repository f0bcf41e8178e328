"""Seeded synthetic inputs for the FP8 quantization + scaled-GEMM workloads.

This module holds no arithmetic of the method: it only draws random tensors
(torch's CPU generator, so the same seed gives the same bytes on any host) in
the shapes and distributions of the pages' workloads.  Both the CUDA path's
tests/benchmarks and the CPU oracle consume these same bytes.

Workloads (shapes and distributions from the pages):

* ``tiny_blockwise``   A fp32 256x1024 ~ N(0,1), then B fp32 1024x512 ~ N(0, 0.02^2),
  seed 0; B is handed to the GEMM as B^T (512x1024).
* ``per_tensor``       x bf16 256x1024 ~ N(0,1), then W bf16 4096x1024 ~ N(0,1), seed 1
  (ROCm/aiter issue #1765, Steps to Reproduce: M, N, K = 256, 4096, 1024).
* ``quant_sweep(n)``   A bf16 n x n ~ N(0,1), seed 2, n in 1024..32768
  (pytorch/ao PR #2592, Performance table).
* ``llama4(N, K)``     M = 16640 tokens; x bf16 MxK ~ N(0,1), W bf16 NxK ~ U(-1/sqrt(K), 1/sqrt(K))
  (nn.Linear's default kaiming-uniform init, fan_in = K), grad_out bf16 MxN ~ N(0,1),
  seed 3, drawn in that order (pytorch/ao PR #2785, Benchmarks table).
* ``long_k(K)``        grad_out^T bf16 256xK ~ N(0,1), then x bf16 Kx512 ~ U(-1/sqrt(512), 1/sqrt(512)),
  seed 4, K in {128000, 128128, 128256} (pytorch/ao PR #4209, What Changed / Findings So Far).
"""
from __future__ import annotations

import math
import torch

LLAMA4_M = 16640
LLAMA4_SHAPES = ((5120, 8192), (8192, 5120))
QUANT_SWEEP_SIZES = (1024, 2048, 4096, 8192, 16384, 32768)
LONG_K_VALUES = (128000, 128128, 128256)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _uniform(shape, bound, g, dtype):
    return ((torch.rand(shape, generator=g, dtype=torch.float32) * 2.0 - 1.0) * bound).to(dtype)


def tiny_blockwise():
    """Returns (A fp32 256x1024, Bt fp32 512x1024)."""
    g = _gen(0)
    A = torch.randn(256, 1024, generator=g, dtype=torch.float32)
    B = torch.randn(1024, 512, generator=g, dtype=torch.float32) * 0.02
    return A, B.t().contiguous()


def per_tensor():
    """Returns (x bf16 256x1024, W bf16 4096x1024)."""
    g = _gen(1)
    x = torch.randn(256, 1024, generator=g, dtype=torch.float32).to(torch.bfloat16)
    W = torch.randn(4096, 1024, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return x, W


def quant_sweep(n: int, m: int | None = None):
    """Square (or n x m) bf16 matrix ~ N(0,1)."""
    g = _gen(2)
    return torch.randn(n, m if m is not None else n, generator=g, dtype=torch.float32).to(torch.bfloat16)


def llama4(N: int, K: int, M: int = LLAMA4_M):
    """Returns (x bf16 MxK, W bf16 NxK, grad_out bf16 MxN)."""
    g = _gen(3)
    x = torch.randn(M, K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    W = _uniform((N, K), 1.0 / math.sqrt(K), g, torch.bfloat16)
    dy = torch.randn(M, N, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return x, W, dy


def long_k(K: int, M: int = 256, N: int = 512):
    """Returns (grad_out^T bf16 MxK, x bf16 KxN)."""
    g = _gen(4)
    goT = torch.randn(M, K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    x = _uniform((K, N), 1.0 / math.sqrt(N), g, torch.bfloat16)
    return goT, x


def random_matrix(rows: int, cols: int, seed: int, dtype=torch.bfloat16, scale: float = 1.0):
    """Generic N(0, scale^2) matrix for edge-case tests."""
    g = _gen(seed)
    return (torch.randn(rows, cols, generator=g, dtype=torch.float32) * scale).to(dtype)


def random_e4m3_bytes(rows: int, cols: int, seed: int):
    """Uniformly random finite e4m3 codes (NaN patterns 0x7F/0xFF excluded)."""
    g = _gen(seed)
    b = torch.randint(0, 254, (rows, cols), generator=g, dtype=torch.int32)
    b = b + (b >= 127).to(torch.int32)          # skip 0x7F
    return b.to(torch.uint8)

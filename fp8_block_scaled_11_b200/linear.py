"""FP8 blockwise linear forward + backward step, composed from the library's
quantization and scaled-GEMM calls (no autograd; buffers preallocated).

The composition is the one pytorch/ao PR #2785 "integrate torch._scaled_mm
into Float8BlockwiseLinear and add bench script" benchmarks (Benchmarks table:
eager linear forward + backward at Llama4 shapes), with the scale recipes of
pytorch/ao PR #4209 (Findings So Far and review thread):

  forward  y  = x . W^T     A = x  (1x128 along K),         B^T = W   (128x128)
  dgrad    dx = dy . W      A = dy (1x128 along N),         B^T = W^T (128x128, same tiles)
  wgrad    dW = dy^T . x    A = dy^T (1x128 along tokens),  B^T = x^T (1x128 along tokens)

x: M x K, W: N x K, dy: M x N (all bf16); outputs bf16.  Three quantization
launches per step -- x in both 1x128 directions from one read, W 128x128, dy
in both directions from one read -- and three GEMM launches.  dgrad reads the
forward's W_q and scale grid in their stored orientation (B MN-major,
fp8_scaled_gemm_ex), so W needs no transposed copy; ``dgrad_wt_copy=True``
instead has the 128x128 launch also write the transposed bytes and grid and
dgrad read them K-major (the same result, 42 MB more written per layer).
With ``pow2=True`` every quantization uses the power-of-two scale rule and
the GEMMs the matching power-of-two recipes on the block-scaled MMA (whole-K
accumulation in TMEM, no per-K-block promotion): the fast-accumulation
variant of pytorch/pytorch issue #159940 (Describe the bug: USE_FAST_ACCUM)
in its B200 form, for the speed / accuracy ablation.  Those recipes read
K-major operands only: pow2=True needs dgrad_wt_copy=True.
"""
from __future__ import annotations

import torch

from . import ops


class Fp8LinearStep:
    """Preallocated buffers for one (M, N, K) linear layer's fwd + bwd."""

    LAUNCHES_PER_STEP = 6

    def __init__(self, M: int, N: int, K: int, device="cuda", dgrad_wt_copy: bool = False, pow2: bool = False):
        self.M, self.N, self.K = M, N, K
        if pow2 and not dgrad_wt_copy:
            raise ValueError("the power-of-two recipes read K-major operands only (dgrad_wt_copy=True)")
        self.dgrad_wt_copy = dgrad_wt_copy
        self.pow2 = pow2
        self.rule = ops.SCALE_RULE_POW2 if pow2 else ops.SCALE_RULE_FP32
        self.modes = ((ops.SCALE_BLOCK_1x128_128x128_POW2, ops.SCALE_BLOCK_1x128_1x128_POW2) if pow2
                      else (ops.SCALE_BLOCK_1x128_128x128, ops.SCALE_BLOCK_1x128_1x128))
        d = device
        u8 = torch.uint8
        g = ops.colmajor_grid
        cd = lambda a: (a + 127) // 128
        # forward / dgrad operands
        self.xq, self.xs = torch.empty((M, K), dtype=u8, device=d), g(M, cd(K), d)
        self.wq, self.ws = torch.empty((N, K), dtype=u8, device=d), g(cd(N), cd(K), d)
        self.wtq = self.wts = None
        if dgrad_wt_copy:
            self.wtq, self.wts = torch.empty((K, N), dtype=u8, device=d), g(cd(K), cd(N), d)
        self.dyq, self.dys = torch.empty((M, N), dtype=u8, device=d), g(M, cd(N), d)
        # wgrad operands (quantized along tokens, stored transposed)
        self.dytq, self.dyts = torch.empty((N, M), dtype=u8, device=d), g(N, cd(M), d)
        self.xtq, self.xts = torch.empty((K, M), dtype=u8, device=d), g(K, cd(M), d)
        # outputs
        bf = torch.bfloat16
        self.y = torch.empty((M, N), dtype=bf, device=d)
        self.dx = torch.empty((M, K), dtype=bf, device=d)
        self.dW = torch.empty((N, K), dtype=bf, device=d)
        ws = max(ops.fp8_scaled_gemm_workspace_size(M, N, K, self.modes[0]),
                 ops.fp8_scaled_gemm_workspace_size(M, K, N, self.modes[0]),
                 ops.fp8_scaled_gemm_workspace_size(N, K, M, self.modes[1]))
        self.workspace = torch.empty((max(ws, 16),), dtype=u8, device=d)

    def quantize(self, x: torch.Tensor, W: torch.Tensor, dy: torch.Tensor):
        ops.fp8_quant_1x128_dual(x, out=(self.xq, self.xs, self.xtq, self.xts), rule=self.rule)
        ops.fp8_quant_128x128(W, want_q=True, want_qt=self.dgrad_wt_copy,
                              out=(self.wq, self.ws, self.wtq, self.wts), rule=self.rule)
        ops.fp8_quant_1x128_dual(dy, out=(self.dyq, self.dys, self.dytq, self.dyts), rule=self.rule)

    def gemms(self, mark=None):
        """The three GEMMs; `mark(i)` (optional) is called before GEMM i and
        after the last one (i = 3), e.g. to record CUDA events between them."""
        B2, B3 = self.modes
        mark = mark or (lambda i: None)
        mark(0)
        ops.fp8_scaled_gemm(self.xq, self.wq, self.xs, self.ws, B2, out=self.y, workspace=self.workspace)
        mark(1)
        if self.dgrad_wt_copy:
            ops.fp8_scaled_gemm(self.dyq, self.wtq, self.dys, self.wts, B2, out=self.dx, workspace=self.workspace)
        else:
            ops.fp8_scaled_gemm_ex(self.dyq, self.wq, ops.MAJOR_MN, self.dys, self.ws, B2, out=self.dx,
                                   workspace=self.workspace)
        mark(2)
        ops.fp8_scaled_gemm(self.dytq, self.xtq, self.dyts, self.xts, B3, out=self.dW, workspace=self.workspace)
        mark(3)

    def run(self, x: torch.Tensor, W: torch.Tensor, dy: torch.Tensor):
        self.quantize(x, W, dy)
        self.gemms()
        return self.y, self.dx, self.dW

    def flops(self) -> float:
        return 3 * self.gemm_flops()

    def gemm_flops(self) -> float:
        """Flops of each of the three GEMMs (they are equal: 2 M N K)."""
        return 2.0 * self.M * self.N * self.K

    def quant_bytes(self) -> float:
        """Algorithmic HBM bytes of the three quantization launches: each bf16
        input read once (2 B per element), its e4m3 outputs written (1 B per
        element each: two for x and dy, one for W unless the transposed copy
        is kept), plus 4 bytes per scale written."""
        M, N, K = self.M, self.N, self.K
        cd = lambda a: (a + 127) // 128
        copies = 2 if self.dgrad_wt_copy else 1
        b = 0.0
        b += M * K * 4 + 4 * M * cd(K) + 4 * K * cd(M)     # x: 1x128 along K and along tokens
        b += N * K * (2 + copies) + copies * 4 * cd(N) * cd(K)   # W 128x128 (+ transposed copy)
        b += M * N * 4 + 4 * M * cd(N) + 4 * N * cd(M)     # dy: 1x128 along N and along tokens
        return b

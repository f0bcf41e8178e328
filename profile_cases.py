"""Single-kernel cases for profiling (ncu) and per-kernel timing.

  python profile_cases.py <case> [--reps R] [--time]

Cases (seeded inputs of the workloads, operands prepared before the loop so
only the named kernel runs R times):
  gemm_fwd     Llama4 forward GEMM 16640 x 5120 x 8192, 1x128 x 128x128, bf16 out
  gemm_wgrad   Llama4 wgrad GEMM 5120 x 8192 x 16640, 1x128 x 1x128, bf16 out
  gemm_dgrad   Llama4 dgrad GEMM 16640 x 8192 x 5120 (dy . W), 1x128 x 128x128, bf16 out, W_q read MN-major
  gemm_dgrad_wt        the same reading the 128x128 kernel's transposed copy of W_q (K-major)
  gemm_tensor  16640 x 5120 x 8192 per-tensor scales, bf16 out
  gemm_rowwise 16640 x 5120 x 8192 rowwise scales, bf16 out
  gemm_fwd_quant       the forward GEMM with its output quantized 1x128 in the epilogue (bf16 out stored)
  gemm_fwd_quant_only  the same without storing the bf16 output
  gemm_fwd_then_quant  the forward GEMM, then fp8_quant_1x128 of its output (two launches)
  gemm_longk   256 x 512 x 128128 (k_blocks 1001), 1x128 x 128x128, split-K, bf16 out
  gemm_longk_mn        the same with x (K x 512) quantized as stored and read MN-major
  gemm_longk_1x128     the long-K GEMM with the 1x128 x 1x128 recipe
  <gemm case>_pow2     gemm_fwd, gemm_dgrad_wt, gemm_wgrad, gemm_longk, gemm_longk_1x128 with
                       power-of-two scales on the block-scaled MMA (the fast-accumulation variant)
  gemm_grouped         grouped GEMM: 8 groups x 2080 tokens over (N, K) = (5120, 8192), 1x128 x 128x128
  gemm_grouped_ragged  the same with ragged group sizes (4000, 1, 127, 129, 3000, 0, 5000, 4383)
  quant_rows   1x128 quantization of a 32768 x 32768 bf16 matrix
  quant_cols   1x128 along rows (transposed output) of a 16640 x 8192 bf16 matrix
  quant_dual   both 1x128 directions from one read of a 16640 x 8192 bf16 matrix
  quant_tile   128x128 quantization (with transposed copy) of a 32768 x 32768 bf16 matrix
  gemm_tiny            256 x 512 x 1024, 1x128 x 128x128, bf16 out (the tiny blockwise case)
  gemm_pertensor_small 256 x 4096 x 1024 per-tensor scales, bf16 out
  gemm_rowwise_small   256 x 4096 x 1024 rowwise scales, bf16 out
  quant_rows_<n>, quant_tile_<n>   the quantization sweep at n x n bf16 (n = 1024 ... 32768)
With --time, each launch is timed with CUDA events and the mean is printed.

  python profile_cases.py configs [--reps R] [--graph]

times every case above (the median of three rounds of R timed launches each)
and prints one table; with --graph each round replays a CUDA graph of the R
launches (device time, without the host's per-call work).
"""
from __future__ import annotations

import argparse
import sys

import torch

from fp8_block_scaled_11_b200 import inputs, ops


# block recipe -> the same recipe with power-of-two scales (block-scaled MMA)
_POW2_MODE = {ops.SCALE_BLOCK_1x128_128x128: ops.SCALE_BLOCK_1x128_128x128_POW2,
              ops.SCALE_BLOCK_1x128_1x128: ops.SCALE_BLOCK_1x128_1x128_POW2}


def _gemm_case(name):
    M = inputs.LLAMA4_M
    # "<case>_pow2": the case's operands quantized with the power-of-two rule,
    # multiplied by the power-of-two recipe
    pow2 = name.endswith("_pow2")
    if pow2:
        name = name[:-len("_pow2")]
    R = ops.SCALE_RULE_POW2 if pow2 else ops.SCALE_RULE_FP32
    if name == "gemm_tiny":
        A, Bt = inputs.tiny_blockwise()
        qa, sa = ops.fp8_quant_1x128(A.cuda())
        qb, sb, _, _ = ops.fp8_quant_128x128(Bt.cuda())
        mode = ops.SCALE_BLOCK_1x128_128x128
        out = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * 256 * 512 * 1024
    elif name in ("gemm_pertensor_small", "gemm_rowwise_small"):
        x, W = inputs.per_tensor()
        xd, Wd = x.cuda(), W.cuda()
        if name == "gemm_pertensor_small":
            (qa, sa), (qb, sb) = ops.fp8_quant_tensor(xd), ops.fp8_quant_tensor(Wd)
            mode = ops.SCALE_TENSOR
        else:
            (qa, sa), (qb, sb) = ops.fp8_quant_rowwise(xd), ops.fp8_quant_rowwise(Wd)
            mode = ops.SCALE_ROWWISE
        out = torch.empty((256, 4096), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * 256 * 4096 * 1024
    elif name in ("gemm_fwd", "gemm_tensor", "gemm_rowwise"):
        x, W, _ = inputs.llama4(5120, 8192)
        x, W = x.cuda(), W.cuda()
        if name == "gemm_fwd":
            qa, sa = ops.fp8_quant_1x128(x, rule=R)
            qb, sb, _, _ = ops.fp8_quant_128x128(W, rule=R)
            mode = ops.SCALE_BLOCK_1x128_128x128
        elif name == "gemm_rowwise":
            (qa, sa), (qb, sb) = ops.fp8_quant_rowwise(x), ops.fp8_quant_rowwise(W)
            mode = ops.SCALE_ROWWISE
        else:
            qa, sa = ops.fp8_quant_tensor(x)
            qb, sb = ops.fp8_quant_tensor(W)
            mode = ops.SCALE_TENSOR
        out = torch.empty((M, 5120), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * M * 5120 * 8192
    elif name in ("gemm_dgrad", "gemm_dgrad_wt"):
        _, W, dy = inputs.llama4(5120, 8192)
        qa, sa = ops.fp8_quant_1x128(dy.cuda(), rule=R)
        mode = ops.SCALE_BLOCK_1x128_128x128
        out = torch.empty((M, 8192), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * M * 8192 * 5120
        if name == "gemm_dgrad":
            # W_q read in its stored orientation (MN-major B)
            qw, sw, _, _ = ops.fp8_quant_128x128(W.cuda())
            torch.cuda.synchronize()
            return (lambda: ops.fp8_scaled_gemm_ex(qa, qw, ops.MAJOR_MN, sa, sw, mode, out=out)), flops, "TFLOP/s"
        _, _, qb, sb = ops.fp8_quant_128x128(W.cuda(), want_q=False, want_qt=True, rule=R)
    elif name == "gemm_wgrad":
        x, _, dy = inputs.llama4(5120, 8192)
        qa, sa = ops.fp8_quant_1x128(dy.cuda(), transpose_out=True, rule=R)
        qb, sb = ops.fp8_quant_1x128(x.cuda(), transpose_out=True, rule=R)
        mode = ops.SCALE_BLOCK_1x128_1x128
        out = torch.empty((5120, 8192), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * M * 5120 * 8192
    elif name == "gemm_longk_mn":
        # x (K x 512) quantized 128x128 as stored and read MN-major
        goT, x = inputs.long_k(128128)
        qa, sa = ops.fp8_quant_1x128(goT.cuda())
        qb, sb, _, _ = ops.fp8_quant_128x128(x.cuda())
        mode = ops.SCALE_BLOCK_1x128_128x128
        out = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * 256 * 512 * 128128
        ws = ops.fp8_scaled_gemm_workspace_size(256, 512, 128128, mode)
        wsb = torch.empty((max(ws, 16),), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        return (lambda: ops.fp8_scaled_gemm_ex(qa, qb, ops.MAJOR_MN, sa, sb, mode, out=out, workspace=wsb)), flops, \
            "TFLOP/s"
    elif name == "gemm_longk_1x128":
        goT, x = inputs.long_k(128128)
        qa, sa = ops.fp8_quant_1x128(goT.cuda(), rule=R)
        qb, sb = ops.fp8_quant_1x128(x.cuda(), transpose_out=True, rule=R)
        mode = ops.SCALE_BLOCK_1x128_1x128
        out = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * 256 * 512 * 128128
    else:
        goT, x = inputs.long_k(128128)
        qa, sa = ops.fp8_quant_1x128(goT.cuda(), rule=R)
        _, _, qb, sb = ops.fp8_quant_128x128(x.cuda(), want_q=False, want_qt=True, rule=R)
        mode = ops.SCALE_BLOCK_1x128_128x128
        out = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
        flops = 2.0 * 256 * 512 * 128128
    if pow2:
        mode = _POW2_MODE[mode]
    ws = ops.fp8_scaled_gemm_workspace_size(qa.shape[0], qb.shape[0], qa.shape[1], mode)
    wsb = torch.empty((max(ws, 16),), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    return (lambda: ops.fp8_scaled_gemm(qa, qb, sa, sb, mode, out=out, workspace=wsb)), flops, "TFLOP/s"


def _grouped_case(name):
    """8 groups over the Llama4 layer shape (N, K) = (5120, 8192), 16640 tokens:
    equal counts (gemm_grouped) or ragged ones (gemm_grouped_ragged)."""
    rows = [2080] * 8 if name == "gemm_grouped" else [4000, 1, 127, 129, 3000, 0, 5000, 4383]
    N, K, G = 5120, 8192, len(rows)
    x = inputs.random_matrix(sum(rows), K, seed=11, dtype=torch.bfloat16).cuda()
    W = inputs.random_matrix(G * N, K, seed=12, dtype=torch.bfloat16, scale=K ** -0.5).cuda()
    qa, sa = ops.fp8_quant_1x128(x)
    qb = torch.empty((G * N, K), dtype=torch.uint8, device="cuda")
    sb = ops.grouped_scale_grids(G, N, K, "cuda")
    for g in range(G):
        ops.fp8_quant_128x128(W[g * N:(g + 1) * N], out=(qb[g * N:(g + 1) * N], ops.grouped_grid_view(sb, g, N),
                                                          None, None))
    out = torch.empty((sum(rows), N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    return (lambda: ops.fp8_scaled_gemm_grouped(qa, qb, rows, sa, sb, N, out=out)), 2.0 * sum(rows) * N * K, \
        "TFLOP/s"


def _fused_case(name):
    x, W, _ = inputs.llama4(5120, 8192)
    qa, sa = ops.fp8_quant_1x128(x.cuda())
    qb, sb, _, _ = ops.fp8_quant_128x128(W.cuda())
    mode = ops.SCALE_BLOCK_1x128_128x128
    M = inputs.LLAMA4_M
    y = torch.empty((M, 5120), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((M, 5120), dtype=torch.uint8, device="cuda")
    s = ops.colmajor_grid(M, 40, "cuda")
    flops = 2.0 * M * 5120 * 8192
    if name == "gemm_fwd_then_quant":
        def fn():
            ops.fp8_scaled_gemm(qa, qb, sa, sb, mode, out=y)
            ops.fp8_quant_1x128(y, q=q, scale_inv=s)
    else:
        store = name == "gemm_fwd_quant"
        fn = lambda: ops.fp8_scaled_gemm_quant(qa, qb, sa, sb, mode, out=y, store_out=store, q_out=q, scale_out=s)
    torch.cuda.synchronize()
    return fn, flops, "TFLOP/s"


def _quant_case(name):
    parts = name.split("_")
    if len(parts) == 3 and parts[2].isdigit():
        # the quantization sweep: quant_rows_<n> / quant_tile_<n>
        n = int(parts[2])
        x = inputs.quant_sweep(n).cuda()
        if parts[1] == "rows":
            q, s = ops.fp8_quant_1x128(x)
            nbytes = x.numel() * 3 + 4 * s.numel()
            fn = lambda: ops.fp8_quant_1x128(x, q=q, scale_inv=s)
        else:
            out = ops.fp8_quant_128x128(x)
            nbytes = x.numel() * 3 + 4 * out[1].numel()
            fn = lambda: ops.fp8_quant_128x128(x, out=out)
        torch.cuda.synchronize()
        return fn, nbytes, "GB/s"
    if name == "quant_cols":
        x = inputs.llama4(5120, 8192)[0].cuda()
        q, s = ops.fp8_quant_1x128(x, transpose_out=True)
        nbytes = x.numel() * 3 + 4 * s.numel()
        fn = lambda: ops.fp8_quant_1x128(x, transpose_out=True, q=q, scale_inv=s)
    elif name == "quant_dual":
        x = inputs.llama4(5120, 8192)[0].cuda()
        out = ops.fp8_quant_1x128_dual(x)
        nbytes = x.numel() * 4 + 4 * (out[1].numel() + out[3].numel())
        fn = lambda: ops.fp8_quant_1x128_dual(x, out=out)
    else:
        x = inputs.quant_sweep(32768).cuda()
        if name == "quant_rows":
            q, s = ops.fp8_quant_1x128(x)
            nbytes = x.numel() * 3 + 4 * s.numel()
            fn = lambda: ops.fp8_quant_1x128(x, q=q, scale_inv=s)
        else:
            out = ops.fp8_quant_128x128(x, want_q=True, want_qt=True)
            nbytes = x.numel() * 4 + 8 * out[1].numel()
            fn = lambda: ops.fp8_quant_128x128(x, want_q=True, want_qt=True, out=out)
    torch.cuda.synchronize()
    return fn, nbytes, "GB/s"


CONFIG_CASES = (["gemm_tiny", "gemm_pertensor_small", "gemm_rowwise_small", "gemm_fwd", "gemm_dgrad", "gemm_dgrad_wt",
                 "gemm_wgrad", "gemm_tensor", "gemm_rowwise", "gemm_longk", "gemm_fwd_then_quant",
                 "gemm_fwd_quant", "gemm_fwd_quant_only", "gemm_longk_mn", "gemm_grouped", "gemm_grouped_ragged",
                 "gemm_longk_1x128", "gemm_fwd_pow2", "gemm_dgrad_wt_pow2", "gemm_wgrad_pow2", "gemm_longk_pow2",
                 "gemm_longk_1x128_pow2", "quant_dual"]
                + [f"quant_rows_{n}" for n in inputs.QUANT_SWEEP_SIZES]
                + [f"quant_tile_{n}" for n in inputs.QUANT_SWEEP_SIZES])


def _case(name):
    if name in ("gemm_fwd_quant", "gemm_fwd_quant_only", "gemm_fwd_then_quant"):
        return _fused_case(name)
    if name in ("gemm_grouped", "gemm_grouped_ragged"):
        return _grouped_case(name)
    return _gemm_case(name) if name.startswith("gemm") else _quant_case(name)


def _time(case, reps, graph=False):
    """Median of three rounds of `reps` back-to-back launches, ms per launch.
    graph=True: the rounds replay a CUDA graph of the `reps` launches, so the
    host's per-call work (argument checks, tensor-map encoding) is not in the
    timed region -- the device-side time of launch-bound cases."""
    fn, work, unit = _case(case)
    fn()
    torch.cuda.synchronize()
    run = fn
    if graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        run = g.replay
    rounds = []
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        if graph:
            run()
        else:
            for _ in range(reps):
                run()
        b.record()
        torch.cuda.synchronize()
        rounds.append(a.elapsed_time(b) / reps)
    st = ops.fp8bs_check_device_error()
    if st != 0:
        raise RuntimeError(f"{case}: {ops.fp8bs_status_string(st)}")
    ms = sorted(rounds)[1]
    return ms, work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9), unit


def configs(reps, graph=False):
    print(f"{'case':22s} {'us/launch':>10s} {'rate':>10s}" + ("  (CUDA graph)" if graph else ""))
    for case in CONFIG_CASES:
        try:
            ms, rate, unit = _time(case, reps, graph)
        except RuntimeError as e:            # a launch sequence that a graph cannot capture
            if not graph:
                raise
            print(f"{case:22s} {'n/a':>10s} ({str(e).splitlines()[0][:60]})")
            torch.cuda.synchronize()
            continue
        print(f"{case:22s} {ms * 1e3:10.1f} {rate:10.1f} {unit}")
        torch.cuda.empty_cache()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--graph", action="store_true", help="configs: time replays of a CUDA graph of the launches")
    a = ap.parse_args(argv)
    if a.case == "configs":
        return configs(a.reps, a.graph)
    fn, work, unit = _case(a.case)
    fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * a.reps)]
    for i in range(a.reps):
        if a.time:
            ev[2 * i].record()
        fn()
        if a.time:
            ev[2 * i + 1].record()
    torch.cuda.synchronize()
    st = ops.fp8bs_check_device_error()
    if st != 0:
        print(ops.fp8bs_status_string(st), file=sys.stderr)
        return 1
    if a.time:
        ms = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(a.reps)]
        mean = sum(ms) / len(ms)
        rate = work / (mean * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
        print(f"{a.case}: {mean * 1e3:.1f} us/launch (mean of {a.reps}), {rate:.1f} {unit}")
    return 0


if __name__ == "__main__":
    sys.exit(main())

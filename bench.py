"""Benchmark of the FP8 blockwise hot path on B200.

One step = the Llama4-shape FP8 linear forward + backward for both layer
shapes (N, K) = (5120, 8192) and (8192, 5120) at M = 16640 tokens: per shape
five dynamic-quantization launches (x 1x128, x^T along tokens, W 128x128 with
its transpose, dy 1x128, dy^T along tokens) and three scaled GEMMs (forward
and dgrad with 1x128 x 128x128 scales, wgrad with 1x128 x 1x128), bf16 out.
This is the workload of pytorch/ao PR #2785 "integrate torch._scaled_mm into
Float8BlockwiseLinear and add bench script" (Benchmarks table).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one process per GPU): every rank runs the same per-GPU
workload on its own batch (weak scaling, no collective on the data path); the
time is the max over ranks.  `--impl reference` times the CPU oracle instead
(rank 0 only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "blockwise FP8 GEMM TFLOP/s (% of B200 FP8 peak); quant GB/s (% of HBM)"
UNIT = "TFLOP/s"
# The pages' own figure for this workload: fp8 torch._scaled_mm eager fwd+bwd,
# 7746.98 us at (5120, 8192) and 7783.31 us at (8192, 5120), hardware not stated.
PAGES_FP8_US = (7746.98, 7783.31)
FP8_SPEC_TFLOPS = 4500.0

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of each
# GEMM of the step, from an ncu capture, keyed by a hash of the sources of the
# kernel the step's GEMMs run on (the single-CTA GEMM).  A changed kernel
# reports null until it is captured again; an old figure is never re-keyed to
# new sources.
GEMM_TRAFFIC = {
    # ncu 1-pass launch list of `bench.py --steps 2 --warmup 3 --no-e2e --no-cpu-baseline
    # --sustained-s 0 --no-ablation`, mean of the two timed steps
    "266e9182b27a3e3e": {
        "fwd 16640x5120x8192": 570.9e6, "dgrad 16640x8192x5120": 559.9e6, "wgrad 5120x8192x16640": 812.9e6,
        "fwd 16640x8192x5120": 558.5e6, "dgrad 16640x5120x8192": 566.8e6, "wgrad 8192x5120x16640": 834.5e6,
    },
}
GEMM_SOURCES = ("gemm_kernel.cuh", "ptx.cuh")


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (ms) across the process group;
    identity on one rank.  Every rank must call it at the same point."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def throughput_tflops(world, flops_per_step_per_rank, steps, ms_max):
    """Whole-job throughput under weak scaling: all ranks' flops over the
    slowest rank's time."""
    return world * flops_per_step_per_rank * steps / (ms_max * 1e-3) / 1e12


def kernel_hash():
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "fp8_block_scaled_11_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling: every 20 ms from start() to
    stop(); only the samples whose timestamps fall inside the timed region
    [t_begin, t_end] (host wall-clock seconds) are reported."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
            return
        # the timed region starts only once samples are flowing (nvidia-smi can
        # take a while to print its first one)
        t_end = time.time() + 5.0
        while len(self.lines) < 2 and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    @staticmethod
    def parse(lines, t_begin, t_end):
        """Median SM clock, max clock, median power and the throttle reasons
        seen, over the samples taken inside [t_begin, t_end]."""
        mhz, mx, pw, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, cmax, power = float(parts[2]), float(parts[3]), float(parts[4])
            except ValueError:
                continue
            if not (t_begin <= ts <= t_end):
                continue
            mhz.append(clk)
            mx.append(cmax)
            pw.append(power)
            for nm, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w": statistics.median(pw) if pw else None, "reasons": sorted(reasons),
                "samples": len(mhz), "period_ms": ClockSampler.PERIOD_MS}

    def stop(self, t_begin: float, t_end: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        return self.parse(self.lines, t_begin, t_end)


# ------------------------------------------------------------------------ GPU arm
def run_gpu(args):
    import torch
    import torch.distributed as dist

    from fp8_block_scaled_11_b200 import inputs, ops
    from fp8_block_scaled_11_b200.linear import Fp8LinearStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ops.lib()
    M = inputs.LLAMA4_M
    shapes = inputs.LLAMA4_SHAPES
    steps = [Fp8LinearStep(M, N, K) for N, K in shapes]
    data = []
    for N, K in shapes:
        x, W, dy = inputs.llama4(N, K)
        data.append((x, W, dy))
    dev_data = [tuple(t.cuda() for t in d) for d in data]
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    def one_step(events=None):
        for st, (x, W, dy) in zip(steps, dev_data):
            if events is None:
                st.run(x, W, dy)
            else:
                # events: before quantization, then before / after each GEMM
                e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
                e[0].record(stream)
                st.quantize(x, W, dy)
                st.gemms(mark=lambda i: e[1 + i].record(stream))
                events.append((st, e))

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    st_err = ops.fp8bs_check_device_error()
    if st_err != 0:
        raise SystemExit(f"device error after warm-up: {ops.fp8bs_status_string(st_err)}")

    # ---- timed region: K steps, CUDA events on the launching stream
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    events = []
    wall0 = time.time()
    t0.record(stream)
    for _ in range(args.steps):
        one_step(events)
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier()
    clocks = sampler.stop(wall0, wall1)
    ms_total = t0.elapsed_time(t1)
    quant_ms = sum(e[0].elapsed_time(e[1]) for _, e in events)
    gemm_ms = sum(e[1].elapsed_time(e[4]) for _, e in events)
    # per GEMM of the step (layer shape i, GEMM g = fwd / dgrad / wgrad): summed event time
    per_gemm_ms = [sum(e[1 + g].elapsed_time(e[2 + g]) for st, e in events if st is steps[i])
                   for i in range(len(steps)) for g in range(3)]
    vals = max_over_ranks([ms_total, quant_ms, gemm_ms] + per_gemm_ms, world, "cuda")
    ms_total, quant_ms, gemm_ms, per_gemm_ms = vals[0], vals[1], vals[2], vals[3:]
    fwd_ms = per_gemm_ms[0]

    flops_step = sum(st.flops() for st in steps)
    qbytes_step = sum(st.quant_bytes() for st in steps)
    ms_step = ms_total / args.steps
    value = throughput_tflops(world, flops_step, args.steps, ms_total)
    gemm_tflops = throughput_tflops(1, flops_step, args.steps, gemm_ms)
    fwd_avg_us = fwd_ms * 1e3 / args.steps
    fwd_tflops = steps[0].gemm_flops() / (fwd_avg_us * 1e-6) / 1e12
    quant_gbs = qbytes_step * args.steps / (quant_ms * 1e-3) / 1e9

    peaks, peak_src = measured_peaks()
    timed_region_s = ms_total * 1e-3
    sustained = timed_region_s > 2.0
    bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    fp8_peak = 2.0 * bf16          # fp8 / bf16 dense ratio 4.5 / 2.25
    traffic = GEMM_TRAFFIC.get(kernel_hash(), {})
    gemm_list = gemm_roofline_list(steps, per_gemm_ms, args.steps, fp8_peak, traffic)
    tr = gemm_list[0]["traffic"]

    # ---- sustained: the same step back to back for several seconds (the GPU
    # settles under its power cap), against the sustained peak
    sus = None
    if args.sustained_s > 0:
        sus = run_sustained(args, world, local, one_step, steps, flops_step, peaks, barrier)

    # ---- end to end: host (pinned) inputs -> device, the step, results -> host
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, world, steps, shapes, data, flops_step, barrier)

    # ---- the fast-accumulation ablation: the same step with power-of-two
    # scales on the block-scaled MMA (no per-K-block promotion)
    abl = None
    if not args.no_ablation:
        abl = run_ablation(args, world, dev_data, shapes, barrier, ms_step, per_gemm_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(args.cpu_rows)

    pages_tflops = 2 * 3 * 2.0 * M * 5120 * 8192 / (sum(PAGES_FP8_US) * 1e-6) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": round(value / world / pages_tflops, 3),
        "dtype": "e4m3 x e4m3 -> fp32 accumulate, bf16 out", "data": "synthetic (seeded N(0,1) / kaiming-uniform bf16)",
        "config": {
            "workload": "Llama4-shape FP8 linear fwd+bwd, M=16640, (N,K)=(5120,8192) and (8192,5120); "
                        "fwd/dgrad 1x128 x 128x128 (dgrad reads W_q as stored, MN-major), wgrad 1x128 x 1x128 "
                        "(along tokens); dynamic quant included",
            "parallelism": f"dp{world} (independent per-GPU batches, no data-path collective)",
            "l2": "inputs larger than L2 (x alone is 272 MB); no flush",
            "vs_baseline_ref": f"pages' fp8 _scaled_mm eager fwd+bwd ({PAGES_FP8_US[0]}+{PAGES_FP8_US[1]} us, "
                               f"hardware not stated) = {pages_tflops:.1f} TFLOP/s per GPU",
        },
        "breakdown": {
            "gemm_tflops": round(gemm_tflops, 1),
            "gemm_frac_of_fp8_spec": round(gemm_tflops / FP8_SPEC_TFLOPS, 3),
            "quant_gbs": round(quant_gbs, 1),
            "quant_frac_of_hbm": round(quant_gbs / peaks["hbm_gbs"], 3),
            "quant_ms_per_step": round(quant_ms / args.steps, 4),
            "gemm_ms_per_step": round(gemm_ms / args.steps, 4),
        },
        "roofline": {
            "kernel": "gemm_fp8_kernel<1x128 x 128x128>, forward GEMM 16640 x 5120 x 8192 (bf16 out)",
            "bound": "tensor", "achieved": round(fwd_tflops, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
            "frac": round(fwd_tflops / fp8_peak, 3), "traffic": tr,
            "algorithmic_per_launch": f"{steps[0].gemm_flops():.4g} flop; 348.6 MB (operands + bf16 output)",
            "peak_source": f"2 x {'sustained' if sustained else 'burst'} bf16 of {peak_src} "
                           f"({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'fallback'}), fp8/bf16 ratio 2",
            "avg_launch_us": round(fwd_avg_us, 1),
        },
        "roofline_gemms": gemm_list,
        "sustained": sus,
        "fast_accum_ablation": abl,
        "clocks": clocks,
        "gpu_launches": Fp8LinearStep.LAUNCHES_PER_STEP * len(steps) * args.steps,
        "e2e": e2e,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


GEMM_NAMES = ("fwd", "dgrad", "wgrad")


def gemm_shapes(st):
    """(M, N, K) of the step's fwd, dgrad and wgrad GEMMs and their recipes."""
    M, N, K = st.M, st.N, st.K
    return ((M, N, K, "1x128 x 128x128"), (M, K, N, "1x128 x 128x128"), (N, K, M, "1x128 x 1x128"))


def gemm_algorithmic_bytes(M, N, K, recipe):
    """Operands read once (e4m3), scales read once, bf16 output written once."""
    kb, nb = (K + 127) // 128, (N + 127) // 128
    sb = nb * kb if recipe == "1x128 x 128x128" else N * kb
    return M * K + N * K + 4 * (M * kb + sb) + 2 * M * N


def gemm_roofline_list(steps, per_gemm_ms, nsteps, fp8_peak, traffic):
    out = []
    for i, st in enumerate(steps):
        for g, (M, N, K, recipe) in enumerate(gemm_shapes(st)):
            us = per_gemm_ms[3 * i + g] * 1e3 / nsteps
            tflops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            key = f"{GEMM_NAMES[g]} {M}x{N}x{K}"
            out.append({"gemm": key, "recipe": recipe,
                        "kernel": ("gemm_fp8_kernel<3>" if g == 2 else
                                   "gemm_fp8_kernel<2>, B MN-major" if g == 1 else "gemm_fp8_kernel<2>"),
                        "bound": "tensor", "avg_launch_us": round(us, 1), "achieved": round(tflops, 1),
                        "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(tflops / fp8_peak, 3),
                        "algorithmic_bytes": gemm_algorithmic_bytes(M, N, K, recipe),
                        "traffic": traffic.get(key)})
    return out


def run_ablation(args, world, dev_data, shapes, barrier, promoted_ms_step, promoted_gemm_ms):
    """The step with every scale rounded down to a power of two and the GEMMs
    on the block-scaled MMA (whole-K fp32 accumulation in TMEM): W warm-up
    and K timed steps with per-GEMM CUDA events, as the main measurement.
    The accuracy side of the ablation is the parity tests' (against the oracle
    with the same power-of-two rule)."""
    import torch
    from fp8_block_scaled_11_b200 import inputs, ops
    from fp8_block_scaled_11_b200.linear import Fp8LinearStep

    M = inputs.LLAMA4_M
    steps = [Fp8LinearStep(M, N, K, pow2=True, dgrad_wt_copy=True) for N, K in shapes]
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        for st, (x, W, dy) in zip(steps, dev_data):
            st.run(x, W, dy)
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    events = []
    t0.record(stream)
    for _ in range(args.steps):
        for st, (x, W, dy) in zip(steps, dev_data):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            st.quantize(x, W, dy)
            st.gemms(mark=lambda i: e[i].record(stream))
            events.append((st, e))
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    st_err = ops.fp8bs_check_device_error()
    if st_err != 0:
        raise SystemExit(f"device error in the ablation: {ops.fp8bs_status_string(st_err)}")
    per_gemm = [sum(e[g].elapsed_time(e[g + 1]) for st, e in events if st is steps[i])
                for i in range(len(steps)) for g in range(3)]
    vals = max_over_ranks([t0.elapsed_time(t1)] + per_gemm, world, "cuda")
    ms_step = vals[0] / args.steps
    per_gemm = vals[1:]
    flops_step = sum(st.flops() for st in steps)
    names = [f"{GEMM_NAMES[g]} {M_}x{N_}x{K_}" for st in steps
             for g, (M_, N_, K_, _) in enumerate(gemm_shapes(st))]
    return {
        "recipe": "the step's recipes with power-of-two (UE8M0) scales: tcgen05.mma kind::mxf8f6f4.block_scale, "
                  "whole-K fp32 accumulation in TMEM, no per-K-block promotion (gemm_fp8_bs_kernel)",
        "ms_per_step": round(ms_step, 4),
        "value": round(world * flops_step / (ms_step * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "step_speedup_vs_promoted": round(promoted_ms_step / ms_step, 3),
        "gemm_us": {n: round(v * 1e3 / args.steps, 1) for n, v in zip(names, per_gemm)},
        "gemm_speedup_vs_promoted": {n: round(a / b, 3) for n, a, b in zip(names, promoted_gemm_ms, per_gemm)},
    }


def run_sustained(args, world, local, one_step, steps, flops_step, peaks, barrier):
    """The step back to back for at least args.sustained_s seconds of device
    time (no per-GEMM events inside, one pair of events around each block of
    steps), with its own clock record; the forward GEMM's share comes from a
    final evented step.  Peak: 2 x the sustained bf16 figure."""
    import torch
    stream = torch.cuda.current_stream()
    # steps per block sized from one timed step
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    one_step()
    b.record(stream)
    torch.cuda.synchronize()
    est_ms = max(a.elapsed_time(b), 0.1)
    block = max(1, int(200.0 / est_ms))
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    total_ms, nsteps = 0.0, 0
    while total_ms < args.sustained_s * 1e3:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(block):
            one_step()
        b.record(stream)
        b.synchronize()
        total_ms += a.elapsed_time(b)
        nsteps += block
    # the last blocks' steps carry the settled clocks: time one more evented step
    ev = []
    one_step(ev)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier()
    clocks = sampler.stop(wall0, wall1)
    fwd_us = ev[0][1][1].elapsed_time(ev[0][1][2]) * 1e3
    total_ms, fwd_us = max_over_ranks([total_ms, fwd_us], world, "cuda")
    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]
    fwd_tflops = steps[0].gemm_flops() / (fwd_us * 1e-6) / 1e12
    return {"seconds": round(total_ms * 1e-3, 2), "steps": nsteps, "ms_per_step": round(total_ms / nsteps, 4),
            "value": round(throughput_tflops(world, flops_step, nsteps, total_ms), 2), "unit": UNIT,
            "fwd_gemm_us": round(fwd_us, 1), "fwd_gemm_tflops": round(fwd_tflops, 1),
            "fwd_frac_of_sustained_peak": round(fwd_tflops / fp8_peak, 3),
            "peak": round(fp8_peak, 1), "peak_source": "2 x bf16_tflops_sustained (MEASURED_PEAKS.json)",
            "clocks": clocks}


def run_e2e(args, world, steps, shapes, data, flops_step, barrier):
    """End to end through the public API from pinned host memory: every step
    copies its inputs host -> device, runs the quantization + GEMMs, and reads
    all three results back.  Copies overlap compute as a pipelined trainer
    would: inputs of step i+1 upload (copy stream) and outputs of step i-1
    download (second copy stream) while step i computes, on two device
    buffer sets; events order each set's reuse."""
    import torch

    from fp8_block_scaled_11_b200.linear import Fp8LinearStep

    M = steps[0].M
    host_in = [tuple(t.pin_memory() for t in d) for d in data]
    host_out = [tuple(torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in (st.y, st.dx, st.dW))
                for st in steps]
    # buffer set 0 reuses the benchmark's step objects, set 1 is a second copy
    sets = [steps, [Fp8LinearStep(M, N, K) for N, K in shapes]]
    dev_in = [[tuple(torch.empty_like(t, device="cuda") for t in d) for d in data] for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    n_e2e = max(2, min(args.steps, 10))

    def run(n):
        ev_in, ev_comp, ev_out = {}, {}, {}
        for i in range(n):
            k = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])          # set k's inputs no longer read
                for (xh, Wh, dyh), (xd, Wd, dyd) in zip(host_in, dev_in[k]):
                    xd.copy_(xh, non_blocking=True)
                    Wd.copy_(Wh, non_blocking=True)
                    dyd.copy_(dyh, non_blocking=True)
                ev_in[i] = torch.cuda.Event()
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[i])
                if i >= 2:
                    s_comp.wait_event(ev_out[i - 2])         # set k's outputs already read back
                for st, (xd, Wd, dyd) in zip(sets[k], dev_in[k]):
                    st.run(xd, Wd, dyd)
                ev_comp[i] = torch.cuda.Event()
                ev_comp[i].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                for st, outs in zip(sets[k], host_out):
                    for o, dsrc in zip(outs, (st.y, st.dx, st.dW)):
                        o.copy_(dsrc, non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record(s_out)
        return ev_out[n - 1]

    run(2)
    torch.cuda.synchronize()
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    last = run(n_e2e)
    s_in.wait_event(last)
    b.record(s_in)
    torch.cuda.synchronize()
    barrier()
    e_ms = max_over_ranks([a.elapsed_time(b)], world, "cuda")[0]
    bi = sum(sum(t.numel() * t.element_size() for t in d) for d in host_in)
    bo = sum(sum(t.numel() * t.element_size() for t in o) for o in host_out)
    return {"value": round(throughput_tflops(world, flops_step, n_e2e, e_ms), 2), "unit": UNIT,
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": n_e2e,
            "path": "pinned host tensors -> ops (C ABI) -> pinned host tensors; H2D, compute and D2H on "
                    "three streams with two device buffer sets"}


# ------------------------------------------------------------------------ oracle (CPU) arm
class OracleSample:
    """The oracle, as it stands, on a bounded sample of the same workload.  Per
    layer shape and per step: quantize (1x128) `rows` token rows of x and dy,
    the first 128-row band of W (128x128) and of W^T, and the first 128 rows of
    x^T and dy^T along all tokens; then compute, in fp64, output rows x the
    first 128 columns of the forward and dgrad GEMMs and the first 128 x 128
    block of the wgrad GEMM.  Value = the sampled GEMM FLOPs / wall time of the
    quantization + GEMM calls (input generation excluded)."""

    def __init__(self, rows: int):
        import numpy as np
        import torch

        import oracle
        from fp8_block_scaled_11_b200 import inputs

        oracle.lib()
        self.oracle = oracle
        self.rows = rows
        self.data = []
        for N, K in inputs.LLAMA4_SHAPES:
            x, W, dy = inputs.llama4(N, K)
            self.data.append((N, K, x.view(torch.uint16).numpy(), W.view(torch.uint16).numpy(),
                              dy.view(torch.uint16).numpy()))
        self.M = inputs.LLAMA4_M
        self.idx = np.arange(rows, dtype=np.int64)
        self.band = np.arange(128, dtype=np.int64)

    def step(self):
        o = self.oracle
        flops = 0.0
        t = time.perf_counter()
        for N, K, xb, Wb, dyb in self.data:
            qx, sx = o.quant_1x128(xb, rows=self.idx)
            qw, sw = o.quant_128x128(Wb, rblocks=[0])                  # W rows 0..127
            qwt, swt = o.quant_128x128(Wb, transpose=True, rblocks=[0])  # W^T rows 0..127
            qdy, sdy = o.quant_1x128(dyb, rows=self.idx)
            qdyt, sdyt = o.quant_1x128(dyb, transpose=True, rows=self.band)
            qxt, sxt = o.quant_1x128(xb, transpose=True, rows=self.band)
            o.gemm(qx, qw, sx, sw, o.SCALE_BLOCK_1x128_128x128)
            o.gemm(qdy, qwt, sdy, swt, o.SCALE_BLOCK_1x128_128x128)
            o.gemm(qdyt, qxt, sdyt, sxt, o.SCALE_BLOCK_1x128_1x128)
            flops += 2.0 * (self.rows * 128 * K + self.rows * 128 * N + 128 * 128 * self.M)
        secs = time.perf_counter() - t
        return flops, secs

    def describe(self):
        return (f"per layer shape and step: {self.rows} token rows x 128 output columns of fwd and dgrad, "
                f"a 128x128 block of wgrad over all 16640 tokens, with the quantization those need "
                f"(W / W^T 128-row bands, x / dy rows, x^T / dy^T 128-row bands); fp64 GEMM oracle")


def _cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline_sample(rows: int, budget_s: float = 12.0):
    """Timed oracle sample for the main line (about budget_s of CPU work)."""
    smp = OracleSample(rows)
    flops = secs = 0.0
    n = 0
    while secs < budget_s and n < 50:
        f, s_ = smp.step()
        flops += f
        secs += s_
        n += 1
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "seconds": round(secs, 2), "sample": f"{n} sampled steps; " + smp.describe()}


def run_oracle_configs(args):
    """The CPU oracle, as it stands, timed on every workload of the benchmark
    set on this host's cores (input generation excluded): the tiny blockwise
    GEMM, the per-tensor and rowwise GEMMs, the quantization sweep (both block
    shapes, every size), the long-K GEMM at k_blocks 1001 (both recipes) in
    full, and the Llama4 step on its bounded sample (as the cpu_baseline leg).
    One JSON line per workload; then the tiny GEMM and the 4096^2 sweep point
    again on one thread (a child process with OMP_NUM_THREADS=1)."""
    import numpy as np
    import torch

    import oracle
    from fp8_block_scaled_11_b200 import inputs

    oracle.lib()
    only = set(args.oracle_subset.split(",")) if args.oracle_subset else None
    cores = _cores()

    def bits(t):
        t = t.contiguous()
        return t.view(torch.uint16).numpy() if t.dtype == torch.bfloat16 else t.numpy()

    def emit(workload, secs, work, unit, **extra):
        d = {"workload": workload, "oracle_s": round(secs, 3), "cores": cores, "rate": work / secs, "unit": unit}
        d.update(extra)
        print(json.dumps(d), flush=True)

    def timed(fn):
        t = time.perf_counter()
        r = fn()
        return r, time.perf_counter() - t

    if only is None or "tiny" in only:
        A, Bt = inputs.tiny_blockwise()
        Ab, Btb = bits(A), bits(Bt)

        def tiny():
            qa, sa = oracle.quant_1x128(Ab)
            qb, sb = oracle.quant_128x128(Btb)
            return oracle.gemm(qa, qb, sa, sb, oracle.SCALE_BLOCK_1x128_128x128)
        _, secs = timed(tiny)
        emit("tiny blockwise 256x512x1024 (quant + GEMM)", secs, 2.0 * 256 * 512 * 1024 / 1e12, "TFLOP/s")
    if only is None or "pertensor" in only:
        x, W = inputs.per_tensor()
        xb, Wb = bits(x), bits(W)
        for name, qf, mode in (("per-tensor", oracle.quant_tensor, oracle.SCALE_TENSOR),
                               ("rowwise", oracle.quant_rowwise, oracle.SCALE_ROWWISE)):
            def run():
                qx, sx = qf(xb)
                qw, sw = qf(Wb)
                return oracle.gemm(qx, qw, sx, sw, mode)
            _, secs = timed(run)
            emit(f"{name} 256x4096x1024 (quant + GEMM)", secs, 2.0 * 256 * 4096 * 1024 / 1e12, "TFLOP/s")
    sizes = inputs.QUANT_SWEEP_SIZES if only is None else [n for n in inputs.QUANT_SWEEP_SIZES
                                                           if f"sweep{n}" in only]
    for n in sizes:
        xb = bits(inputs.quant_sweep(n))
        for name, fn, sbytes in (("1x128", oracle.quant_1x128, 4 * n * ((n + 127) // 128)),
                                 ("128x128", oracle.quant_128x128, 4 * ((n + 127) // 128) ** 2)):
            _, secs = timed(lambda: fn(xb))
            emit(f"quant {name} {n}x{n} bf16", secs, (3.0 * n * n + sbytes) / 1e9, "GB/s")
        del xb
    if only is None or "longk" in only:
        K = 128128
        goT, x = inputs.long_k(K)
        gb, xb = bits(goT), bits(x)
        for name, mode in (("1x128 x 128x128", oracle.SCALE_BLOCK_1x128_128x128),
                           ("1x128 x 1x128", oracle.SCALE_BLOCK_1x128_1x128)):
            def run():
                qa, sa = oracle.quant_1x128(gb)
                if mode == oracle.SCALE_BLOCK_1x128_128x128:
                    qb, sb = oracle.quant_128x128(xb, transpose=True)
                else:
                    qb, sb = oracle.quant_1x128(xb, transpose=True)
                return oracle.gemm(qa, qb, sa, sb, mode)
            _, secs = timed(run)
            emit(f"long-K 256x512x{K} {name} (quant + GEMM)", secs, 2.0 * 256 * 512 * K / 1e12, "TFLOP/s")
    if only is None or "llama4" in only:
        smp = OracleSample(args.cpu_rows)
        flops, secs = smp.step()
        emit("Llama4 fwd+bwd step, bounded sample", secs, flops / 1e12, "TFLOP/s", sample=smp.describe())
    if only is None and os.environ.get("OMP_NUM_THREADS") != "1":
        env = dict(os.environ, OMP_NUM_THREADS="1")
        subprocess.run([sys.executable, os.path.abspath(__file__), "--oracle-configs",
                        "--oracle-subset", "tiny,sweep4096"], env=env, check=True)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    smp = OracleSample(args.cpu_rows)
    for _ in range(args.warmup):
        smp.step()
    flops = secs = 0.0
    for _ in range(args.steps):
        f, s_ = smp.step()
        flops += f
        secs += s_
    value = round(flops / secs / 1e12, 6)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3 / args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded N(0,1) / kaiming-uniform bf16)",
        "config": {"workload": "Llama4-shape FP8 linear fwd+bwd, M=16640, (N,K)=(5120,8192) and (8192,5120); "
                               "each step a bounded sample (see cpu_baseline.sample)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cores(), "kind": "oracle",
                         "sample": smp.describe()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)   # ~0.34 s timed: enough clock samples
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=32)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ablation", action="store_true",
                    help="skip the fast-accumulation ablation (power-of-two scales, block-scaled MMA)")
    ap.add_argument("--sustained-s", type=float, default=3.0,
                    help="seconds of back-to-back steps for the sustained-clock figure (0: skip)")
    ap.add_argument("--oracle-configs", action="store_true",
                    help="time the CPU oracle on every workload and print one JSON line per workload")
    ap.add_argument("--oracle-subset", default="", help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.oracle_configs:
        run_oracle_configs(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()

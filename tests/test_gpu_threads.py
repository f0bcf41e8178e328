"""Concurrent first use from several host threads: in a fresh process, eight
threads start at once on their own CUDA streams and each runs the
dual-direction quantization, the 128x128 quantization, a blockwise GEMM, the
same GEMM reading B MN-major, and the power-of-two quantizations with the
block-scaled GEMM (the library's per-device set-up and per-kernel launch
attributes are all first touched concurrently).  Every thread's results must equal the
single-threaded ones bit for bit."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys, threading
sys.path.insert(0, sys.argv[1])
import torch
from fp8_block_scaled_11_b200 import build, inputs, ops

build.build()
torch.cuda.init()
x = inputs.random_matrix(512, 1024, seed=61, dtype=torch.bfloat16).cuda()
W = inputs.random_matrix(768, 1024, seed=62, dtype=torch.bfloat16).cuda()
Wt = W.t().contiguous()
torch.cuda.synchronize()

def work():
    q, s, qt, st = ops.fp8_quant_1x128_dual(x)
    wq, ws, _, _ = ops.fp8_quant_128x128(W)
    y = ops.fp8_scaled_gemm(q, wq, s, ws, ops.SCALE_BLOCK_1x128_128x128, out_dtype=torch.float32)
    wk, wks, _, _ = ops.fp8_quant_128x128(Wt)
    ymn = ops.fp8_scaled_gemm_ex(q, wk, ops.MAJOR_MN, s, wks, ops.SCALE_BLOCK_1x128_128x128, out_dtype=torch.float32)
    q2, s2 = ops.fp8_quant_1x128(x, rule=ops.SCALE_RULE_POW2)
    w2, ws2, _, _ = ops.fp8_quant_128x128(W, rule=ops.SCALE_RULE_POW2)
    y2 = ops.fp8_scaled_gemm(q2, w2, s2, ws2, ops.SCALE_BLOCK_1x128_128x128_POW2, out_dtype=torch.float32)
    return [q, s, qt, st, wq, ws, y, wk, wks, ymn, q2, s2, w2, ws2, y2]

results, errors = [None] * 8, []
start = threading.Barrier(8)

def thread(i):
    try:
        stream = torch.cuda.Stream()
        start.wait()
        with torch.cuda.stream(stream):
            out = work()
        stream.synchronize()
        results[i] = [t.cpu() for t in out]
    except Exception as e:           # reported below
        errors.append(repr(e))

ts = [threading.Thread(target=thread, args=(i,)) for i in range(8)]
for t in ts: t.start()
for t in ts: t.join()
assert not errors, errors
assert ops.fp8bs_check_device_error() == 0
ref = [t.cpu() for t in work()]
torch.cuda.synchronize()
for r in results:
    for a, b in zip(r, ref):
        assert torch.equal(a.contiguous(), b.contiguous())
print("threads ok")
'''


def test_concurrent_first_use_from_threads():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "threads ok" in r.stdout

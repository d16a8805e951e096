"""Concurrent callers: four host threads, each on its own CUDA stream, make their
first calls into the library at the same time (a fresh process, so every
per-device cache is still empty) and must get exactly the results of a
single-threaded run.  ctypes drops the GIL during the foreign calls, so the
calls really overlap on the host.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, threading
sys.path.insert(0, sys.argv[1])
import torch
import rmsnorm_qknorm_b200 as qk
from rmsnorm_qknorm_b200 import workloads as W

def work(seed, stream):
    with torch.cuda.stream(stream):
        inp = W.make_qknorm_inputs("decode", seed=seed, device="cuda", tokens=96)
        qo, ko = qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], inp["n_seg"])
        p16 = qk.rmsnorm_partial_stats(inp["q"], 16)
        fx = W.make_flashnorm_inputs(seed=seed, device="cuda", M=192, K=256, N=768)
        Wf = qk.flashnorm_fold_weights(fx["w"], fx["W"])
        inv = torch.empty(192, dtype=torch.float32, device="cuda")
        y = qk.flashnorm_proj(fx["x"], Wf, fx["eps"], inv_rms_out=inv)
        wq, wk = W.make_qkv_norm_weights(256, 256, seed=seed, device="cuda")
        z = qk.qkv_proj_qknorm(fx["x"], Wf, 256, 256, 256, wq, wk, fx["eps"])
    stream.synchronize()
    return [t.cpu() for t in (qo, ko, p16, y, z)]

streams = [torch.cuda.Stream() for _ in range(4)]
start = threading.Barrier(4)
results = [None] * 4
errors = []
def run(i):
    try:
        start.wait()
        results[i] = work(i, streams[i])
    except Exception as e:  # reported below
        errors.append(repr(e))
threads = [threading.Thread(target=run, args=(i,)) for i in range(4)]
for t in threads: t.start()
for t in threads: t.join()
assert not errors, errors
for i in range(4):  # the same calls again, one thread at a time
    ref = work(i, streams[i])
    for a, b in zip(results[i], ref):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b), i
assert qk.load_library().qkn_check_device(None) == 0
print("ok")
'''


def test_concurrent_first_calls_match_serial(cuda_lib):
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-4000:]

"""The benchmark's end-to-end path for the projections: row chunks uploaded,
projected and downloaded on three overlapped streams must give exactly the
single device call's output (rows are independent and the kernels' per-row
arithmetic does not depend on the batch)."""
from __future__ import annotations

import importlib.util
import os

import pytest
import torch

import rmsnorm_qknorm_b200 as qk
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("M", [1000, 4099])
def test_host_pipeline_matches_device_call(cuda_lib, M):
    bench = _bench()
    dev = torch.device("cuda", 0)
    inp = W.make_flashnorm_inputs(seed=M, device=dev, M=M, K=512, N=768)
    Wf = qk.flashnorm_fold_weights(inp["w"], inp["W"])
    inv = torch.empty(M, dtype=torch.float32, device=dev)
    ref = qk.flashnorm_proj(inp["x"], Wf, inp["eps"], inv_rms_out=inv)
    wq, wk = W.make_qkv_norm_weights(256, 256, seed=M, device=dev)
    ref_qkv = qk.qkv_proj_qknorm(inp["x"], Wf, 256, 256, 256, wq, wk, inp["eps"])
    hx = inp["x"].cpu().pin_memory()
    hy = torch.empty(M, 768, dtype=torch.bfloat16).pin_memory()
    step = bench.host_pipeline(
        hx, hy, lambda dx, dy, dinv, _s: qk.flashnorm_proj(dx, Wf, inp["eps"], inv_rms_out=dinv, out=dy), dev)
    step(0)
    step(1)
    torch.cuda.synchronize()
    assert torch.equal(hy.view(torch.int16), ref.cpu().view(torch.int16))
    hz = torch.empty(M, 768, dtype=torch.bfloat16).pin_memory()
    step = bench.host_pipeline(
        hx, hz, lambda dx, dy, dinv, _s: qk.qkv_proj_qknorm(dx, Wf, 256, 256, 256, wq, wk, inp["eps"],
                                                            inv_rms_out=dinv, out=dy), dev)
    step(0)
    torch.cuda.synchronize()
    assert torch.equal(hz.view(torch.int16), ref_qkv.cpu().view(torch.int16))

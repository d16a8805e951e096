"""qknorm_fused_host: QK-Norm of rows held in host memory, streamed through a device workspace.

The chunked pipeline must give exactly what qknorm_fused gives on the same
rows on the device (same kernels, rows are independent), whatever the chunk
size, and hence the oracle's parity bar; results are compared bit for bit
with the device call and to 1 bf16 ulp with the fp64 oracle.
"""
from __future__ import annotations

import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import assert_bf16_close, assert_f32_close
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _device_ref(inp, wl):
    q, k = inp["q"].to(DEV), inp["k"].to(DEV)
    qo, ko = qk.qknorm_fused(q, k, inp["wq"].to(DEV), inp["wk"].to(DEV), wl.eps, wl.n_seg)
    torch.cuda.synchronize()
    return qo.cpu(), ko.cpu()


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("ws_rows", [1, 7, 1000])
def test_host_matches_device_call(cuda_lib, pinned, ws_rows):
    wl = W.QKNORM_WORKLOADS["prefill_gqa"]
    inp = W.make_qknorm_inputs(wl, seed=ws_rows, device="cpu", tokens=333)
    q, k = inp["q"], inp["k"]
    if pinned:
        q, k = q.pin_memory(), k.pin_memory()
    row_bytes = (wl.dq + wl.dk) * q.element_size()
    ws = torch.empty(3 * (ws_rows * row_bytes + 512), dtype=torch.uint8, device=DEV)
    qo, ko = qk.qknorm_fused_host(q, k, inp["wq"].to(DEV), inp["wk"].to(DEV), wl.eps, wl.n_seg, workspace=ws)
    torch.cuda.synchronize()
    rq, rk = _device_ref(inp, wl)
    assert torch.equal(qo.view(torch.int16), rq.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), rk.view(torch.int16))
    assert_bf16_close(qo, oracle.rmsnorm(inp["q"], inp["wq"], wl.eps), what="q")


def test_host_default_workspace_several_chunks(cuda_lib):
    # 3000 rows of 12 KiB: the default workspace holds 64 MiB chunks, but the
    # chunk is sized from the bytes moved (16 MiB here), so three chunks run
    wl = W.QKNORM_WORKLOADS["prefill_gqa"]
    inp = W.make_qknorm_inputs(wl, seed=11, device="cpu", tokens=3000)
    q, k = inp["q"].pin_memory(), inp["k"].pin_memory()
    qo, ko = qk.qknorm_fused_host(q, k, inp["wq"].to(DEV), inp["wk"].to(DEV), wl.eps, wl.n_seg)
    torch.cuda.synchronize()
    rq, rk = _device_ref(inp, wl)
    assert torch.equal(qo.view(torch.int16), rq.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), rk.view(torch.int16))


def test_host_in_place_fp32_q_only(cuda_lib):
    wl = W.QKNORM_WORKLOADS["tiny"]
    inp = W.make_qknorm_inputs(wl, seed=3, device="cpu", tokens=50)
    ref = oracle.rmsnorm(inp["q"], inp["wq"], wl.eps)
    q = inp["q"].clone().pin_memory()
    ws = torch.empty(3 * 16 * wl.dq * 4, dtype=torch.uint8, device=DEV)  # 16 rows per chunk
    out, none = qk.qknorm_fused_host(q, None, inp["wq"].to(DEV), None, wl.eps, wl.n_seg, q_out=q, workspace=ws)
    torch.cuda.synchronize()
    assert none is None and out.data_ptr() == q.data_ptr()
    assert_f32_close(q, ref, what="q in place")


def test_host_ordered_on_caller_stream(cuda_lib):
    # a side stream: the call's work starts after that stream's earlier work and ends before its later work
    wl = W.QKNORM_WORKLOADS["decode"]
    inp = W.make_qknorm_inputs(wl, seed=4, device="cpu")
    s = torch.cuda.Stream()
    wq, wk = inp["wq"].to(DEV), inp["wk"].to(DEV)
    with torch.cuda.stream(s):
        wq2 = torch.zeros_like(wq)
        wq2.copy_(wq)  # queued on s before the call: the call must see the copied weights
        qo, ko = qk.qknorm_fused_host(inp["q"].pin_memory(), inp["k"].pin_memory(), wq2, wk, wl.eps, wl.n_seg)
        done = torch.cuda.Event()
        done.record(s)
    done.synchronize()
    rq, rk = _device_ref(inp, wl)
    assert torch.equal(qo.view(torch.int16), rq.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), rk.view(torch.int16))


def test_host_empty(cuda_lib):
    wl = W.QKNORM_WORKLOADS["decode"]
    q = torch.empty((0, wl.dq), dtype=torch.bfloat16)
    w = torch.ones(wl.dq, dtype=torch.bfloat16, device=DEV)
    qo, _ = qk.qknorm_fused_host(q, None, w, None)
    assert qo.shape == (0, wl.dq)

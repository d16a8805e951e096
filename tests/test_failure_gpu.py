"""Bounded device-side waits, exercised without faulting the GPU.

A one-shot test hook makes one warp of the staged norm kernel skip the copies
of its first tile, so its mbarrier wait can never complete.  The wait must
give up on its own after the armed limit, record the failure in the device
error word, drain the copies it did issue and let the kernel exit; the host
then reads QKN_ERR_TIMEOUT from qkn_check_device, the word is cleared, and the
next (normal) call on the same context is correct.
"""
from __future__ import annotations

import ctypes
import time

import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import assert_bf16_close
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
QKN_OK, QKN_ERR_TIMEOUT = 0, 7


def _lib():
    lib = qk.load_library()
    lib.qkn_testing_arm_wait_fault.argtypes = [ctypes.c_uint64]
    lib.qkn_testing_arm_wait_fault.restype = ctypes.c_int
    return lib


def test_wait_gives_up_and_reports_timeout(cuda_lib):
    lib = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.qkn_check_device(stream) == QKN_OK  # clean before
    inp = W.make_qknorm_inputs("prefill_gqa", seed=5, device="cuda", tokens=2048)
    assert lib.qkn_testing_arm_wait_fault(50_000_000) == QKN_OK  # 50 ms limit
    t0 = time.time()
    qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], inp["n_seg"])
    st = lib.qkn_check_device(stream)  # synchronises the stream
    elapsed = time.time() - t0
    assert st == QKN_ERR_TIMEOUT, lib.qkn_last_error()
    assert b"gave up" in lib.qkn_last_error()
    assert elapsed < 10.0  # two limited waits (the stage and its drain), not a hang
    # the word is cleared and the context still works: a normal call is correct
    assert lib.qkn_check_device(stream) == QKN_OK
    qo, ko = qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], inp["n_seg"])
    assert lib.qkn_check_device(stream) == QKN_OK
    assert_bf16_close(qo, oracle.rmsnorm(inp["q"].cpu(), inp["wq"].cpu(), inp["eps"]), "after fault q")
    assert_bf16_close(ko, oracle.rmsnorm(inp["k"].cpu(), inp["wk"].cpu(), inp["eps"]), "after fault k")


def test_exchange_wait_gives_up_and_reports_timeout(cuda_lib):
    # the fused QKV kernel's cross-CTA exchange: one warp never counts itself in, so the
    # waits of its row block's q section run out; the kernel records it and returns
    lib = qk.load_library()
    lib.qkn_testing_arm_exchange_fault.argtypes = [ctypes.c_uint64]
    lib.qkn_testing_arm_exchange_fault.restype = ctypes.c_int
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.qkn_check_device(stream) == QKN_OK
    M, K, nq, nk, nv = 512, 256, 1024, 512, 256
    inp = W.make_flashnorm_inputs(seed=2, device="cuda", M=M, K=K, N=nq + nk + nv)
    wq, wk = W.make_qkv_norm_weights(nq, nk, device="cuda")
    Wf = qk.flashnorm_fold_weights(inp["w"], inp["W"])
    assert lib.qkn_testing_arm_exchange_fault(50_000_000) == QKN_OK  # 50 ms limit
    t0 = time.time()
    qk.qkv_proj_qknorm(inp["x"], Wf, nq, nk, nv, wq, wk, inp["eps"])
    st = lib.qkn_check_device(stream)
    elapsed = time.time() - t0
    assert st == QKN_ERR_TIMEOUT, lib.qkn_last_error()
    assert b"fused QKV 1" in lib.qkn_last_error()
    assert elapsed < 10.0
    assert lib.qkn_check_device(stream) == QKN_OK  # cleared
    # the next call on the same context is normal and correct
    y = qk.qkv_proj_qknorm(inp["x"], Wf, nq, nk, nv, wq, wk, inp["eps"])
    assert lib.qkn_check_device(stream) == QKN_OK
    ref = oracle.qkv_proj_qknorm(inp["x"].cpu(), inp["w"].cpu(), inp["W"].cpu(), wq.cpu(), wk.cpu(), nq, nk,
                                 inp["eps"], inp["eps"])
    yd = y.cpu().double().numpy()
    assert float(((yd - ref) ** 2).sum() ** 0.5 / (ref ** 2).sum() ** 0.5) <= 1e-2

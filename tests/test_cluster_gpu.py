"""GPU parity of the cluster path: rows spread over the CTAs of a thread-block cluster.

qknorm_fused and rmsnorm_partial_stats take it for 16-byte-aligned rows with
more than 8 segments that the staged kernel's shared-memory ring does not
hold (rows of more than about 40 KiB), and for rows wider than one CTA's
registers hold (more than 65536 bf16 / 32768 fp32 elements).  Each CTA forms
the partial sums of squares of the segments its slice touches and the CTAs
exchange only those scalars through distributed shared memory.  Bars as everywhere: bf16 within 1 ulp of
RNE(oracle), fp32 within 1e-5 relative, partial sums within 1e-5 relative,
bitwise identical between runs.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import assert_bf16_close, assert_f32_close
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(wl_name, T, dq, dk, n_seg, seed=0):
    wl = W.QKNORM_WORKLOADS[wl_name]
    inp = W.make_qknorm_inputs(wl, seed=seed, device="cpu", tokens=T, dq=dq, dk=dk)
    q, k = inp["q"].to(DEV), inp["k"].to(DEV)
    qo, ko = qk.qknorm_fused(q, k, inp["wq"].to(DEV), inp["wk"].to(DEV), wl.eps, n_seg)
    torch.cuda.synchronize()
    check = assert_f32_close if wl.dtype == "f32" else assert_bf16_close
    check(qo, oracle.rmsnorm(inp["q"], inp["wq"], wl.eps), what=f"q d={dq} n_seg={n_seg}")
    check(ko, oracle.rmsnorm(inp["k"], inp["wk"], wl.eps), what=f"k d={dk} n_seg={n_seg}")
    return q, k, inp, qo, ko


@pytest.mark.parametrize("wl_name", ["prefill_gqa", "tiny"])
@pytest.mark.parametrize("n_seg", [16, 64])
@pytest.mark.parametrize("dq", [4096, 32768])
def test_many_segments(cuda_lib, wl_name, n_seg, dq):
    # 16 and 64 segments (the register kernel stops at 8): q 4096 + k 1024 rows go
    # through the staged kernel's many-segment statistic, q rows of 32768 (64 / 128
    # KiB) through the cluster; ragged token count
    _run(wl_name, 37, dq, 1024, n_seg, seed=n_seg)


@pytest.mark.parametrize("wl_name,dq,dk,n_seg", [
    ("prefill_gqa", 81920, 4096, 8),     # bf16, 10240 chunks: 8 CTAs of 1280
    ("prefill_gqa", 131072, 256, 4),     # bf16, the widest row one cluster holds (8 x 2048 chunks)
    ("prefill_gqa", 65600, 72, 1),       # bf16, k rows of 9 chunks leave the last three CTAs' slices empty
    ("tiny", 40960, 4096, 16),           # fp32, 10240 chunks
])
def test_rows_wider_than_a_cta(cuda_lib, wl_name, dq, dk, n_seg):
    _run(wl_name, 5, dq, dk, n_seg, seed=dq % 97)


def test_partial_stats_cluster_paths(cuda_lib):
    # segment partials (the scalars SwiftQK exchanges) from both cluster routes
    wl = W.QKNORM_WORKLOADS["prefill_gqa"]
    for T, d, n_seg in ((9, 1024, 32), (4, 98304, 8)):
        inp = W.make_qknorm_inputs(wl, seed=d, device="cpu", tokens=T, dq=d, dk=8)
        got = qk.rmsnorm_partial_stats(inp["q"].to(DEV), n_seg)
        torch.cuda.synchronize()
        ref = oracle.segment_partials(inp["q"], n_seg)
        np.testing.assert_allclose(got.cpu().double().numpy(), ref, rtol=1e-5, atol=0)


def test_cluster_path_deterministic_and_in_place(cuda_lib):
    q, k, inp, qo, ko = _run("prefill_gqa", 23, 81920, 1024, 16, seed=3)
    wq, wk = inp["wq"].to(DEV), inp["wk"].to(DEV)
    qo2, ko2 = qk.qknorm_fused(q, k, wq, wk, 1e-6, 16)
    q3, k3 = q.clone(), k.clone()
    qk.qknorm_fused(q3, k3, wq, wk, 1e-6, 16, inplace=True)
    torch.cuda.synchronize()
    for a, b in ((qo, qo2), (ko, ko2), (qo, q3), (ko, k3)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert qk.load_library().qkn_check_device(None) == 0, qk.load_library().qkn_last_error()

"""The CTA-pair projection kernel against the oracle and the single-CTA kernel.

``QKN_GEMM_KERNEL`` selects the kernel that serves flashnorm_proj calls with a
given or separately computed 1/rms (and qkv_norm_proj's unscaled projection):
the default ``pair`` (two CTAs of a cluster per 256 x 256 tile,
tcgen05.mma.cta_group::2) or ``single`` (one CTA per 128 x 256 tile, also the
kernel of the in-kernel statistics form).  Both accumulate every output in
the same k order in fp32 and scale and round it the same way, so their
outputs must agree bit for bit; each is also checked against the fp64 oracle
(relative Frobenius error <= 1e-2 with the original w and W) on shapes with
ragged row and column tiles, including pair tiles whose odd CTA holds no
valid row or no valid W' row.
"""
from __future__ import annotations

import os

import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import PROJ_FROB_TOL, frobenius_rel
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


class kernel:
    """Context manager selecting the projection kernel for the calls inside it."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        self.prev = os.environ.get("QKN_GEMM_KERNEL")
        os.environ["QKN_GEMM_KERNEL"] = self.name

    def __exit__(self, *exc):
        if self.prev is None:
            os.environ.pop("QKN_GEMM_KERNEL", None)
        else:
            os.environ["QKN_GEMM_KERNEL"] = self.prev
        return False


@pytest.mark.parametrize("M,K,N", [
    (256, 64, 256),      # one pair tile
    (300, 520, 776),     # ragged rows and columns: the last pair tile's odd CTA holds 8 valid W' rows
    (129, 512, 264),     # the odd CTA of the only row block holds no valid row
    (1, 8, 8),           # smallest problem
    (1000, 1024, 1032),  # several tiles per pair, ragged everywhere
])
def test_pair_matches_single_and_oracle(cuda_lib, M, K, N):
    inp = W.make_flashnorm_inputs(seed=M + N, M=M, K=K, N=N)
    x = inp["x"].to(DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
    inv = torch.empty(M, dtype=torch.float32, device=DEV)
    with kernel("pair"):
        yp = qk.flashnorm_proj(x, Wf, inp["eps"], inv_rms_out=inv)
        yp_given = qk.flashnorm_proj(x, Wf, inp["eps"], inv_rms=inv)
    with kernel("single"):
        ys = qk.flashnorm_proj(x, Wf, inp["eps"], inv_rms_out=inv)
    torch.cuda.synchronize()
    assert torch.equal(yp.view(torch.int16), ys.view(torch.int16)), "pair and single-CTA outputs differ"
    assert torch.equal(yp.view(torch.int16), yp_given.view(torch.int16))
    ref = oracle.norm_then_project(inp["x"], inp["w"], inp["W"], inp["eps"])
    assert frobenius_rel(yp, ref) <= PROJ_FROB_TOL
    assert qk.load_library().qkn_check_device(None) == 0, qk.load_library().qkn_last_error()


def test_pair_unscaled_projection(cuda_lib):
    # qkv_norm_proj's projection (no row scaling) on the pair kernel
    M, K, nq, nk, nv = 300, 256, 264, 136, 136
    inp = W.make_flashnorm_inputs(seed=31, M=M, K=K, N=nq + nk + nv)
    g = torch.Generator().manual_seed(32)
    wq, wk, wv = ((1 + 0.1 * torch.randn(n, generator=g)).to(torch.bfloat16).to(DEV) for n in (nq, nk, nv))
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
    x = inp["x"].to(DEV)
    with kernel("pair"):
        a = qk.qkv_norm_proj(x, Wf, nq, nk, nv, wq, wk, wv, 1e-6, 1)
    with kernel("single"):
        b = qk.qkv_norm_proj(x, Wf, nq, nk, nv, wq, wk, wv, 1e-6, 1)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_pair_deterministic_and_row_major_weights(cuda_lib):
    M, K, N = 640, 768, 520
    inp = W.make_flashnorm_inputs(seed=33, M=M, K=K, N=N)
    x = inp["x"].to(DEV)
    Wk = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV), k_major=True)
    Wr = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV), k_major=False)
    inv = torch.empty(M, dtype=torch.float32, device=DEV)
    with kernel("pair"):
        a = qk.flashnorm_proj(x, Wk, inp["eps"], inv_rms_out=inv)
        b = qk.flashnorm_proj(x, Wk, inp["eps"], inv_rms_out=inv)
        c = qk.flashnorm_proj(x, Wr, inp["eps"], inv_rms_out=inv, k_major=False)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


@pytest.mark.slow
def test_pair_full_size_matches_single(cuda_lib):
    # the benchmark's workload: every element of the pair kernel's output equals the single-CTA kernel's
    wl = W.FLASHNORM_WORKLOAD
    inp = W.make_flashnorm_inputs(seed=0, device=DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"], inp["W"])
    inv = torch.empty(wl.M, dtype=torch.float32, device=DEV)
    with kernel("pair"):
        yp = qk.flashnorm_proj(inp["x"], Wf, wl.eps, inv_rms_out=inv)
    with kernel("single"):
        ys = qk.flashnorm_proj(inp["x"], Wf, wl.eps, inv_rms_out=inv)
    torch.cuda.synchronize()
    assert torch.equal(yp.view(torch.int16), ys.view(torch.int16))
    assert qk.load_library().qkn_check_device(None) == 0, qk.load_library().qkn_last_error()

"""GPU parity of qkv_proj_qknorm (QKV projection with QK-Norm in the GEMM epilogue).

Bars:
* against the fp64 oracle with the ORIGINAL weights (RMSNorm(x; w_in) W, then
  QK-Norm of the q and k slices): relative Frobenius error <= 1e-2 per section,
  the projection tolerance (W' is rounded to bf16 once, the GEMM accumulates
  in fp32, y is rounded to bf16 once);
* against the oracle fed the bf16 W' the GPU used: <= 4e-3 per section and at
  least 99 % of the elements within 1 bf16 ulp of RNE(oracle) -- only fp32
  accumulation order and the final rounding remain;
* bit-identical between runs, with a given workspace or an internal one, and
  with a given 1/rms vector equal to the statistics pass's.
Shapes span several 128-row and 256-column tiles with ragged tails, q / k / v
sections that end inside a tile, nv = 0 and the GQA split.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import PROJ_FROB_TOL, bf16_bits, bf16_ulp_distance, frobenius_rel
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(M, K, nq, nk, nv, seed, wdt=torch.bfloat16):
    inp = W.make_flashnorm_inputs(seed=seed, M=M, K=K, N=nq + nk + nv)
    g = torch.Generator().manual_seed(seed + 1)
    wq = (1 + 0.1 * torch.randn(nq, generator=g)).to(wdt)
    wk = (1 + 0.1 * torch.randn(nk, generator=g)).to(wdt)
    return inp["x"], inp["w"], inp["W"], wq, wk, inp["eps"]


def _sections(nq, nk, nv):
    out = [("q", 0, nq), ("k", nq, nq + nk)]
    if nv:
        out.append(("v", nq + nk, nq + nk + nv))
    return out


def _check(y, ref, ref_used, nq, nk, nv, what):
    y = y.cpu()
    for name, lo, hi in _sections(nq, nk, nv):
        err = frobenius_rel(y[:, lo:hi], ref[:, lo:hi])
        assert err <= PROJ_FROB_TOL, f"{what} {name}: relative Frobenius error {err:.3e} vs oracle"
        err2 = frobenius_rel(y[:, lo:hi], ref_used[:, lo:hi])
        assert err2 <= 4e-3, f"{what} {name}: {err2:.3e} vs oracle with the GPU's W'"
        ulp = bf16_ulp_distance(bf16_bits(y[:, lo:hi]), oracle.round_bf16_bits(ref_used[:, lo:hi]))
        assert (ulp <= 1).mean() >= 0.99, f"{what} {name}: only {(ulp <= 1).mean():.4f} within 1 ulp"


def _run(M, K, nq, nk, nv, seed=0, wdt=torch.bfloat16, mode="stats"):
    x, w_in, Wm, wq, wk, eps = _inputs(M, K, nq, nk, nv, seed, wdt)
    xd = x.to(DEV)
    Wf = qk.flashnorm_fold_weights(w_in.to(DEV), Wm.to(DEV), k_major=True)
    kw = {}
    if mode == "unit":
        kw["input_norm"] = False
    y = qk.qkv_proj_qknorm(xd, Wf, nq, nk, nv, wq.to(DEV), wk.to(DEV), eps, **kw)
    torch.cuda.synchronize()
    Wf_used = Wf.float().cpu().T.contiguous()  # [K, N], the bf16 folded weights as fp32
    if mode == "unit":
        ref = oracle.qkv_proj_qknorm(x, None, oracle.fold_weights(w_in, Wm), wq, wk, nq, nk, eps, eps,
                                     input_norm=False)
        ref_used = oracle.qkv_proj_qknorm(x, None, Wf_used, wq, wk, nq, nk, eps, eps, input_norm=False)
    else:
        ref = oracle.qkv_proj_qknorm(x, w_in, Wm, wq, wk, nq, nk, eps, eps)
        ref_used = oracle.qkv_proj_qknorm(x, torch.ones(K), Wf_used, wq, wk, nq, nk, eps, eps)
    _check(y, ref, ref_used, nq, nk, nv, f"M={M} K={K} nq={nq} nk={nk} nv={nv} {mode}")
    return y


@pytest.mark.parametrize("M,K,nq,nk,nv", [
    (128, 64, 256, 256, 256),       # one tile per section
    (300, 200, 520, 264, 136),      # ragged rows, sections ending inside tiles
    (129, 512, 1024, 512, 0),       # no v section, one row in the last row block
    (512, 1024, 5120, 1024, 1024),  # the GQA split: 20 q tiles, 4 k tiles per row block
    (1, 8, 8, 8, 8),                # smallest problem
])
def test_parity_vs_oracle(cuda_lib, M, K, nq, nk, nv):
    _run(M, K, nq, nk, nv, seed=M + nq)


def test_fp32_weights_and_no_input_norm(cuda_lib):
    _run(200, 256, 512, 256, 256, seed=3, wdt=torch.float32)
    _run(200, 256, 512, 256, 256, seed=4, mode="unit")


def test_given_inv_rms_workspace_and_determinism(cuda_lib):
    M, K, nq, nk, nv = 640, 512, 1024, 1024, 512
    x, w_in, Wm, wq, wk, eps = _inputs(M, K, nq, nk, nv, seed=7)
    xd, wq, wk = x.to(DEV), wq.to(DEV), wk.to(DEV)
    Wf = qk.flashnorm_fold_weights(w_in.to(DEV), Wm.to(DEV))
    inv = torch.empty(M, dtype=torch.float32, device=DEV)
    a = qk.qkv_proj_qknorm(xd, Wf, nq, nk, nv, wq, wk, eps, inv_rms_out=inv)
    b = qk.qkv_proj_qknorm(xd, Wf, nq, nk, nv, wq, wk, eps, inv_rms=inv)
    ws = torch.empty(qk.qkv_proj_qknorm_workspace_bytes(M, nq, nk, nv), dtype=torch.uint8, device=DEV)
    c = qk.qkv_proj_qknorm(xd, Wf, nq, nk, nv, wq, wk, eps, inv_rms=inv, workspace=ws)
    d = qk.qkv_proj_qknorm(xd, Wf, nq, nk, nv, wq, wk, eps, inv_rms=inv, workspace=ws)
    torch.cuda.synchronize()
    for t in (b, c, d):
        assert torch.equal(a.view(torch.int16), t.view(torch.int16))
    np.testing.assert_allclose(inv.cpu().double().numpy(), oracle.inv_rms(x, eps), rtol=1e-5)
    assert qk.load_library().qkn_check_device(None) == 0, qk.load_library().qkn_last_error()


def test_matches_two_step_device_path(cuda_lib):
    # projection with the 1/rms epilogue, then qknorm_fused on the q and k column blocks:
    # the same function with one extra bf16 rounding of u in between
    M, K, nq, nk, nv = 384, 768, 1024, 512, 512
    x, w_in, Wm, wq, wk, eps = _inputs(M, K, nq, nk, nv, seed=11)
    xd, wq, wk = x.to(DEV), wq.to(DEV), wk.to(DEV)
    Wf = qk.flashnorm_fold_weights(w_in.to(DEV), Wm.to(DEV))
    inv = torch.empty(M, dtype=torch.float32, device=DEV)
    y = qk.qkv_proj_qknorm(xd, Wf, nq, nk, nv, wq, wk, eps, inv_rms_out=inv)
    u = qk.flashnorm_proj(xd, Wf, eps, inv_rms=inv)
    qk.qknorm_fused(u[:, :nq], u[:, nq:nq + nk], wq, wk, eps, 1, inplace=True)
    torch.cuda.synchronize()
    assert frobenius_rel(y.cpu(), u.cpu().double().numpy()) <= 8e-3
    assert torch.equal(y[:, nq + nk:].view(torch.int16), u[:, nq + nk:].view(torch.int16))  # v: same epilogue


@pytest.mark.slow
def test_full_size_every_row_block(cuda_lib):
    # x [8192, 4096] with W [4096, 12288] split q | k | v = 4096 each: one row of every
    # 128-row tile block (and the last row), all N columns, against the oracle
    from test_flashnorm_gpu import block_rows
    wl = W.FLASHNORM_WORKLOAD
    nq = nk = nv = wl.N // 3
    inp = W.make_flashnorm_inputs(seed=0, device=DEV)
    g = torch.Generator().manual_seed(1)
    wq = (1 + 0.1 * torch.randn(nq, generator=g)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(nk, generator=g)).to(torch.bfloat16)
    Wf = qk.flashnorm_fold_weights(inp["w"], inp["W"])
    y = qk.qkv_proj_qknorm(inp["x"], Wf, nq, nk, nv, wq.to(DEV), wk.to(DEV), wl.eps)
    torch.cuda.synchronize()
    rows = block_rows(wl.M, seed=4)
    rd = rows.to(DEV)
    xs = inp["x"][rd].cpu()
    ref = oracle.qkv_proj_qknorm(xs, inp["w"].cpu(), inp["W"].cpu(), wq, wk, nq, nk, wl.eps, wl.eps)
    ref_used = oracle.qkv_proj_qknorm(xs, torch.ones(wl.K), Wf.float().cpu().T.contiguous(), wq, wk, nq, nk,
                                      wl.eps, wl.eps)
    _check(y[rd], ref, ref_used, nq, nk, nv, "full size, one row per 128-row block")
    assert torch.isfinite(y.float()).all()
    assert qk.load_library().qkn_check_device(None) == 0, qk.load_library().qkn_last_error()

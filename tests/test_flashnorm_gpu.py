"""GPU parity of flashnorm_fold_weights and flashnorm_proj against the fp64 oracle.

* fold: bf16 w times bf16 W is exact in fp32, so W' must equal the oracle's
  product rounded once to bf16 bit for bit; with fp32 w it may differ by one
  bf16 ulp (the fp32 product is itself rounded).
* projection: relative Frobenius error <= 1e-2 against RMSNorm(x) W computed
  in fp64 with the ORIGINAL w and W (FlashNorm's claim is exact equality, so
  the only differences are bf16 rounding of W', of y, and fp32 accumulation);
  the 1/rms vector it used is checked to 1e-5 relative.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import (PROJ_FROB_TOL, assert_bf16_close, assert_f32_close, bf16_bits, bf16_ulp_distance,
                    frobenius_rel)
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(M, K, N, seed=0):
    inp = W.make_flashnorm_inputs(seed=seed, M=M, K=K, N=N)
    return inp["x"], inp["w"], inp["W"], inp["eps"]


@pytest.mark.parametrize("k_major", [True, False])
@pytest.mark.parametrize("K,N", [(64, 64), (200, 136), (4096, 264), (13, 17), (64, 100), (20, 24)])
def test_fold_bit_exact_bf16_weights(cuda_lib, k_major, K, N):
    # multiples of 8 take the 16-byte tile kernels; 13 x 17, 64 x 100 (N) and
    # 20 x 24 (K, for the K-major output) the element-wise ones
    _, w, Wm, _ = _inputs(8, K, N, seed=K + N)
    out = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV), k_major=k_major)
    torch.cuda.synchronize()
    ref = oracle.round_bf16_bits(oracle.fold_weights(w, Wm))
    got = bf16_bits(out)
    if k_major:
        got = got.T
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("k_major", [True, False])
def test_fold_fp32_weights_within_one_ulp(cuda_lib, k_major):
    _, w, Wm, _ = _inputs(8, 256, 512, seed=1)
    w32 = (1 + 0.1 * torch.randn(256, generator=torch.Generator().manual_seed(2)))
    out = qk.flashnorm_fold_weights(w32.to(DEV), Wm.to(DEV), k_major=k_major)
    torch.cuda.synchronize()
    ref = oracle.round_bf16_bits(oracle.fold_weights(w32, Wm))
    got = bf16_bits(out)
    assert bf16_ulp_distance(got.T if k_major else got, ref).max() <= 1


def _proj_check(M, K, N, seed=0, in_kernel_stats=False):
    x, w, Wm, eps = _inputs(M, K, N, seed=seed)
    xd = x.to(DEV)
    Wf = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV), k_major=True)
    if in_kernel_stats:
        y = qk.flashnorm_proj(xd, Wf, eps, in_kernel_stats=True)  # 1/rms computed inside the projection kernel
    else:
        inv_out = torch.empty(M, dtype=torch.float32, device=DEV)
        y = qk.flashnorm_proj(xd, Wf, eps, inv_rms_out=inv_out)  # separate statistics pass
    torch.cuda.synchronize()
    ref = oracle.norm_then_project(x, w, Wm, eps)
    err = frobenius_rel(y, ref)
    assert err <= PROJ_FROB_TOL, f"M={M} K={K} N={N}: relative Frobenius error {err:.3e}"
    if not in_kernel_stats:
        assert_f32_close(inv_out, oracle.inv_rms(x, eps), what="inv_rms")
    # tighter: against the oracle's deferred form with the bf16-rounded W' the GPU used,
    # only fp32 accumulation and the final bf16 rounding remain
    Wf_used = Wf.float().cpu().T.contiguous()
    ref2 = oracle.flashnorm_deferred(x, Wf_used, eps)
    err2 = frobenius_rel(y, ref2)
    assert err2 <= 4e-3, f"vs deferred form with the GPU's W': {err2:.3e}"
    return y, ref, err


@pytest.mark.parametrize("in_kernel_stats", [False, True])
@pytest.mark.parametrize("M,K,N", [(128, 64, 256), (300, 200, 520), (129, 4096, 264), (1, 8, 8),
                                   (640, 512, 1024)])
def test_proj_parity_ragged(cuda_lib, M, K, N, in_kernel_stats):
    _proj_check(M, K, N, seed=M, in_kernel_stats=in_kernel_stats)


def test_proj_statistics_paths_agree(cuda_lib):
    # in-kernel 1/rms vs the separate statistics pass: same math, different summation
    # order, so y agrees to one bf16 ulp; a given 1/rms reproduces y bit for bit
    x, w, Wm, eps = _inputs(256, 1024, 512, seed=9)
    xd = x.to(DEV)
    Wf = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV))
    y1 = qk.flashnorm_proj(xd, Wf, eps, in_kernel_stats=True)
    inv = torch.empty(256, dtype=torch.float32, device=DEV)
    y2 = qk.flashnorm_proj(xd, Wf, eps, inv_rms_out=inv)
    y3 = qk.flashnorm_proj(xd, Wf, eps, inv_rms=inv)
    torch.cuda.synchronize()
    assert bf16_ulp_distance(bf16_bits(y1), bf16_bits(y2)).max() <= 1
    assert torch.equal(y2.view(torch.int16), y3.view(torch.int16))


def test_proj_default_is_the_separate_pass(cuda_lib):
    # without inv_rms / inv_rms_out the binding supplies the workspace itself, so the
    # default call is the separate statistics pass, bit for bit
    x, w, Wm, eps = _inputs(300, 512, 264, seed=12)
    xd = x.to(DEV)
    Wf = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV))
    inv = torch.empty(300, dtype=torch.float32, device=DEV)
    a = qk.flashnorm_proj(xd, Wf, eps)
    b = qk.flashnorm_proj(xd, Wf, eps, inv_rms_out=inv)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("M,K", [(1, 8), (300, 4096), (1029, 1000)])
def test_inv_rms_alone(cuda_lib, M, K):
    # FlashNorm's row statistic on its own: within 1e-5 of the oracle, and bit for
    # bit the values the projection writes to inv_rms_out
    x, w, Wm, eps = _inputs(M, K, 64, seed=M + K)
    xd = x.to(DEV)
    inv = qk.flashnorm_inv_rms(xd, eps)
    Wf = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV))
    inv_out = torch.empty(M, dtype=torch.float32, device=DEV)
    qk.flashnorm_proj(xd, Wf, eps, inv_rms_out=inv_out)
    torch.cuda.synchronize()
    assert_f32_close(inv, oracle.inv_rms(x, eps), what="inv_rms")
    assert torch.equal(inv, inv_out)


def test_proj_with_unit_scale_is_plain_gemm(cuda_lib):
    # a given 1/rms of 1 turns the kernel into y = x W'^T (W' = W^T for w = 1): the GEMM alone
    M, K, N = 256, 512, 768
    x, w, Wm, _ = _inputs(M, K, N, seed=4)
    Wf = qk.flashnorm_fold_weights(torch.ones(K, dtype=torch.bfloat16, device=DEV), Wm.to(DEV))
    ones = torch.ones(M, dtype=torch.float32, device=DEV)
    y = qk.flashnorm_proj(x.to(DEV), Wf, inv_rms=ones)
    torch.cuda.synchronize()
    ref = oracle.as_f64(x) @ oracle.as_f64(Wm)  # library matmul: a textbook GEMM reference
    assert frobenius_rel(y, ref) <= 4e-3


def test_proj_deterministic(cuda_lib):
    x, w, Wm, eps = _inputs(512, 1024, 1024, seed=5)
    xd = x.to(DEV)
    Wf = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV))
    inv = torch.empty(512, dtype=torch.float32, device=DEV)
    for kw in ({"in_kernel_stats": True}, {"inv_rms_out": inv}, {}):
        a = qk.flashnorm_proj(xd, Wf, eps, **kw)
        b = qk.flashnorm_proj(xd, Wf, eps, **kw)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def block_rows(M, bm=128, seed=3):
    """One row at a seeded offset inside every bm-row block, plus the first and last rows."""
    g = torch.Generator().manual_seed(seed)
    nblk = (M + bm - 1) // bm
    rows = [b * bm + int(torch.randint(0, min(bm, M - b * bm), (1,), generator=g)) for b in range(nblk)]
    return torch.tensor(sorted(set(rows) | {0, M - 1}))


@pytest.mark.slow
def test_proj_full_size_every_row_block(cuda_lib):
    # the benchmark's workload x[8192,4096] W[4096,12288]: one row of every 128-row
    # tile block (and the last row) across all N columns against the oracle
    wl = W.FLASHNORM_WORKLOAD
    inp = W.make_flashnorm_inputs(seed=0, device=DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"], inp["W"])
    inv = torch.empty(wl.M, dtype=torch.float32, device=DEV)
    y = qk.flashnorm_proj(inp["x"], Wf, wl.eps, inv_rms_out=inv)  # the benchmark's form
    y_in = qk.flashnorm_proj(inp["x"], Wf, wl.eps, in_kernel_stats=True)  # 1/rms inside the kernel
    torch.cuda.synchronize()
    assert bf16_ulp_distance(bf16_bits(y_in), bf16_bits(y)).max() <= 1
    rows = block_rows(wl.M)
    rd = rows.to(DEV)
    xs = inp["x"][rd].cpu()
    ys = y[rd].cpu()
    # with the original w and W: the projection tolerance
    ref = oracle.norm_then_project(xs, inp["w"].cpu(), inp["W"].cpu(), wl.eps)
    err = frobenius_rel(ys, ref)
    assert err <= PROJ_FROB_TOL, f"full-size relative Frobenius error {err:.3e}"
    # with the bf16 W' the GPU used: only accumulation order and the output rounding remain
    ref_used = oracle.flashnorm_deferred(xs, Wf.float().cpu().T.contiguous(), wl.eps)
    ulp = bf16_ulp_distance(bf16_bits(ys), oracle.round_bf16_bits(ref_used))
    frac = float((ulp <= 1).mean())
    assert frac >= 0.99, f"only {frac:.4f} of the sampled elements within 1 bf16 ulp of RNE(oracle with W')"
    assert frobenius_rel(ys, ref_used) <= 4e-3
    np.testing.assert_allclose(inv[rd].cpu().double().numpy(), oracle.inv_rms(xs, wl.eps), rtol=1e-5)
    assert torch.isfinite(y.float()).all()


def test_device_error_word_clear(cuda_lib):
    # the projection kernel's bounded waits never gave up in this process
    lib = qk.load_library()
    assert lib.qkn_check_device(None) == 0, lib.qkn_last_error()


@pytest.mark.parametrize("in_kernel_stats", [False, True])
def test_row_major_folded_weights(cuda_lib, in_kernel_stats):
    # W' handed over row-major ([K, N]) is copied K-major inside the call: the result is the
    # K-major call's, bit for bit
    M, K, N = 300, 520, 776
    x, w, Wm, eps = _inputs(M, K, N, seed=21)
    xd = x.to(DEV)
    Wk = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV), k_major=True)
    Wr = qk.flashnorm_fold_weights(w.to(DEV), Wm.to(DEV), k_major=False)
    kw = {"in_kernel_stats": True} if in_kernel_stats else {"inv_rms_out": torch.empty(M, dtype=torch.float32, device=DEV)}
    a = qk.flashnorm_proj(xd, Wk, eps, **kw)
    b = qk.flashnorm_proj(xd, Wr, eps, k_major=False, **kw)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert frobenius_rel(b, oracle.norm_then_project(x, w, Wm, eps)) <= PROJ_FROB_TOL

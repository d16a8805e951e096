"""Guard-region checks: no kernel writes outside the output it was given.

Every output here lives inside a larger buffer pre-filled with a sentinel
byte: 4 KiB of guard before it, 4 KiB after it, and -- where the entry point
takes a row pitch -- padding columns between the end of each row and the next
row (ld_out > d).  After the call, every sentinel byte must be intact.  This
covers writes past a row's end, into the pitch padding, past the last row, in
a ragged tail, in the last partial 128 x 256 GEMM tile, and before the first
element.  Each case also checks the values it wrote against the oracle, so a
kernel that wrote nothing cannot pass.

One case per kernel family: the staged kernel (generic, narrow and
many-segment flavours), the register kernel (streaming and one-shot), the
cluster kernel, the element-wise kernel, the partial statistics, the apply
step of tensor-parallel QK-Norm, the fold (both layouts), the row statistic,
the projection GEMMs (CTA pair and single CTA; given, separate and
in-kernel 1/rms; K-major and row-major W'), the fused QKV + QK-Norm GEMM, the RMSNorm-elimination form,
the no-allocation projection, and the host-buffer pipeline.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import (PARTIAL_REL_TOL, PROJ_FROB_TOL, assert_bf16_close, assert_f32_close, frobenius_rel)
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096   # bytes of sentinel before and after every output
SENT = 0xA5    # sentinel byte (bf16 0xA5A5 / fp32 0xA5A5A5A5: small negative numbers no kernel here produces)


class Guarded:
    """A [rows, cols] output view with row pitch ld inside a sentinel-filled buffer."""

    def __init__(self, rows: int, cols: int, dtype: torch.dtype, ld: int | None = None, device=DEV,
                 pin: bool = False):
        self.rows, self.cols, self.dtype = rows, cols, dtype
        self.ld = cols if ld is None else ld
        self.esz = torch.empty(0, dtype=dtype).element_size()
        body = rows * self.ld * self.esz
        if device == "cpu":
            self.raw = torch.full((GUARD + body + GUARD,), SENT, dtype=torch.uint8, pin_memory=pin)
        else:
            self.raw = torch.full((GUARD + body + GUARD,), SENT, dtype=torch.uint8, device=device)
        full = self.raw[GUARD:GUARD + body].view(dtype).view(rows, self.ld)
        self.view = full if self.ld == cols else full[:, :cols]

    def check(self, what: str) -> None:
        raw = self.raw.cpu().numpy()
        before, after = raw[:GUARD], raw[len(raw) - GUARD:]
        assert (before == SENT).all(), f"{what}: {int((before != SENT).sum())} guard bytes before the output written"
        assert (after == SENT).all(), f"{what}: {int((after != SENT).sum())} guard bytes after the output written"
        if self.ld > self.cols and self.rows > 0:
            body = raw[GUARD:len(raw) - GUARD].reshape(self.rows, self.ld * self.esz)
            pad = body[:, self.cols * self.esz:]
            bad = np.argwhere(pad != SENT)
            assert bad.size == 0, (f"{what}: {len(bad)} pitch-padding bytes written, first at row {bad[0][0]} "
                                   f"byte {bad[0][1]} past the row end")


def _qk_case(T, dq, dk, n_seg, dtype, pad, seed):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(T, dq, generator=g) * 2).to(dtype).to(DEV)
    k = (torch.randn(T, dk, generator=g) * 2).to(dtype).to(DEV) if dk else None
    wq = (1 + 0.1 * torch.randn(dq, generator=g)).to(dtype).to(DEV)
    wk = (1 + 0.1 * torch.randn(dk, generator=g)).to(dtype).to(DEV) if dk else None
    gq = Guarded(T, dq, dtype, dq + pad)
    gk = Guarded(T, dk, dtype, dk + pad) if dk else None
    qk.qknorm_fused(q, k, wq, wk, 1e-6, n_seg, q_out=gq.view, k_out=gk.view if gk else None)
    torch.cuda.synchronize()
    return q, k, wq, wk, gq, gk


def _check_norm(out, x, w, what):
    ref = oracle.rmsnorm(x.cpu(), w.cpu(), 1e-6)
    if out.dtype == torch.bfloat16:
        assert_bf16_close(out.contiguous(), ref, what)
    else:
        assert_f32_close(out.contiguous(), ref, what=what)


@pytest.mark.parametrize("family,T,dq,dk,n_seg,dtype", [
    ("staged generic", 37, 4096, 4096, 8, torch.bfloat16),
    ("staged narrow (wide q beside narrow k)", 41, 5120, 1024, 8, torch.bfloat16),
    ("staged many segments", 29, 2048, 2048, 16, torch.bfloat16),
    ("staged many segments fp32", 23, 2560, 1280, 64, torch.float32),
    ("register streaming", 3001, 1024, 1024, 4, torch.bfloat16),
    ("register streaming 128-wide", 1003, 128, 128, 1, torch.bfloat16),
    ("register one-shot (rows past the staging ring)", 5, 32768, 0, 8, torch.bfloat16),
    ("cluster (rows spanning CTAs)", 3, 131072, 0, 4, torch.bfloat16),
    ("element-wise (width not a multiple of 8)", 19, 1000, 100, 4, torch.bfloat16),
])
def test_norm_kernels_stay_inside_outputs(cuda_lib, family, T, dq, dk, n_seg, dtype):
    pad = 24 if dtype == torch.bfloat16 else 12  # 48 bytes of pitch padding per row
    q, k, wq, wk, gq, gk = _qk_case(T, dq, dk, n_seg, dtype, pad, seed=T + dq)
    gq.check(f"{family} q")
    _check_norm(gq.view, q, wq, f"{family} q")
    if gk is not None:
        gk.check(f"{family} k")
        _check_norm(gk.view, k, wk, f"{family} k")


@pytest.mark.parametrize("rows,d,n_seg", [(37, 4096, 8), (301, 1024, 4), (29, 2048, 16), (7, 5120, 64),
                                          (3, 131072, 4), (19, 1000, 4)])
def test_partial_stats_stay_inside_output(cuda_lib, rows, d, n_seg):
    g = torch.Generator().manual_seed(d + n_seg)
    x = torch.randn(rows, d, generator=g).to(torch.bfloat16).to(DEV)
    out = Guarded(rows, n_seg, torch.float32)
    qk.rmsnorm_partial_stats(x, n_seg, out=out.view)
    torch.cuda.synchronize()
    out.check(f"partials rows={rows} d={d} n_seg={n_seg}")
    assert_f32_close(out.view, oracle.segment_partials(x.cpu(), n_seg), tol=PARTIAL_REL_TOL, what="partials")


def test_apply_partials_stays_inside_output(cuda_lib):
    rows, d, shards = 301, 640, 4
    g = torch.Generator().manual_seed(11)
    x_full = torch.randn(rows, d * shards, generator=g).to(torch.bfloat16).to(DEV)
    w_full = (1 + 0.1 * torch.randn(d * shards, generator=g)).to(torch.bfloat16).to(DEV)
    partial = qk.rmsnorm_partial_stats(x_full, shards)
    for s in range(shards):
        xs = x_full[:, s * d:(s + 1) * d]
        out = Guarded(rows, d, torch.bfloat16, d + 40)
        qk.rmsnorm_apply_partials(xs, w_full[s * d:(s + 1) * d], partial, d * shards, 1e-6, out=out.view)
        torch.cuda.synchronize()
        out.check(f"apply shard {s}")
        ref = oracle.rmsnorm(x_full.cpu(), w_full.cpu(), 1e-6)[:, s * d:(s + 1) * d]
        assert_bf16_close(out.view.contiguous(), ref, f"apply shard {s}")


@pytest.mark.parametrize("k_major", [True, False])
@pytest.mark.parametrize("K,N", [(200, 136), (4096, 264), (13, 17)])
def test_fold_stays_inside_output(cuda_lib, k_major, K, N):
    inp = W.make_flashnorm_inputs(seed=K, M=8, K=K, N=N)
    rows, cols = (N, K) if k_major else (K, N)
    out = Guarded(rows, cols, torch.bfloat16)
    qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV), k_major=k_major, out=out.view)
    torch.cuda.synchronize()
    out.check(f"fold K={K} N={N} k_major={k_major}")
    got = out.view.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.round_bf16_bits(oracle.fold_weights(inp["w"], inp["W"]))
    np.testing.assert_array_equal(got.T if k_major else got, ref)


def test_inv_rms_stays_inside_output(cuda_lib):
    inp = W.make_flashnorm_inputs(seed=2, M=1001, K=520, N=8)
    out = Guarded(1, 1001, torch.float32)
    qk.flashnorm_inv_rms(inp["x"].to(DEV), inp["eps"], out=out.view[0])
    torch.cuda.synchronize()
    out.check("flashnorm_inv_rms")
    assert_f32_close(out.view[0], oracle.inv_rms(inp["x"], inp["eps"]), what="inv_rms")


# M, K, N: ragged last row block (M % 128) and last column tile (N % 256, N % 32 = 8)
PROJ_SHAPE = (300, 520, 776)


@pytest.mark.parametrize("gemm_kernel", ["pair", "single"])
@pytest.mark.parametrize("mode", ["separate stats", "in-kernel stats", "given inv_rms", "row-major W'"])
def test_projection_stays_inside_output(cuda_lib, mode, gemm_kernel, monkeypatch):
    # the CTA-pair kernel (default) and the single-CTA kernel; the in-kernel
    # statistics form always runs on the single-CTA kernel
    monkeypatch.setenv("QKN_GEMM_KERNEL", gemm_kernel)
    M, K, N = PROJ_SHAPE
    inp = W.make_flashnorm_inputs(seed=5, M=M, K=K, N=N)
    x = inp["x"].to(DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV), k_major=(mode != "row-major W'"))
    y = Guarded(M, N, torch.bfloat16)
    inv = Guarded(1, M, torch.float32)
    kw = {"out": y.view}
    if mode == "in-kernel stats":
        kw["in_kernel_stats"] = True
    elif mode == "given inv_rms":
        qk.flashnorm_inv_rms(x, inp["eps"], out=inv.view[0])
        kw["inv_rms"] = inv.view[0]
    else:
        kw["inv_rms_out"] = inv.view[0]
        if mode == "row-major W'":
            kw["k_major"] = False
    qk.flashnorm_proj(x, Wf, inp["eps"], **kw)
    torch.cuda.synchronize()
    y.check(f"flashnorm_proj y ({mode})")
    inv.check(f"flashnorm_proj inv_rms ({mode})")
    ref = oracle.norm_then_project(inp["x"], inp["w"], inp["W"], inp["eps"])
    assert frobenius_rel(y.view, ref) <= PROJ_FROB_TOL


def test_noalloc_projection_stays_inside_output(cuda_lib):
    M, K, N = PROJ_SHAPE
    lib = qk.load_library()
    f = lib.flashnorm_proj_noalloc
    p, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [p, p, p, i64, i64, i64, ctypes.c_int, ctypes.c_float, p]
    f.restype = ctypes.c_int
    inp = W.make_flashnorm_inputs(seed=6, M=M, K=K, N=N)
    x = inp["x"].to(DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
    y = Guarded(M, N, torch.bfloat16)
    st = f(x.data_ptr(), Wf.data_ptr(), y.view.data_ptr(), M, N, K, 1, inp["eps"],
           torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.qkn_last_error().decode()
    torch.cuda.synchronize()
    y.check("flashnorm_proj_noalloc y")
    assert frobenius_rel(y.view, oracle.norm_then_project(inp["x"], inp["w"], inp["W"], inp["eps"])) <= PROJ_FROB_TOL


def test_fused_qkv_stays_inside_outputs(cuda_lib):
    M, K, nq, nk, nv = 300, 200, 520, 264, 136  # ragged rows, sections ending inside tiles
    inp = W.make_flashnorm_inputs(seed=9, M=M, K=K, N=nq + nk + nv)
    g = torch.Generator().manual_seed(10)
    wq = (1 + 0.1 * torch.randn(nq, generator=g)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(nk, generator=g)).to(torch.bfloat16)
    x = inp["x"].to(DEV)
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
    y = Guarded(M, nq + nk + nv, torch.bfloat16)
    inv = Guarded(1, M, torch.float32)
    nws = qk.qkv_proj_qknorm_workspace_bytes(M, nq, nk, nv)
    ws = Guarded(1, nws, torch.uint8)
    qk.qkv_proj_qknorm(x, Wf, nq, nk, nv, wq.to(DEV), wk.to(DEV), inp["eps"], inv_rms_out=inv.view[0],
                       workspace=ws.view[0], out=y.view)
    torch.cuda.synchronize()
    y.check("qkv_proj_qknorm y")
    inv.check("qkv_proj_qknorm inv_rms")
    ws.check("qkv_proj_qknorm workspace")
    ref = oracle.qkv_proj_qknorm(inp["x"], inp["w"], inp["W"], wq, wk, nq, nk, inp["eps"], inp["eps"])
    assert frobenius_rel(y.view, ref) <= PROJ_FROB_TOL


def test_rmsnorm_elimination_stays_inside_output(cuda_lib):
    M, K, nq, nk, nv = 200, 256, 264, 136, 136
    inp = W.make_flashnorm_inputs(seed=12, M=M, K=K, N=nq + nk + nv)
    g = torch.Generator().manual_seed(13)
    wq, wk, wv = ((1 + 0.1 * torch.randn(n, generator=g)).to(torch.bfloat16).to(DEV) for n in (nq, nk, nv))
    Wf = qk.flashnorm_fold_weights(inp["w"].to(DEV), inp["W"].to(DEV))
    y = Guarded(M, nq + nk + nv, torch.bfloat16)
    qk.qkv_norm_proj(inp["x"].to(DEV), Wf, nq, nk, nv, wq, wk, wv, 1e-6, 1, out=y.view)
    torch.cuda.synchronize()
    y.check("qkv_norm_proj y")
    assert torch.isfinite(y.view.float()).all()


def test_host_pipeline_stays_inside_host_outputs(cuda_lib):
    inp = W.make_qknorm_inputs("prefill_gqa", seed=3, tokens=2049)
    T, dq, dk = inp["q"].shape[0], inp["q"].shape[1], inp["k"].shape[1]
    hq, hk = inp["q"].pin_memory(), inp["k"].pin_memory()
    oq = Guarded(T, dq, torch.bfloat16, device="cpu", pin=True)
    ok = Guarded(T, dk, torch.bfloat16, device="cpu", pin=True)
    qk.qknorm_fused_host(hq, hk, inp["wq"].to(DEV), inp["wk"].to(DEV), inp["eps"], inp["n_seg"],
                         q_out=oq.view, k_out=ok.view)
    torch.cuda.synchronize()
    oq.check("qknorm_fused_host q_out")
    ok.check("qknorm_fused_host k_out")
    _check_norm(oq.view, inp["q"], inp["wq"], "host pipeline q")
    _check_norm(ok.view, inp["k"], inp["wk"], "host pipeline k")

"""GPU parity of qknorm_fused and rmsnorm_partial_stats against the fp64 oracle.

Every case calls the CUDA library through its C ABI (via the thin binding) and
compares element by element with the oracle on the same inputs, copied back
to the host exactly:

* fp32 outputs: relative error <= 1e-5; bf16 outputs: within 1 bf16 ulp of the
  oracle rounded once (round-to-nearest-even); partial sums: relative 1e-5.

Sizes: every workload at oracle-friendly sizes that span several blocks with a
ragged tail, the two small workloads at full size, and the two large ones at
full size in the exact launch configuration the benchmark times, every row
checked against the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import assert_bf16_close, assert_f32_close, PARTIAL_REL_TOL
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check(out: torch.Tensor, x: torch.Tensor, w: torch.Tensor, eps: float, what: str):
    ref = oracle.rmsnorm(x.cpu(), w.cpu(), eps)
    if out.dtype == torch.bfloat16:
        return assert_bf16_close(out, ref, what)
    return assert_f32_close(out, ref, what=what)


def run_pair(inp, **kw):
    return qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], inp["n_seg"], **kw)


def to_dev(inp):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


# ------------------------------------------------------------- the four workloads


@pytest.mark.parametrize("name,tokens", [("tiny", None), ("decode", None), ("prefill_gqa", 203),
                                         ("long_context", 301), ("narrow_rows", 3001)])
def test_workload_parity_oracle_sized(cuda_lib, name, tokens):
    inp = to_dev(W.make_qknorm_inputs(name, seed=0, tokens=tokens))
    qo, ko = run_pair(inp)
    torch.cuda.synchronize()
    check(qo, inp["q"], inp["wq"], inp["eps"], f"{name} q")
    check(ko, inp["k"], inp["wk"], inp["eps"], f"{name} k")


def _full_size_all_rows(name, chunk=8192, parts=5):
    """The workload at full size in the benchmark's launch configuration: every
    row of q and k against the oracle (in chunks of rows, so the fp64 copies
    stay small), determinism, and the same rows normalised by several shorter
    launches giving the same bits as the one long launch."""
    wl = W.QKNORM_WORKLOADS[name]
    T = wl.tokens
    inp = W.make_qknorm_inputs(name, seed=0, device=DEV)
    qo, ko = run_pair(inp)
    qo2, ko2 = run_pair(inp)
    torch.cuda.synchronize()
    # determinism: bitwise-equal outputs on a second call
    assert torch.equal(qo.view(torch.int16), qo2.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), ko2.view(torch.int16))
    del qo2, ko2
    # the same rows in `parts` shorter launches of unequal length (ragged ends)
    cuts = sorted({0, T} | {int(T * f) + 1 for f in (0.13, 0.4, 0.41, 0.77)[:parts - 1]})
    for a, b in zip(cuts[:-1], cuts[1:]):
        qs, ks = qk.qknorm_fused(inp["q"][a:b], inp["k"][a:b], inp["wq"], inp["wk"], wl.eps, wl.n_seg)
        torch.cuda.synchronize()
        assert torch.equal(qs.view(torch.int16), qo[a:b].view(torch.int16)), f"{name} q rows {a}:{b}"
        assert torch.equal(ks.view(torch.int16), ko[a:b].view(torch.int16)), f"{name} k rows {a}:{b}"
    # every row against the oracle
    wq, wk = inp["wq"].cpu(), inp["wk"].cpu()
    for r0 in range(0, T, chunk):
        r1 = min(T, r0 + chunk)
        check(qo[r0:r1], inp["q"][r0:r1], wq, wl.eps, f"{name} q rows {r0}:{r1}")
        check(ko[r0:r1], inp["k"][r0:r1], wk, wl.eps, f"{name} k rows {r0}:{r1}")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill_gqa", "long_context", "narrow_rows"])
def test_workload_parity_full_size(cuda_lib, name):
    _full_size_all_rows(name)


# ------------------------------------------------------------------ n_seg coverage


@pytest.mark.parametrize("n_seg", [1, 2, 4, 5, 8, 16, 64])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_n_seg(cuda_lib, n_seg, dtype):
    T, d = 37, 1280  # 1280 = 2^8 * 5: every n_seg above divides it
    g = torch.Generator().manual_seed(n_seg)
    x = (torch.randn(T, d, generator=g) * 3).to(dtype).to(DEV)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(dtype).to(DEV)
    y, _ = qk.qknorm_fused(x, None, w, None, 1e-6, n_seg)
    torch.cuda.synchronize()
    check(y, x, w, 1e-6, f"n_seg={n_seg}")
    p = qk.rmsnorm_partial_stats(x, n_seg)
    torch.cuda.synchronize()
    ref = oracle.segment_partials(x.cpu(), n_seg)
    assert_f32_close(p, ref, tol=PARTIAL_REL_TOL, what=f"partials n_seg={n_seg}")


# ------------------------------------------------------------- shapes and layouts


@pytest.mark.parametrize("d", [1, 3, 8, 24, 100, 520, 1000, 4104, 65536, 65544, 131072, 131080])
def test_widths(cuda_lib, d):
    # odd widths and widths not a multiple of 8 take the element-wise kernel;
    # 65536 bf16 is the widest row one CTA holds, 65544 .. 131072 spread over a
    # cluster of CTAs, and 131080 is past the cluster path (element-wise again)
    T = 3 if d >= 65536 else 19
    g = torch.Generator().manual_seed(d)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16).to(DEV)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16).to(DEV)
    y, _ = qk.qknorm_fused(x, None, w, None, 1e-6, 1)
    torch.cuda.synchronize()
    check(y, x, w, 1e-6, f"d={d}")


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 17, 255, 257, 1025])
def test_ragged_token_counts(cuda_lib, T):
    inp = to_dev(W.make_qknorm_inputs("prefill_gqa", seed=T, tokens=T))
    qo, ko = run_pair(inp)
    torch.cuda.synchronize()
    check(qo, inp["q"], inp["wq"], inp["eps"], f"T={T} q")
    check(ko, inp["k"], inp["wk"], inp["eps"], f"T={T} k")


def test_empty(cuda_lib):
    x = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    w = torch.ones(128, dtype=torch.bfloat16, device=DEV)
    y, _ = qk.qknorm_fused(x, x, w, w, 1e-6, 4)
    assert y.shape == (0, 128)


def test_fused_qkv_views_in_place(cuda_lib):
    # q and k as strided views of one [T, dq + 2 dk] projection output, normalised in place
    T, dq, dk = 96, 640, 128
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(T, dq + 2 * dk, generator=g).to(torch.bfloat16).to(DEV)
    wq = (1 + 0.1 * torch.randn(dq, generator=g)).to(torch.bfloat16).to(DEV)
    wk = (1 + 0.1 * torch.randn(dk, generator=g)).to(torch.bfloat16).to(DEV)
    before = qkv.clone()
    q, k = qkv[:, :dq], qkv[:, dq:dq + dk]
    qk.qknorm_fused(q, k, wq, wk, 1e-6, 8, inplace=True)
    torch.cuda.synchronize()
    check(qkv[:, :dq], before[:, :dq], wq, 1e-6, "in-place q view")
    check(qkv[:, dq:dq + dk], before[:, dq:dq + dk], wk, 1e-6, "in-place k view")
    assert torch.equal(qkv[:, dq + dk:], before[:, dq + dk:])  # v untouched


def test_strided_unaligned_pitch(cuda_lib):
    # a pitch that breaks 16-byte row alignment takes the element-wise kernel
    T, d = 33, 256
    g = torch.Generator().manual_seed(5)
    buf = torch.randn(T, d + 3, generator=g).to(torch.bfloat16).to(DEV)
    x = buf[:, :d]
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16).to(DEV)
    out = torch.empty(T, d + 5, dtype=torch.bfloat16, device=DEV)[:, :d]
    y, _ = qk.qknorm_fused(x, None, w, None, 1e-6, 4, q_out=out)
    torch.cuda.synchronize()
    assert y.data_ptr() == out.data_ptr()
    check(y, x.contiguous(), w, 1e-6, "unaligned pitch")


@pytest.mark.parametrize("act,wdt", [(torch.bfloat16, torch.float32), (torch.float32, torch.bfloat16)])
def test_mixed_weight_dtype(cuda_lib, act, wdt):
    T, d = 40, 2048
    g = torch.Generator().manual_seed(11)
    x = torch.randn(T, d, generator=g).to(act).to(DEV)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(wdt).to(DEV)
    y, _ = qk.qknorm_fused(x, x, w, w, 1e-6, 4)
    torch.cuda.synchronize()
    check(y, x, w, 1e-6, f"act={act} w={wdt}")


# -------------------------------------------------------------- degenerate values


def test_zero_rows_and_special_values(cuda_lib):
    d = 512
    x = torch.randn(6, d).to(torch.bfloat16)
    x[0] = 0.0                      # zero row, eps > 0 -> 0
    x[1, 7] = float("inf")          # inf -> NaN/inf in that row only
    x[2, 9] = float("nan")
    x[3] = 1e-30                    # tiny: eps dominates
    x[4] = 3e38                     # near bf16 max: the fp32 sum of squares overflows
    w = torch.ones(d, dtype=torch.bfloat16)
    xd, wd = x.to(DEV), w.to(DEV)
    y, _ = qk.qknorm_fused(xd, None, wd, None, 1e-6, 1)
    torch.cuda.synchronize()
    yc = y.float().cpu()
    assert torch.all(yc[0] == 0)
    assert torch.isnan(yc[1]).sum() + torch.isinf(yc[1]).sum() > 0
    assert torch.isnan(yc[2]).all()
    # fp32 statistics: S = inf gives inv = 0, so the row comes out as zeros
    # (the documented range limit of fp32 statistics; the fp64 oracle has none)
    assert torch.all(yc[4] == 0)
    ref3 = oracle.rmsnorm(x[3:4], w, 1e-6)
    assert_bf16_close(y[3:4], ref3, "tiny row")
    assert torch.equal(yc[5], yc[5])  # finite row untouched by neighbours
    assert_bf16_close(y[5:6], oracle.rmsnorm(x[5:6], w, 1e-6), "row after special values")


def test_zero_row_eps_zero_is_nan(cuda_lib):
    x = torch.zeros(2, 64, dtype=torch.float32, device=DEV)
    w = torch.ones(64, dtype=torch.float32, device=DEV)
    y, _ = qk.qknorm_fused(x, None, w, None, 0.0, 2)
    torch.cuda.synchronize()
    assert torch.isnan(y).all()


def test_scale_invariance_on_gpu(cuda_lib):
    # RMSNorm(c x) = RMSNorm(x) for a power-of-two c (exact scaling, eps tiny)
    x = torch.randn(64, 1024).to(torch.bfloat16).to(DEV)
    w = (1 + 0.1 * torch.randn(1024)).to(torch.bfloat16).to(DEV)
    a, _ = qk.qknorm_fused(x, None, w, None, 0.0, 8)
    b, _ = qk.qknorm_fused(x * 64, None, w, None, 0.0, 8)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_partial_stats_full_size_rows(cuda_lib):
    inp = W.make_qknorm_inputs("prefill_gqa", seed=0, device=DEV, tokens=4096)
    for key in ("q", "k"):
        p = qk.rmsnorm_partial_stats(inp[key], 8)
        torch.cuda.synchronize()
        ref = oracle.segment_partials(inp[key].cpu(), 8)
        assert_f32_close(p, ref, tol=PARTIAL_REL_TOL, what=f"partials {key}")
        # the combined statistic of the partials is the full-row statistic
        full = oracle.segment_partials(inp[key].cpu(), 1)[:, 0]
        np.testing.assert_allclose(oracle.combine_partials(p.cpu().double().numpy()), full, rtol=1e-5)


# --------------------------------------------------- a row's bits do not depend on its partner


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,n_seg", [(256, 1), (256, 8), (512, 4), (512, 8), (1024, 2), (1024, 8), (1000, 8),
                                     (1024, 16), (8192, 8)])
def test_rows_same_bits_beside_any_partner(cuda_lib, dtype, d, n_seg):
    # q and k share a launch only when each would take the same kernel on its own;
    # so rows normalised beside a 5120-wide job (the prefill arrangement), beside a
    # 512-wide one, or alone come out bit for bit the same, and the partial sums of
    # rmsnorm_partial_stats reproduce them (1000: the element-wise kernel)
    if dtype == torch.float32 and d == 1000:
        pytest.skip("1000 fp32 elements: 250 chunks, not a multiple of the segment count")
    T = 4099
    g = torch.Generator().manual_seed(d + n_seg)
    x = (torch.randn(T, d, generator=g) * 2).to(dtype).to(DEV)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(dtype).to(DEV)
    y, _ = qk.qknorm_fused(x, None, w, None, 1e-6, n_seg)
    xw = torch.randn(T, 5120, generator=g).to(dtype).to(DEV)
    ww = (1 + 0.1 * torch.randn(5120, generator=g)).to(dtype).to(DEV)
    xn = torch.randn(T, 512, generator=g).to(dtype).to(DEV)
    wn = (1 + 0.1 * torch.randn(512, generator=g)).to(dtype).to(DEV)
    y2, y3 = qk.qknorm_fused(xw, x, ww, w, 1e-6, n_seg)
    y4, y5 = qk.qknorm_fused(x, xn, w, wn, 1e-6, n_seg)
    yw, _ = qk.qknorm_fused(xw, None, ww, None, 1e-6, n_seg)
    yn, _ = qk.qknorm_fused(xn, None, wn, None, 1e-6, n_seg)
    p = qk.rmsnorm_partial_stats(x, n_seg)
    y6 = qk.rmsnorm_apply_partials(x, w, p, d, 1e-6)
    torch.cuda.synchronize()
    check(y, x, w, 1e-6, f"d={d} n_seg={n_seg} alone")
    bits = (lambda t: t.view(torch.int16)) if dtype == torch.bfloat16 else (lambda t: t.view(torch.int32))
    for other, what in ((y3, "beside 5120"), (y4, "beside 512"), (y6, "from rmsnorm_partial_stats")):
        assert torch.equal(bits(other), bits(y)), f"d={d} n_seg={n_seg}: {what} differs from alone"
    assert torch.equal(bits(y2), bits(yw)) and torch.equal(bits(y5), bits(yn)), "the partner's rows changed"
    assert_f32_close(p, oracle.segment_partials(x.cpu(), n_seg), tol=PARTIAL_REL_TOL, what=f"partials d={d}")


@pytest.mark.parametrize("d,n_seg", [(20480, 4), (20480, 16), (65536, 8)])
def test_wide_rows_partials_reproduce_fused(cuda_lib, d, n_seg):
    # rows past the staging ring (bf16: 40 and 128 KiB) are spread over the CTAs of a
    # cluster; the statistics alone take the same kernel, so their partials reproduce
    # qknorm_fused bit for bit, and the rows come out the same beside a narrow partner
    T = 129
    g = torch.Generator().manual_seed(d + n_seg)
    x = (torch.randn(T, d, generator=g) * 2).to(torch.bfloat16).to(DEV)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16).to(DEV)
    xn = torch.randn(T, 512, generator=g).to(torch.bfloat16).to(DEV)
    wn = torch.ones(512, dtype=torch.bfloat16, device=DEV)
    y, _ = qk.qknorm_fused(x, None, w, None, 1e-6, n_seg)
    y3, yn = qk.qknorm_fused(x, xn, w, wn, 1e-6, n_seg)
    p = qk.rmsnorm_partial_stats(x, n_seg)
    y2 = qk.rmsnorm_apply_partials(x, w, p, d, 1e-6)
    torch.cuda.synchronize()
    check(y, x, w, 1e-6, f"wide d={d} n_seg={n_seg}")
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16)), "partials do not reproduce qknorm_fused"
    assert torch.equal(y3.view(torch.int16), y.view(torch.int16)), "the narrow partner changed the rows"
    assert_f32_close(p, oracle.segment_partials(x.cpu(), n_seg), tol=PARTIAL_REL_TOL, what=f"partials d={d}")


@pytest.mark.parametrize("dq,dk,n_seg", [(128, 128, 1), (640, 128, 1), (1536, 256, 8), (1024, 1024, 4),
                                         (2048, 512, 2)])
def test_register_kernel_many_rows(cuda_lib, dq, dk, n_seg):
    # rows up to 4096 bytes (both tensors) are held in registers (normalised by
    # persistent blocks that stream the rows, several groups per block): many groups, a
    # ragged last one; the first rows again in a short launch give the same bits; the
    # statistics alone (register kernel up to 4096-byte rows) against the oracle
    T = 3001
    inp = W.make_qknorm_inputs("prefill_gqa", seed=dq + dk, device=DEV, tokens=T, dq=dq, dk=dk)
    qo, ko = qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], n_seg)
    qs, ks = qk.qknorm_fused(inp["q"][:67], inp["k"][:67], inp["wq"], inp["wk"], inp["eps"], n_seg)
    p = qk.rmsnorm_partial_stats(inp["q"], n_seg)
    torch.cuda.synchronize()
    check(qo, inp["q"], inp["wq"], inp["eps"], f"q d={dq}")
    check(ko, inp["k"], inp["wk"], inp["eps"], f"k d={dk}")
    assert torch.equal(qo[:67].view(torch.int16), qs.view(torch.int16))
    assert torch.equal(ko[:67].view(torch.int16), ks.view(torch.int16))
    assert_f32_close(p, oracle.segment_partials(inp["q"].cpu(), n_seg), tol=PARTIAL_REL_TOL, what="partials")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dq,dk,n_seg", [(4096, 1024, 16), (5120, 1024, 64), (5120, 5120, 40), (2048, 256, 32),
                                         (1024, 128, 16)])
def test_many_segments_staged(cuda_lib, dtype, dq, dk, n_seg):
    # 9 .. 64 segments: rows wider than 4 KiB through the staged kernel's many-segment
    # statistic (segments of 2 chunks: lanes skip segments; a count that is not a
    # power of two), narrower launches (2048 + 256 and 1024 + 128 bf16) through the
    # streaming register kernel's; ragged T, the partial sums themselves, and the same
    # bits from a short launch
    if dtype == torch.float32 and (dq // n_seg) % 4:
        pytest.skip("segments not whole fp32 chunks")
    T = 301
    g = torch.Generator().manual_seed(dq + dk + n_seg)
    q = (torch.randn(T, dq, generator=g) * 2).to(dtype).to(DEV)
    k = torch.randn(T, dk, generator=g).to(dtype).to(DEV)
    wq = (1 + 0.1 * torch.randn(dq, generator=g)).to(dtype).to(DEV)
    wk = (1 + 0.1 * torch.randn(dk, generator=g)).to(dtype).to(DEV)
    qo, ko = qk.qknorm_fused(q, k, wq, wk, 1e-6, n_seg)
    qs, ks = qk.qknorm_fused(q[:5], k[:5], wq, wk, 1e-6, n_seg)
    p = qk.rmsnorm_partial_stats(q, n_seg)
    torch.cuda.synchronize()
    check(qo, q, wq, 1e-6, f"q d={dq} n_seg={n_seg}")
    check(ko, k, wk, 1e-6, f"k d={dk} n_seg={n_seg}")
    bits = (lambda t: t.view(torch.int16)) if dtype == torch.bfloat16 else (lambda t: t)
    assert torch.equal(bits(qo[:5]), bits(qs)) and torch.equal(bits(ko[:5]), bits(ks))
    assert_f32_close(p, oracle.segment_partials(q.cpu(), n_seg), tol=PARTIAL_REL_TOL, what=f"partials n_seg={n_seg}")


@pytest.mark.parametrize("T,d,pad,n_seg,dtype", [
    (20001, 1024, 0, 8, torch.bfloat16),    # a segment is one chunk slot of each thread
    (20001, 1024, 40, 4, torch.bfloat16),   # two slots; pitched rows
    (200001, 128, 0, 1, torch.bfloat16),    # one segment: the whole row
    (40001, 64, 8, 2, torch.bfloat16),      # one chunk per row (one thread), pitched
    (30001, 1024, 0, 8, torch.float32),     # 4 KiB fp32 rows: 32 threads per row
    (30001, 2048, 0, 2, torch.bfloat16),    # four slots
    (20001, 640, 0, 8, torch.bfloat16),     # segments of 10 chunks over 16 threads: per-chunk index
    (60001, 512, 8, 16, torch.bfloat16),    # many segments, pitched
    (10001, 2048, 0, 64, torch.bfloat16),   # many segments, 4 KiB rows
])
def test_partial_stats_narrow_rows(cuda_lib, T, d, pad, n_seg, dtype):
    # the statistics alone of rows up to 4 KiB (the one-shot register kernel, and
    # for more than 8 segments the streaming one; segments of 1, 2 or 4 chunk slots
    # per thread, whole rows, and other widths): many row groups, a ragged last
    # one, pitched rows; the partials are the ones qknorm_fused combines for the
    # same rows (its output is reproduced bit for bit from them) and match the oracle
    g = torch.Generator().manual_seed(T + d + n_seg)
    x_full = (torch.randn(T, d + pad, generator=g) * 2).to(dtype).to(DEV)
    x = x_full[:, :d]
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(dtype).to(DEV)
    p = qk.rmsnorm_partial_stats(x, n_seg)
    y, _ = qk.qknorm_fused(x, None, w, None, 1e-6, n_seg)
    y2 = qk.rmsnorm_apply_partials(x, w, p, d, 1e-6)
    torch.cuda.synchronize()
    bits = (lambda t: t.view(torch.int16)) if dtype == torch.bfloat16 else (lambda t: t.view(torch.int32))
    assert torch.equal(bits(y2), bits(y))
    assert_f32_close(p, oracle.segment_partials(x.cpu(), n_seg), tol=PARTIAL_REL_TOL,
                     what=f"partials T={T} d={d} n_seg={n_seg}")


@pytest.mark.parametrize("T,dq,dk", [(50001, 128, 128), (20001, 1024, 1024), (10001, 2048, 512)])
def test_register_stream_many_groups(cuda_lib, T, dq, dk):
    # enough rows that each persistent block of the streaming register kernel walks
    # several row groups (loading the next while normalising the current), across
    # the q / k job boundary; sampled rows against the oracle, a short launch bitwise
    inp = W.make_qknorm_inputs("prefill_gqa", seed=T, device=DEV, tokens=T, dq=dq, dk=dk)
    qo, ko = qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], 4)
    qs, ks = qk.qknorm_fused(inp["q"][-300:], inp["k"][-300:], inp["wq"], inp["wk"], inp["eps"], 4)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(T)
    rows = torch.cat([torch.randint(0, T, (500,), generator=g), torch.arange(T - 40, T)]).to(DEV)
    check(qo[rows], inp["q"][rows], inp["wq"], inp["eps"], f"q T={T} d={dq}")
    check(ko[rows], inp["k"][rows], inp["wk"], inp["eps"], f"k T={T} d={dk}")
    assert torch.equal(qo[-300:].view(torch.int16), qs.view(torch.int16))
    assert torch.equal(ko[-300:].view(torch.int16), ks.view(torch.int16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dq,dk,n_seg", [(128, 128, 16), (256, 512, 32), (512, 512, 64), (1024, 128, 16),
                                         (1024, 1024, 64), (2048, 256, 32)])
def test_register_stream_many_segments(cuda_lib, dtype, dq, dk, n_seg):
    # rows of at most 4 KiB with 9 .. 64 segments: the streaming register kernel's
    # many-segment statistic (chunk sums parked in shared memory, each segment added
    # in chunk order); several row groups per persistent block, a ragged last group,
    # every row against the oracle, the partial sums, a short launch bit for bit
    if (dq * dtype.itemsize > 4096 or dk * dtype.itemsize > 4096
            or (dk // n_seg) * dtype.itemsize % 16 or (dq // n_seg) * dtype.itemsize % 16):
        pytest.skip("rows wider than 4 KiB or segments not whole 16-byte chunks")
    T = 20001
    g = torch.Generator().manual_seed(dq + dk + n_seg)
    q = (torch.randn(T, dq, generator=g) * 2).to(dtype).to(DEV)
    k = torch.randn(T, dk, generator=g).to(dtype).to(DEV)
    wq = (1 + 0.1 * torch.randn(dq, generator=g)).to(dtype).to(DEV)
    wk = (1 + 0.1 * torch.randn(dk, generator=g)).to(dtype).to(DEV)
    qo, ko = qk.qknorm_fused(q, k, wq, wk, 1e-6, n_seg)
    qs, ks = qk.qknorm_fused(q[-77:], k[-77:], wq, wk, 1e-6, n_seg)
    pq = qk.rmsnorm_partial_stats(q, n_seg)
    pk = qk.rmsnorm_partial_stats(k[:333], n_seg)
    torch.cuda.synchronize()
    check(qo, q, wq, 1e-6, f"q d={dq} n_seg={n_seg}")
    check(ko, k, wk, 1e-6, f"k d={dk} n_seg={n_seg}")
    bits = (lambda t: t.view(torch.int16)) if dtype == torch.bfloat16 else (lambda t: t)
    assert torch.equal(bits(qo[-77:]), bits(qs)) and torch.equal(bits(ko[-77:]), bits(ks))
    assert_f32_close(pq, oracle.segment_partials(q.cpu(), n_seg), tol=PARTIAL_REL_TOL, what="q partials")
    assert_f32_close(pk, oracle.segment_partials(k[:333].cpu(), n_seg), tol=PARTIAL_REL_TOL, what="k partials")


@pytest.mark.parametrize("act,wdt", [(torch.float32, torch.float32), (torch.bfloat16, torch.float32),
                                     (torch.float32, torch.bfloat16)])
def test_register_stream_in_place_and_dtypes(cuda_lib, act, wdt):
    # the streaming register kernel in place (each row read and written by its own
    # threads, the next rows already loading) and with every dtype pairing
    T, dq, dk = 40000, 512, 128
    g = torch.Generator().manual_seed(17)
    q = (torch.randn(T, dq, generator=g) * 3).to(act).to(DEV)
    k = torch.randn(T, dk, generator=g).to(act).to(DEV)
    wq = (1 + 0.1 * torch.randn(dq, generator=g)).to(wdt).to(DEV)
    wk = (1 + 0.1 * torch.randn(dk, generator=g)).to(wdt).to(DEV)
    qo, ko = qk.qknorm_fused(q, k, wq, wk, 1e-6, 2)
    q2, k2 = q.clone(), k.clone()
    qk.qknorm_fused(q2, k2, wq, wk, 1e-6, 2, inplace=True)
    torch.cuda.synchronize()
    bits = (lambda t: t.view(torch.int16)) if act == torch.bfloat16 else (lambda t: t.view(torch.int32))
    assert torch.equal(bits(qo), bits(q2)) and torch.equal(bits(ko), bits(k2))
    rows = torch.randint(0, T, (300,), generator=g).to(DEV)
    check(qo[rows], q[rows], wq, 1e-6, "q sampled")
    check(ko[rows], k[rows], wk, 1e-6, "k sampled")


def test_long_launch_matches_short_launch(cuda_lib):
    # batch invariance: rows normalised in a launch of 65536 + 65536 rows and in a
    # launch of a few hundred agree bit for bit
    inp = W.make_qknorm_inputs("long_context", seed=5, device=DEV, tokens=65536)
    qo, ko = run_pair(inp)
    n = 777
    qs, ks = qk.qknorm_fused(inp["q"][:n], inp["k"][:n], inp["wq"], inp["wk"], inp["eps"], inp["n_seg"])
    torch.cuda.synchronize()
    assert torch.equal(qo[:n].view(torch.int16), qs.view(torch.int16))
    assert torch.equal(ko[:n].view(torch.int16), ks.view(torch.int16))
    g = torch.Generator().manual_seed(1)
    rows = torch.randint(0, 65536, (64,), generator=g).to(DEV)
    check(qo[rows], inp["q"][rows], inp["wq"], inp["eps"], "long launch q sampled")


def test_binding_rejects_mismatched_outputs(cuda_lib):
    # caller-provided outputs must have exactly the shape and dtype the call writes:
    # the binding refuses them before anything is launched
    q = torch.randn(16, 256, device=DEV).to(torch.bfloat16)
    w = torch.ones(256, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        qk.qknorm_fused(q, None, w, None, 1e-6, 1, q_out=torch.empty(8, 256, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(ValueError):
        qk.qknorm_fused(q, None, w, None, 1e-6, 1, q_out=torch.empty(16, 256, dtype=torch.float32, device=DEV))
    p = qk.rmsnorm_partial_stats(q, 1)
    with pytest.raises(ValueError):
        qk.rmsnorm_apply_partials(q, w, p, 256, 1e-6, out=torch.empty(16, 128, dtype=torch.bfloat16, device=DEV))
    x = torch.randn(128, 256, device=DEV).to(torch.bfloat16)
    Wf = torch.randn(384, 256, device=DEV).to(torch.bfloat16)
    wqk = torch.ones(128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        qk.flashnorm_proj(x, Wf, 1e-6, out=torch.empty(128, 384, dtype=torch.float32, device=DEV))
    with pytest.raises(ValueError):
        qk.qkv_proj_qknorm(x, Wf, 128, 128, 128, wqk, wqk, 1e-6, out=torch.empty(128, 256, dtype=torch.bfloat16,
                                                                                  device=DEV))
    with pytest.raises(ValueError):
        qk.qkv_norm_proj(x, Wf, 128, 128, 128, wqk, wqk, wqk, 1e-6, out=torch.empty(64, 384, dtype=torch.bfloat16,
                                                                                     device=DEV))
    torch.cuda.synchronize()
    assert qk.load_library().qkn_check_device(None) == 0

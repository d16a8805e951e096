"""GPU parity of the tensor-parallel apply step and of the RMSNorm elimination.

* rmsnorm_apply_partials with the partials of rmsnorm_partial_stats must give
  exactly (bit for bit) what qknorm_fused gives for the same rows and n_seg:
  the same segment sums, combined in the same order, applied the same way.
* SwiftQK's tensor-parallel form emulated on one GPU: the row split into
  shard views, one partial per shard, the [shards, rows] partials combined in
  shard order -- within 1 bf16 ulp of the fp64 oracle.
* tp_qknorm through torch.distributed with one NCCL rank, both exchange
  schedules, and the All-Gather form it is compared with.
* qkv_norm_proj (pre-attention RMSNorm eliminated) against the full oracle
  path RMSNorm(x) W followed by the q / k / v norms: relative Frobenius 1e-2.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch

import oracle
import rmsnorm_qknorm_b200 as qk
from parity import PROJ_FROB_TOL, assert_bf16_close, assert_f32_close, frobenius_rel
from rmsnorm_qknorm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,tokens", [("prefill_gqa", 300), ("long_context", 257), ("tiny", 64)])
def test_apply_partials_reproduces_fused(cuda_lib, name, tokens):
    inp = W.make_qknorm_inputs(name, seed=1, device=DEV, tokens=tokens)
    qo, ko = qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], inp["n_seg"])
    for x, w, y in ((inp["q"], inp["wq"], qo), (inp["k"], inp["wk"], ko)):
        p = qk.rmsnorm_partial_stats(x, inp["n_seg"])
        y2 = qk.rmsnorm_apply_partials(x, w, p, x.shape[1], inp["eps"])
        torch.cuda.synchronize()
        assert torch.equal(y2.view(torch.int16) if y2.dtype == torch.bfloat16 else y2.view(torch.int32),
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32))


@pytest.mark.parametrize("n_seg", [16, 64])
def test_apply_partials_reproduces_fused_many_segments(cuda_lib, n_seg):
    # with more than 8 segments too: the statistics-only partials are bit for bit
    # the ones qknorm_fused combines (the same many-segment statistic)
    inp = W.make_qknorm_inputs("prefill_gqa", seed=n_seg, device=DEV, tokens=200)
    qo, ko = qk.qknorm_fused(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"], n_seg)
    for x, w, y in ((inp["q"], inp["wq"], qo), (inp["k"], inp["wk"], ko)):
        p = qk.rmsnorm_partial_stats(x, n_seg)
        y2 = qk.rmsnorm_apply_partials(x, w, p, x.shape[1], inp["eps"])
        torch.cuda.synchronize()
        assert torch.equal(y2.view(torch.int16), y.view(torch.int16))


@pytest.mark.parametrize("shards", [2, 4, 8])
def test_tensor_parallel_emulated_on_one_gpu(cuda_lib, shards):
    inp = W.make_qknorm_inputs("prefill_gqa", seed=2, device=DEV, tokens=129)
    for x, w in ((inp["q"], inp["wq"]), (inp["k"], inp["wk"])):
        T, d = x.shape
        s = d // shards
        parts = torch.stack([qk.rmsnorm_partial_stats(x[:, j * s:(j + 1) * s], 1)[:, 0] for j in range(shards)])
        y = torch.empty_like(x)
        for j in range(shards):
            qk.rmsnorm_apply_partials(x[:, j * s:(j + 1) * s], w[j * s:(j + 1) * s], parts, d, inp["eps"],
                                      out=y[:, j * s:(j + 1) * s])
        torch.cuda.synchronize()
        assert_bf16_close(y, oracle.rmsnorm(x.cpu(), w.cpu(), inp["eps"]), f"{shards} shards d={d}")


def test_tensor_parallel_full_prefill_sampled(cuda_lib):
    # the prefill GQA workload at full size split 8 ways as the tensor-parallel bench
    # splits it (q 8 x 640, k 8 x 128): every shard's partials, combined in shard
    # order, then each shard's apply; sampled rows against the oracle
    inp = W.make_qknorm_inputs("prefill_gqa", seed=0, device=DEV)
    g = torch.Generator().manual_seed(9)
    rows = torch.randint(0, inp["q"].shape[0], (256,), generator=g).to(DEV)
    for x, w in ((inp["q"], inp["wq"]), (inp["k"], inp["wk"])):
        T, d = x.shape
        s = d // 8
        slices = [x[:, j * s:(j + 1) * s].contiguous() for j in range(8)]
        parts = torch.stack([qk.rmsnorm_partial_stats(sl, 1)[:, 0] for sl in slices])  # [8, T]
        y = torch.cat([qk.rmsnorm_apply_partials(slices[j], w[j * s:(j + 1) * s].contiguous(), parts.t(), d,
                                                 inp["eps"]) for j in range(8)], dim=1)
        torch.cuda.synchronize()
        assert_bf16_close(y[rows], oracle.rmsnorm(x[rows].cpu(), w.cpu(), inp["eps"]), f"8 shards d={d} sampled")


def test_apply_partials_fp32_and_unaligned(cuda_lib):
    g = torch.Generator().manual_seed(4)
    x = torch.randn(33, 100, generator=g).to(DEV)          # d not a multiple of 4: element path
    w = (1 + 0.1 * torch.randn(100, generator=g)).to(DEV)
    p = qk.rmsnorm_partial_stats(x, 4)
    y = qk.rmsnorm_apply_partials(x, w, p, 100, 1e-5)
    torch.cuda.synchronize()
    assert_f32_close(y, oracle.rmsnorm(x.cpu(), w.cpu(), 1e-5), what="fp32 element path")


@pytest.mark.parametrize("d,n_seg", [(8, 1), (64, 2), (136, 1), (1032, 3), (200, 4)])
def test_apply_partials_row_widths(cuda_lib, d, n_seg):
    # narrow rows share a warp (1, 2, 4 ... threads per row), 200 bf16 is not whole
    # chunks per segment; 1000 rows leave a ragged last block
    g = torch.Generator().manual_seed(d)
    x = (torch.randn(1000, d, generator=g) * 3).to(torch.bfloat16).to(DEV)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16).to(DEV)
    p = qk.rmsnorm_partial_stats(x, n_seg)
    y = qk.rmsnorm_apply_partials(x, w, p, d, 1e-6)
    torch.cuda.synchronize()
    assert_bf16_close(y, oracle.rmsnorm(x.cpu(), w.cpu(), 1e-6), f"apply d={d} n_seg={n_seg}")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_tp_qknorm_single_rank_nccl(cuda_lib):
    import torch.distributed as dist
    from rmsnorm_qknorm_b200.tp import allgather_qknorm, tp_qknorm
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        inp = W.make_qknorm_inputs("decode", seed=3, device=DEV, tokens=40)
        qo, ko = tp_qknorm(inp["q"], inp["k"], inp["wq"], inp["wk"], 5120, 5120, inp["eps"])
        q1, k1 = tp_qknorm(inp["q"], inp["k"], inp["wq"], inp["wk"], 5120, 5120, inp["eps"], overlap=False)
        # the All-Gather form the pages compare against: the same rows, normalised whole
        qa, ka = allgather_qknorm(inp["q"], inp["k"], inp["wq"], inp["wk"], inp["eps"])
        torch.cuda.synchronize()
        assert_bf16_close(qo, oracle.rmsnorm(inp["q"].cpu(), inp["wq"].cpu(), inp["eps"]), "tp q")
        assert_bf16_close(ko, oracle.rmsnorm(inp["k"].cpu(), inp["wk"].cpu(), inp["eps"]), "tp k")
        assert_bf16_close(qa, oracle.rmsnorm(inp["q"].cpu(), inp["wq"].cpu(), inp["eps"]), "all-gather q")
        assert_bf16_close(ka, oracle.rmsnorm(inp["k"].cpu(), inp["wk"].cpu(), inp["eps"]), "all-gather k")
        # the two exchange schedules combine the same partials in the same order
        assert torch.equal(q1.view(torch.int16), qo.view(torch.int16))
        assert torch.equal(k1.view(torch.int16), ko.view(torch.int16))
        # captured in a CUDA graph (collectives included) and replayed: the same bits
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            qg, kg = tp_qknorm(inp["q"], inp["k"], inp["wq"], inp["wk"], 5120, 5120, inp["eps"])
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(qg.view(torch.int16), qo.view(torch.int16))
        assert torch.equal(kg.view(torch.int16), ko.view(torch.int16))
        del g
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,K,nq,nk,nv,n_seg", [(200, 256, 256, 128, 128, 4), (64, 512, 512, 128, 0, 8),
                                               (129, 1024, 640, 128, 128, 2)])
def test_qkv_norm_proj_elimination(cuda_lib, M, K, nq, nk, nv, n_seg):
    g = torch.Generator().manual_seed(M + K)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w_pre = (1 + 0.1 * torch.randn(K, generator=g)).to(torch.bfloat16)
    Wm = (torch.randn(K, nq + nk + nv, generator=g) / K ** 0.5).to(torch.bfloat16)
    wq = (1 + 0.1 * torch.randn(nq, generator=g)).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(nk, generator=g)).to(torch.bfloat16)
    wv = (1 + 0.1 * torch.randn(max(nv, 1), generator=g)).to(torch.bfloat16)[:nv]
    Wf = qk.flashnorm_fold_weights(w_pre.to(DEV), Wm.to(DEV))
    y = qk.qkv_norm_proj(x.to(DEV), Wf, nq, nk, nv, wq.to(DEV), wk.to(DEV), wv.to(DEV) if nv else None,
                         1e-6, n_seg)
    torch.cuda.synchronize()
    # full reference path: pre-attention RMSNorm (eps 0, the exact identity) then project, then norms
    u = oracle.norm_then_project(x, w_pre, Wm, 0.0)
    ref = np.concatenate([oracle.rmsnorm(u[:, :nq], wq, 1e-6), oracle.rmsnorm(u[:, nq:nq + nk], wk, 1e-6)]
                         + ([oracle.rmsnorm(u[:, nq + nk:], wv, 1e-6)] if nv else []), axis=1)
    err = frobenius_rel(y, ref)
    assert err <= PROJ_FROB_TOL, f"relative Frobenius error {err:.3e}"

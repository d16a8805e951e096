"""Multi-process host logic on CPU: world size 2 over gloo.

The GPU path needs no collective (tokens are independent); these tests cover
what the ranks do share: seeding, row sharding, the max-over-ranks timing and
the token accounting of the benchmark's value.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rmsnorm_qknorm_b200 import dist as qdist
from rmsnorm_qknorm_b200 import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's elapsed time differs; everyone must see the max
        elapsed = 10.0 + 5.0 * rank
        mx = qdist.max_over_ranks(elapsed)
        tokens = qdist.sum_over_ranks(128.0)
        # strong-scaling shards of one batch: disjoint, covering, reassembled in order
        T = 1001
        start, stop = qdist.shard_rows(T, rank, world)
        inp = W.make_qknorm_inputs("prefill_gqa", seed=0, tokens=T, dq=64, dk=16)
        mine = inp["q"][start:stop].float()
        # reassemble the shards on every rank through padded buffers (shards differ by <= 1 row)
        pad = (T + world - 1) // world
        padded = torch.zeros(pad, 64)
        padded[: stop - start] = mine
        pbufs = [torch.empty(pad, 64) for _ in range(world)]
        dist.all_gather(pbufs, padded)
        spans = [qdist.shard_rows(T, r, world) for r in range(world)]
        gathered = torch.cat([pb[: b - a] for pb, (a, b) in zip(pbufs, spans)])
        # weak scaling: rank seeds give different batches, rank 0 keeps the workload seed
        s0 = qdist.rank_seed(0, rank)
        out[rank] = {
            "max": mx, "tokens": tokens, "shard": (start, stop),
            "reassembled_equal": bool(torch.equal(gathered, inp["q"].float())),
            "seed": s0,
        }
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0]["max"] == res[1]["max"] == 15.0
    assert res[0]["tokens"] == res[1]["tokens"] == 256.0
    assert res[0]["shard"] == (0, 501) and res[1]["shard"] == (501, 1001)
    assert res[0]["reassembled_equal"] and res[1]["reassembled_equal"]
    assert res[0]["seed"] == 0 and res[1]["seed"] != 0


@pytest.mark.parametrize("total,world", [(0, 1), (1, 4), (7, 3), (131072, 8), (16383, 8)])
def test_shard_rows_partition(total, world):
    spans = [qdist.shard_rows(total, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == total
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_shard_rows_rejects_bad_requests():
    with pytest.raises(ValueError):
        qdist.shard_rows(10, 2, 2)
    with pytest.raises(ValueError):
        qdist.shard_rows(10, 0, 0)


def test_max_without_process_group_is_identity():
    assert qdist.max_over_ranks(3.5) == 3.5


def _gather_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from rmsnorm_qknorm_b200.tp import gather_partials
        local = torch.arange(5, dtype=torch.float32) + 100 * rank  # this rank's per-row partials
        g = gather_partials(local)
        out[rank] = g.tolist()
    finally:
        dist.destroy_process_group()


def test_scalar_partials_all_gather_rank_order():
    # tensor-parallel QK-Norm exchanges only [rows] fp32 per rank; the gathered
    # [world, rows] array is in rank order on every rank (the fixed combine order)
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_gather_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    expect = [[float(i) for i in range(5)], [100.0 + i for i in range(5)]]
    assert res[0] == expect and res[1] == expect


def test_gather_without_process_group_is_local():
    from rmsnorm_qknorm_b200.tp import gather_partials
    g = gather_partials(torch.ones(3))
    assert tuple(g.shape) == (1, 3)


def _slices_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from rmsnorm_qknorm_b200.tp import gather_slices
        full = torch.arange(5 * 12, dtype=torch.float32).view(5, 12)
        mine = full[:, rank * 6:(rank + 1) * 6].contiguous()
        out[rank] = bool(torch.equal(gather_slices(mine), full))
    finally:
        dist.destroy_process_group()


def test_gather_slices_reassembles_rows():
    # the All-Gather baseline's exchange: every rank rebuilds the full rows in rank order
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_slices_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] and out[1]


def _tp_flow_worker(rank, world, port, overlap, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from rmsnorm_qknorm_b200 import tp
        seen = []

        def stats(x, o):  # stand-in for the statistic kernel: fp32 sum of squares of the slice
            o.copy_((x.double() ** 2).sum(1).float())

        def apply(x, w, parts_t, d_full, eps, inplace):  # stand-in for the apply kernel
            seen.append(parts_t.clone())
            return x * torch.rsqrt(parts_t.sum(1) / d_full + eps)[:, None] * w

        tp._stats, tp._apply = stats, apply
        g = torch.Generator().manual_seed(7)
        q, k = torch.randn(6, 16, generator=g), torch.randn(6, 8, generator=g)
        dq, dk = 16 // world, 8 // world
        qs, ks = q[:, rank * dq:(rank + 1) * dq], k[:, rank * dk:(rank + 1) * dk]
        wq, wk = torch.ones(dq), torch.ones(dk)
        qo, ko = tp.tp_qknorm(qs, ks, wq, wk, 16, 8, 1e-6, overlap=overlap)
        expect_q = torch.stack([(q[:, j * dq:(j + 1) * dq].double() ** 2).sum(1).float() for j in range(world)], 1)
        expect_k = torch.stack([(k[:, j * dk:(j + 1) * dk].double() ** 2).sum(1).float() for j in range(world)], 1)
        ref_q = qs * torch.rsqrt((q * q).mean(1) + 1e-6)[:, None]
        ref_k = ks * torch.rsqrt((k * k).mean(1) + 1e-6)[:, None]
        out[rank] = {
            "parts_rank_order": bool(torch.equal(seen[0], expect_q) and torch.equal(seen[1], expect_k)),
            "q_close": float((qo - ref_q).abs().max()), "k_close": float((ko - ref_k).abs().max()),
        }
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("overlap", [True, False])
def test_tp_qknorm_exchange_flow(overlap):
    # both exchange schedules of tp_qknorm (q's all-gather in flight while k's
    # statistic runs, or one [2, rows] all-gather) hand every rank the partials
    # of all ranks in rank order, and each rank's slice comes out normalised by
    # the whole row's statistic
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_tp_flow_worker, args=(world, _free_port(), overlap, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r]["parts_rank_order"], r
        assert out[r]["q_close"] < 1e-5 and out[r]["k_close"] < 1e-5, out[r]

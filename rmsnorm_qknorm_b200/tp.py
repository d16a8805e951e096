"""Tensor-parallel QK-Norm across ranks (SwiftQK, abstract).

Each rank holds a contiguous slice of every query (key) row.  The normalising
factor depends on the whole row, so each rank computes its slice's scalar sum
of squares per row (rmsnorm_partial_stats), the ranks exchange only these
scalars (an all-gather of ``[rows]`` fp32 per rank -- 4 bytes per row per
rank instead of the activation slices), and each rank normalises its own
slice from the gathered partials combined in fixed rank order
(rmsnorm_apply_partials).  Every arithmetic step runs in the library's
kernels; this module only moves the scalars with ``torch.distributed``.

``allgather_qknorm`` is the form SwiftQK is measured against: the activation
slices themselves are gathered and the full rows normalised.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import rmsnorm_apply_partials, rmsnorm_partial_stats

__all__ = ["gather_partials", "tp_rmsnorm", "tp_qknorm", "gather_slices", "allgather_qknorm"]


def gather_partials(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather each rank's [rows] fp32 partials into [world, rows] (rank order)."""
    if local.dim() != 1 or local.dtype != torch.float32:
        raise ValueError("local partials must be a 1-D fp32 tensor")
    if not (dist.is_available() and dist.is_initialized()):
        return local.unsqueeze(0)
    world = dist.get_world_size(group)
    out = torch.empty((world * local.shape[0],), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, local.contiguous(), group=group)
    return out.view(world, local.shape[0])


def tp_rmsnorm(x_shard: torch.Tensor, w_shard: torch.Tensor, d_full: int, eps: float = 1e-6, *,
               group=None, inplace: bool = False) -> torch.Tensor:
    """RMSNorm of rows split across ranks: x_shard [rows, d_full / world] on every rank."""
    local = rmsnorm_partial_stats(x_shard, 1)[:, 0].contiguous()
    parts = gather_partials(local, group)  # [world, rows], combined in rank order
    return rmsnorm_apply_partials(x_shard, w_shard, parts, d_full, eps, inplace=inplace)


def _stats(x: torch.Tensor, out: torch.Tensor) -> None:
    """[rows] fp32 sums of squares of the slice x into out (the library's kernel)."""
    rmsnorm_partial_stats(x, 1, out=out.view(-1, 1))


def _apply(x, w, parts_t, d_full, eps, inplace):
    """Normalise the slice x from its gathered partials parts_t [rows, world] (the library's kernel)."""
    return rmsnorm_apply_partials(x, w, parts_t, d_full, eps, inplace=inplace)


def tp_qknorm(q_shard: torch.Tensor, k_shard: torch.Tensor, wq_shard: torch.Tensor,
              wk_shard: torch.Tensor, dq_full: int, dk_full: int, eps: float = 1e-6, *, group=None,
              inplace: bool = False, overlap: bool = True):
    """Layerwise QK-Norm under tensor parallelism; returns the normalised local slices.

    The only data that cross ranks are the per-row scalar sums of squares of
    q's and k's slices.  With ``overlap`` the exchange of q's partials is in
    flight (on the communicator's stream) while k's partials are computed, and
    k's exchange while q's slice is normalised -- the exchange hidden behind
    independent work, as in SwiftQK.  Without it both go in one all-gather of
    ``[2, rows]`` fp32 per rank.  Either way every rank combines the gathered
    partials in rank order, so all ranks get the same statistic bit for bit.
    """
    stats, apply = _stats, _apply
    rows = q_shard.shape[0]
    if k_shard.shape[0] != rows:
        raise ValueError(f"q has {rows} rows but k has {k_shard.shape[0]}")
    dev = q_shard.device
    local = torch.empty((2, rows), dtype=torch.float32, device=dev)
    if not (dist.is_available() and dist.is_initialized()):
        stats(q_shard, local[0])
        stats(k_shard, local[1])
        parts = local.unsqueeze(0)                       # [1, 2, rows]
        return (apply(q_shard, wq_shard, parts[:, 0].t(), dq_full, eps, inplace),
                apply(k_shard, wk_shard, parts[:, 1].t(), dk_full, eps, inplace))
    world = dist.get_world_size(group)
    if overlap:
        gq = torch.empty((world, rows), dtype=torch.float32, device=dev)
        gk = torch.empty((world, rows), dtype=torch.float32, device=dev)
        stats(q_shard, local[0])
        work_q = dist.all_gather_into_tensor(gq.view(-1), local[0], group=group, async_op=True)
        stats(k_shard, local[1])                          # overlaps q's exchange
        work_k = dist.all_gather_into_tensor(gk.view(-1), local[1], group=group, async_op=True)
        work_q.wait()
        qo = apply(q_shard, wq_shard, gq.t(), dq_full, eps, inplace)   # overlaps k's exchange
        work_k.wait()
        ko = apply(k_shard, wk_shard, gk.t(), dk_full, eps, inplace)
        return qo, ko
    gathered = torch.empty((world, 2, rows), dtype=torch.float32, device=dev)
    stats(q_shard, local[0])
    stats(k_shard, local[1])
    dist.all_gather_into_tensor(gathered.view(-1), local.view(-1), group=group)
    return (apply(q_shard, wq_shard, gathered[:, 0].t(), dq_full, eps, inplace),
            apply(k_shard, wk_shard, gathered[:, 1].t(), dk_full, eps, inplace))


def gather_slices(x_shard: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's [rows, d/world] slice into full [rows, d] rows (rank order)."""
    if not (dist.is_available() and dist.is_initialized()):
        return x_shard
    world = dist.get_world_size(group)
    rows, d_loc = x_shard.shape
    buf = torch.empty((world, rows, d_loc), dtype=x_shard.dtype, device=x_shard.device)
    dist.all_gather_into_tensor(buf.view(-1), x_shard.contiguous().view(-1), group=group)
    return buf.permute(1, 0, 2).reshape(rows, world * d_loc)


def allgather_qknorm(q_shard: torch.Tensor, k_shard: torch.Tensor, wq: torch.Tensor, wk: torch.Tensor,
                     eps: float = 1e-6, *, group=None):
    """The All-Gather form SwiftQK is measured against: every rank gathers the full
    q and k rows (the activation slices cross the interconnect) and normalises
    them whole with qknorm_fused; wq, wk are the full weights.  Returns this
    rank's slices of the normalised rows."""
    from . import qknorm_fused
    rank = dist.get_rank(group) if (dist.is_available() and dist.is_initialized()) else 0
    q_full, k_full = gather_slices(q_shard, group), gather_slices(k_shard, group)
    qo, ko = qknorm_fused(q_full, k_full, wq, wk, eps, 1)
    dq, dk = q_shard.shape[1], k_shard.shape[1]
    return qo[:, rank * dq:(rank + 1) * dq], ko[:, rank * dk:(rank + 1) * dk]

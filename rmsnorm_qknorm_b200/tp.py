"""Tensor-parallel QK-Norm across ranks (SwiftQK, abstract).

Each rank holds a contiguous slice of every query (key) row.  The normalising
factor depends on the whole row, so each rank computes its slice's scalar sum
of squares per row (rmsnorm_partial_stats), the ranks exchange only these
scalars (an all-gather of ``[rows]`` fp32 per rank -- 4 bytes per row per
rank instead of the activation slices), and each rank normalises its own
slice from the gathered partials combined in fixed rank order
(rmsnorm_apply_partials).  Every arithmetic step runs in the library's
kernels; this module only moves the scalars with ``torch.distributed``.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import rmsnorm_apply_partials, rmsnorm_partial_stats

__all__ = ["gather_partials", "tp_rmsnorm", "tp_qknorm"]


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


def tp_qknorm(q_shard: torch.Tensor, k_shard: torch.Tensor, wq_shard: torch.Tensor,
              wk_shard: torch.Tensor, dq_full: int, dk_full: int, eps: float = 1e-6, *, group=None,
              inplace: bool = False):
    """Layerwise QK-Norm under tensor parallelism; returns the normalised local slices."""
    return (tp_rmsnorm(q_shard, wq_shard, dq_full, eps, group=group, inplace=inplace),
            tp_rmsnorm(k_shard, wk_shard, dk_full, eps, group=group, inplace=inplace))

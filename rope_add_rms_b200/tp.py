"""Tensor-parallel all-reduce + residual add + RMSNorm across the ranks of a process group.

A row-parallel layer leaves each rank with a partial output; the decoder sums them
(all-reduce), adds the residual and normalises (miniVLLM Layers page, sections
RowParallelLinear and LayerNorm).  Here the collective only moves data: every rank's
partial is gathered into this GPU's memory in rank order (NCCL all-gather over NVLink),
and one kernel of this library sums the gathered parts in rank order, adds the residual
and normalises.  Every rank therefore computes bit-identical y and h.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import nv_allreduce_add_rms_norm


def gather_parts(partial: torch.Tensor, group=None, out: torch.Tensor | None = None):
    """Every rank's ``partial`` in rank order, as views of one [world, *shape] tensor."""
    world = dist.get_world_size(group)
    partial = partial.contiguous()
    if out is None:
        out = torch.empty((world, *partial.shape), dtype=partial.dtype, device=partial.device)
    if out.shape != (world, *partial.shape) or out.dtype != partial.dtype:
        raise ValueError("gather buffer must be [world, *partial.shape] of the same dtype")
    dist.all_gather(list(out.unbind(0)), partial, group=group)
    return list(out.unbind(0))


def allreduce_add_rms_norm(partial: torch.Tensor, residual: torch.Tensor, w, eps: float = 1e-5,
                           group=None, gather_buf: torch.Tensor | None = None,
                           residual_in_place: bool = False):
    """(y, h): h = sum over ranks of ``partial`` (rank order, rounded once) + residual,
    y = RmsNorm(h) * w.  With ``residual_in_place`` h is written over ``residual``."""
    parts = gather_parts(partial, group, gather_buf)
    y = torch.empty_like(residual)
    h = residual if residual_in_place else torch.empty_like(residual)
    nv_allreduce_add_rms_norm(parts, residual, w, y, h, eps)
    return y, h

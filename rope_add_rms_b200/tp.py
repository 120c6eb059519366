"""Tensor-parallel all-reduce + residual add + RMSNorm across the ranks of a process group.

A row-parallel layer leaves each rank with a partial output; the decoder sums them
(all-reduce), adds the residual and normalises (miniVLLM Layers page, sections
RowParallelLinear and LayerNorm).  Two forms, both ending in one kernel of this library
that sums the parts in rank order, adds the residual and normalises, so every rank computes
bit-identical y and h:
  - allreduce_add_rms_norm (the default): the collective only moves data -- every rank's
    partial is gathered into this GPU's memory in rank order (NCCL all-gather);
  - PeerAllReduce: the one-shot form -- the kernel reads the other ranks' partials straight
    from their GPUs' memory (CUDA IPC mappings), after a device-side flag handshake.
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


class PeerAllReduce:
    """The one-shot form: every rank reads the others' partial outputs directly from their
    GPUs' memory (CUDA IPC mappings over NVLink), with no gather.

    Set-up, once per group and shape: each rank allocates, in one device allocation of its
    own, two partial buffers (double buffering) and a flag array of one int64 per rank,
    exports its IPC handle, and all ranks exchange the handles over the process group (an
    all-gather of objects) and map the others'.  Per step: the caller writes this rank's partial into
    ``partial()`` on the current stream, then calls the object, which

      1. advances the step number (epoch 1, 2, ...: every rank must take the same steps);
      2. publishes the epoch into this rank's slot of every rank's flag array
         (nv_tp_publish: after the partial is complete, a system-scope fence and release
         stores);
      3. runs nv_allreduce_add_rms_norm_peers on the parts of this epoch's buffer of every
         rank, which waits on the device (bounded) until every rank has published the epoch.

    The next step's partial goes to the other buffer, so a buffer is rewritten only after
    every rank has finished reading it (a rank publishes step e + 1 after its step-e read,
    which precedes it on the stream).  The collective only carries the handles, once.
    """

    def __init__(self, shape, dtype, group=None, device=None, lib=None):
        from . import (ipc_export, ipc_import, nv_allreduce_add_rms_norm_peers,
                       nv_tp_publish)
        self._lib = lib or {"export": ipc_export, "import": ipc_import,
                            "publish": nv_tp_publish, "reduce": nv_allreduce_add_rms_norm_peers}
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if not 1 <= self.world <= 8:
            raise ValueError("the one-shot form takes 1 to 8 ranks")
        device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.shape = tuple(shape)
        n = 1
        for d in self.shape:
            n *= d
        esz = torch.empty((), dtype=dtype).element_size()
        self.slot_bytes = n * esz
        # one allocation (one handle) per rank: two partial slots, then the flags (zeroed)
        self.flags_off = (2 * self.slot_bytes + 255) // 256 * 256
        self.raw = torch.zeros(self.flags_off + 8 * self.world, dtype=torch.uint8, device=device)
        self.bufs = self.raw[:2 * self.slot_bytes].view(dtype).view(2, *self.shape)
        self.flags = self.raw[self.flags_off:].view(torch.int64)
        mine = (self.rank, self._lib["export"](self.raw))
        table = [None] * self.world
        dist.all_gather_object(table, mine, group=group)
        self.buf_ptrs, self.flag_ptrs, self._mapped = [], [], []
        for r, (rank, handle) in enumerate(table):
            if rank != r:
                raise RuntimeError(f"handle table out of rank order at {r}: {rank}")
            if r == self.rank:
                base = self.raw.data_ptr()
            else:
                base = self._lib["import"](*handle)
                self._mapped.append((base, handle[1]))
            self.buf_ptrs.append(base)
            self.flag_ptrs.append(base + self.flags_off)
        self.epoch = 0

    def partial(self):
        """Where this rank writes its partial output of the next step."""
        return self.bufs[(self.epoch + 1) & 1]

    def part_ptrs(self, epoch):
        """Device addresses of every rank's partial of step ``epoch``, rank order."""
        return [p + (epoch & 1) * self.slot_bytes for p in self.buf_ptrs]

    def __call__(self, residual, w, eps=1e-5, y=None, h=None, stream=None):
        """(y, h): h = sum over ranks of their partials of this step + residual, y =
        RmsNorm(h) * w; bit-identical on every rank."""
        if tuple(residual.shape) != self.shape:
            raise ValueError("residual must have the partial's shape")
        self.epoch += 1
        y = torch.empty_like(residual) if y is None else y
        h = torch.empty_like(residual) if h is None else h
        self._lib["publish"](self.flag_ptrs, self.rank, self.epoch, stream)
        self._lib["reduce"](self.part_ptrs(self.epoch), residual, w, y, h, eps, self.flags,
                            self.epoch, stream=stream)
        return y, h

    def close(self):
        from . import ipc_close
        close = self._lib.get("close", ipc_close)
        for ptr, off in self._mapped:
            close(ptr, off)
        self._mapped = []

"""ZeRO-1 data-parallel step over NCCL: optimizer state sharded by whole tensors.

"Scaling FP8 training to trillion-token LLMs" trains its 7B model data-parallel
on 256 accelerators; this module is the B200 form of that step for the FP8-moment
AdamW.  Each rank holds the full params (fp32) and its own full gradients
(bf16).  One step is:

  1. reduce-scatter of the gradients (NCCL, sum), so each rank receives the
     summed gradients of the tensors it owns;
  2. the FP8-moment AdamW step (the CUDA kernels) on the owned tensors only,
     with the 1/world average folded into the kernel as its gradient
     multiplier (``loss_scale = world``: a constant kernel argument, no
     gradient pre-pass unless clipping or skip-on-non-finite is asked for);
  3. all-gather of the updated params (NCCL), in place: each rank's block of
     the flat param buffer is its input, so nothing is copied first.

The gradients are reduced in their own dtype, bf16, as NCCL sums the buffer
it is given: the step's input is the reduced bf16 gradient.

Tensors are assigned whole to ranks (largest first onto the least-loaded rank),
so a tensor's amax and scale never cross ranks.  For the collectives the flat
buffers are laid out rank block by rank block, each block padded to the same
length (NCCL's reduce-scatter/all-gather take equal parts).
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch
import torch.distributed as dist

from . import ranks

ALIGN = 64  # elements: every tensor view starts 256 B (fp32) / 128 B (bf16) aligned


class ShardLayout:
    """Where every tensor sits in the rank-blocked flat buffers."""

    def __init__(self, numels: List[int], world: int):
        self.numels = [int(n) for n in numels]
        self.world = world
        self.parts = ranks.partition_by_numel(self.numels, world)
        self.owner = [0] * len(numels)
        self.offset = [0] * len(numels)  # element offset inside the owner's block
        sizes = []
        for r, part in enumerate(self.parts):
            off = 0
            for i in part:
                self.owner[i] = r
                self.offset[i] = off
                off += (self.numels[i] + ALIGN - 1) // ALIGN * ALIGN
            sizes.append(off)
        self.block = max(max(sizes), ALIGN)  # padded block length, equal for every rank
        self.total = self.block * world

    def flat_index(self, i: int) -> int:
        """Start of tensor i in the flat (all ranks) buffer."""
        return self.owner[i] * self.block + self.offset[i]

    def views(self, flat: torch.Tensor) -> List[torch.Tensor]:
        return [flat[self.flat_index(i):self.flat_index(i) + n] for i, n in enumerate(self.numels)]

    def block_views(self, block: torch.Tensor, rank: int) -> List[torch.Tensor]:
        """Views of rank `rank`'s own tensors inside its block buffer."""
        return [block[self.offset[i]:self.offset[i] + self.numels[i]] for i in self.parts[rank]]


class TorchCollectives:
    """Reduce-scatter (sum) and all-gather through torch.distributed on the
    tensors' own device: NCCL for CUDA tensors."""

    def __init__(self, group=None):
        self.group = group

    def reduce_scatter(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        dist.reduce_scatter_tensor(out, inp, op=dist.ReduceOp.SUM, group=self.group)

    def all_gather(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        dist.all_gather_into_tensor(out, inp, group=self.group)


class HostCollectives(TorchCollectives):
    """The same collectives through host copies, for a process group without
    device collectives (gloo): device -> host, the collective on the host
    buffers, host -> device."""

    def reduce_scatter(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        h_out = torch.empty(out.shape, dtype=out.dtype)
        dist.reduce_scatter_tensor(h_out, inp.cpu(), op=dist.ReduceOp.SUM, group=self.group)
        out.copy_(h_out)

    def all_gather(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        h_out = torch.empty(out.shape, dtype=out.dtype)
        dist.all_gather_into_tensor(h_out, inp.cpu(), group=self.group)
        out.copy_(h_out)


class ZeroFP8AdamW:
    """ZeRO-1 FP8-moment AdamW.  ``params`` (fp32) and ``grads`` (bf16) are
    the rank-blocked flat buffers of a ShardLayout (``layout.views`` gives the
    per-tensor views a model would use).  ``make_local(p_views, g_views,
    **opt_kw)`` builds the optimizer of the owned shard (by default the CUDA
    FP8AdamW); besides the caller's options it receives ``sr_tensor_ids``,
    the owned tensors' indices in the whole model, which key their
    stochastic-rounding draws.  ``collectives``: TorchCollectives (the
    default: NCCL on CUDA tensors) or HostCollectives."""

    def __init__(self, layout: ShardLayout, params: torch.Tensor, grads: torch.Tensor, *,
                 group=None, make_local: Optional[Callable] = None, collectives=None, **opt_kw):
        self.layout = layout
        self.group = group
        self.comm = collectives if collectives is not None else TorchCollectives(group)
        self.world = layout.world
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        if params.numel() != layout.total or grads.numel() != layout.total:
            raise ValueError("flat buffers must have the layout's padded length")
        self.params, self.grads = params, grads
        b = layout.block
        r = self.rank
        self.p_block = params[r * b:(r + 1) * b]          # this rank's params (a view)
        self.g_block = torch.zeros(b, dtype=grads.dtype, device=grads.device)  # reduced grads
        p_views = layout.block_views(self.p_block, r)
        g_views = layout.block_views(self.g_block, r)
        if make_local is None:
            from .optim import FP8AdamW

            make_local = lambda p, g, **kw: FP8AdamW(p, g, **kw)  # noqa: E731
        # each owned tensor keeps its index in the whole model as its word in
        # the stochastic-rounding counter, so a shard draws the bits a single
        # optimizer over every tensor would
        opt_kw.setdefault("sr_tensor_ids", list(layout.parts[r]))
        self.local = make_local(p_views, g_views, **opt_kw) if p_views else None

    def step(self, **step_kw) -> None:
        # 1. summed gradients of the owned tensors
        if self.world > 1:
            self.comm.reduce_scatter(self.g_block, self.grads)
        else:
            self.g_block.copy_(self.grads)
        # 2. the step on the shard; the average over ranks rides on the
        #    kernel's gradient multiplier
        if self.local is not None:
            ls = float(step_kw.pop("loss_scale", 1.0)) * self.world
            self.local.step(loss_scale=ls, **step_kw)
        # 3. every rank gets every updated param; the input is this rank's
        #    block of the output (NCCL's in-place form)
        if self.world > 1:
            self.comm.all_gather(self.params, self.p_block)

    def close(self) -> None:
        if self.local is not None and hasattr(self.local, "close"):
            self.local.close()

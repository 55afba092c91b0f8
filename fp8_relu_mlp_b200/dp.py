"""Data-parallel exchange for the block across ranks (torch.distributed).

The block shards by tokens: every rank holds W1/W2 and runs its own M tokens.
A training step then needs two exchanges:

* the partial-amax tensor is all-reduced with MAX before the scale update, so
  that every rank derives the same delayed scale s_{t+1} ("A Retrospective on
  Our World Records", Main Track: the scale comes from the amax of step t-1;
  with data parallelism that amax is over all ranks' tokens);
* dW1 and dW2 are all-reduced (summed, optionally averaged), the gradient
  exchange of data-parallel training that the pages' 8-GPU runs do in their
  optimizer -- or reduce-scattered, so that each rank keeps the reduced rows
  of its own shard (h/N rows of each), for an optimizer whose state is
  sharded by rank; that moves half the bytes of an all-reduce.

The dW exchange is issued on a side stream as soon as the dW GEMM is done and
overlaps the dX GEMM, which does not depend on it.  These helpers only move
data through torch.distributed (NCCL on GPUs; gloo works for CPU tensors).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _abi as A


def allreduce_amax(partial_amax: torch.Tensor, group=None, async_op: bool = False):
    """MAX over ranks of the partial-amax tensor, in place."""
    return dist.all_reduce(partial_amax, op=dist.ReduceOp.MAX, group=group, async_op=async_op)


def allreduce_grads(dW1: torch.Tensor, dW2: torch.Tensor, group=None, average: bool = True):
    """SUM (or mean) over ranks of dW1 and dW2, in place."""
    world = dist.get_world_size(group)
    for t in (dW1, dW2):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        if average and world > 1:
            t.div_(world)


def reduce_scatter_grads(dW1: torch.Tensor, dW2: torch.Tensor, shard1: torch.Tensor, shard2: torch.Tensor,
                         group=None, average: bool = True):
    """SUM (or mean) over ranks of dW1 and dW2 [h,d], of which this rank keeps
    rows [r h/N, (r+1) h/N) in shard1 / shard2 [h/N, d]."""
    world = dist.get_world_size(group)
    for full, part in ((dW1, shard1), (dW2, shard2)):
        if full.shape[0] % world != 0 or part.shape[0] * world != full.shape[0]:
            raise ValueError("h must be a multiple of the world size, shards of h/N rows")
        dist.reduce_scatter_tensor(part, full, op=dist.ReduceOp.SUM, group=group)
        if average and world > 1:
            part.div_(world)


def max_over_ranks(x: float, device=None, group=None) -> float:
    """The maximum of a host scalar over all ranks (e.g. a timing)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


class DataParallelStep:
    """One data-parallel training step of an MLPBlock on this rank's tokens.

    Order on the main stream: forward (up-projection, FP8 down-projection),
    dPre, dW; the side stream then all-reduces the partial amax and dW while
    the main stream runs dX; the main stream waits for the side stream, then
    updates the delayed scale from the all-reduced amax and refreshes the W2
    cache (after the caller's optimizer update, in a real training loop)."""

    def __init__(self, blk, group=None, average: bool = True, shard_grads: bool = False):
        """``shard_grads``: reduce-scatter dW1/dW2 into ``self.dW1_shard`` /
        ``self.dW2_shard`` ([h/N, d], this rank's rows) instead of
        all-reducing the full tensors."""
        self.blk = blk
        self.group = group
        self.average = average
        self.side = torch.cuda.Stream(blk.device)
        self.shard_grads = shard_grads
        if shard_grads:
            n = dist.get_world_size(group)
            if blk.h % n != 0:
                raise ValueError("h must be a multiple of the world size to shard the gradients")
            self.dW1_shard = torch.empty(blk.h // n, blk.d, dtype=torch.float32, device=blk.device)
            self.dW2_shard = torch.empty_like(self.dW1_shard)

    def __call__(self, refresh_w2: bool = True, mark=None):
        """``mark(i)``, if given, is called on the main stream at 0 (start),
        1 / 2 (around the dW GEMM) and 3 (end of the step)."""
        b = self.blk
        M, d, h = b.M, b.d, b.h
        mark = mark or (lambda i: None)
        main = torch.cuda.current_stream(b.device)
        mark(0)
        A.fp8mlp_up_proj_fused(M, d, h, b.x, b.W1, b.state, b.post, b.post_fp8, b.partial_amax)
        A.fp8mlp_down_proj_fp8(M, d, h, b.post_fp8, b.W2q_t, b.w2_scale_inv, b.state, b.out)
        # dPre does not read the down-projection's output (it may overlap its tail)
        A.fp8mlp_bwd_dpre(M, d, h, b.dOut, b.W2, b.post, b.dPre, A.LAUNCH_OVERLAP_PREVIOUS)
        mark(1)
        A.fp8mlp_bwd_dw(M, d, h, b.x, b.dPre, b.post, b.dOut, b.dW1, b.dW2)
        mark(2)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            allreduce_amax(b.partial_amax, self.group)
            if self.shard_grads:
                reduce_scatter_grads(b.dW1, b.dW2, self.dW1_shard, self.dW2_shard, self.group, self.average)
            else:
                allreduce_grads(b.dW1, b.dW2, self.group, self.average)
        A.fp8mlp_bwd_dx(M, d, h, b.dPre, b.W1, b.dX)
        main.wait_stream(self.side)
        b.update_scale()
        if refresh_w2:
            b.refresh_w2_cache()
        mark(3)

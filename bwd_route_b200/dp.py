"""Data-parallel training of the gate: one process per GPU, each on its own
shard of the batch, with torch.distributed (NCCL between GPUs) carrying the one
exchange the step has.

Every rank runs the single-GPU step on its [B, N_H] shard with the library's
kernels. The method's per-token terms are independent (routing, forward, d_x,
the straight-through backward of each token), so only two results cross ranks:

- dW and db are sums over tokens of per-token outer products and rows; the full
  batch's dW and db are therefore the sum of the shards'. One all-reduce (sum)
  over the gate's flat gradient buffer gives them to every rank.
- the expert counts are summed in int32, which is exact and independent of the
  order of the sum, so every rank folds the same global usage into ent_ema and
  computes the same lambda_eff bit for bit (the controller state stays
  identical across replicas without broadcasting it).

The load-balance loss stays per shard: each rank's aux term and its logit
gradient are those of its own tokens, as on one GPU.

The order of the cross-rank fp32 sum is the collective library's; within a
rank every sum has a fixed order. Collectives are issued on torch's current
stream, so the gate's kernels must run on that stream as well.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world_tokens(T: int, device, group=None) -> int:
    """The global token count of a step; every rank must hold a shard of the
    same size T (checked with one small all-reduce, on every rank)."""
    t = torch.tensor([T, -T], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    hi, lo = int(t[0]), -int(t[1])
    if hi != lo:
        raise ValueError(f"data-parallel shards differ in size: {lo} to {hi} tokens per rank")
    total = T * dist.get_world_size(group)
    if total >= 2 ** 31:
        raise ValueError(f"{total} tokens per step overflow the int32 expert counts")
    return total


def allreduce_gradients(grads: torch.Tensor, group=None) -> torch.Tensor:
    """Sums the flat [dW | db] buffer over ranks, in place."""
    if grads.dtype != torch.float32 or not grads.is_contiguous():
        raise ValueError("grads must be one contiguous float32 buffer")
    dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=group)
    return grads


def global_counts(counts: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """out = the expert counts summed over ranks (int32, exact). counts, the
    rank's own routing result, is left as it is."""
    if counts.dtype != torch.int32 or out.dtype != torch.int32 or out.shape != counts.shape:
        raise ValueError("counts and out must be int32 tensors of the same shape")
    out.copy_(counts)
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out

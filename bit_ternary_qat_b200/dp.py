"""Data-parallel plumbing of the BitLinear step (host side).

Tokens are sharded across ranks; every rank quantises the same latent weight (the
fixed-order reduction makes gamma and the codes bit-identical on every rank), runs the
forward and backward on its own tokens, and the weight gradient -- a sum over tokens --
is summed over ranks.  Nothing else is exchanged.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(T: int, world: int, rank: int):
    """[start, end) of rank's contiguous token shard of T tokens (sizes differ by <= 1)."""
    base, rem = divmod(T, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def allreduce_weight_grad(dW: torch.Tensor, group=None) -> torch.Tensor:
    """Sum dW over ranks in place (NCCL on GPU, gloo on CPU)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
    return dW


def check_replicated(t: torch.Tensor, group=None) -> bool:
    """True when t is bit-identical on every rank (used for gamma and the codes)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return True
    ws = dist.get_world_size(group)
    gathered = [torch.empty_like(t) for _ in range(ws)]
    dist.all_gather(gathered, t.contiguous(), group=group)
    return all(torch.equal(gathered[0], g) for g in gathered[1:])

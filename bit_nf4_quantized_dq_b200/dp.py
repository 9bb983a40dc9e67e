"""Data parallelism over tokens for the QLoRA linear.

Each rank holds the same frozen NF4 codes and the same adapters and processes its own slice
of the tokens.  The forward and dX need nothing from other ranks; dA = u^T x and dB = dY^T t
are sums over tokens, so the full-batch gradients are the sums of the per-rank gradients.
That sum is the one exchange step: an all-reduce of dA and dB per linear (NCCL over NVLink on
GPUs; gloo works for host tensors).
"""

from __future__ import annotations

from typing import Iterable, Optional, Tuple

import torch
import torch.distributed as dist


def token_shard(total_tokens: int, rank: int, world: int) -> Tuple[int, int]:
    """[start, end) of this rank's tokens: contiguous, sizes differing by at most one."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank / world")
    base, extra = divmod(total_tokens, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(grads: Iterable[torch.Tensor], group: Optional[dist.ProcessGroup] = None,
                            average: bool = False) -> None:
    """Sum (or average) the adapter gradients across the data-parallel group, in place.

    bf16 gradients are reduced in fp32 and written back, so the sum is not rounded to bf16 at
    every hop of the collective."""
    world = dist.get_world_size(group)
    for g in grads:
        if g.dtype == torch.bfloat16:
            acc = g.float()
            dist.all_reduce(acc, group=group)
            if average:
                acc.div_(world)
            g.copy_(acc)
        else:
            dist.all_reduce(g, group=group)
            if average:
                g.div_(world)

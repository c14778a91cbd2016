"""Replica data parallelism for the MoE layer: host-side helpers.

The layer is independent per token, so several GPUs run it as replicas: one
process per GPU, each with a full copy of the weights and its own batch of
tokens.  No tensor crosses GPUs; the process group is used only to line the
ranks up (barrier) and to take the slowest rank's time.  Throughput is weak
scaling: every rank processes a full batch, so the job's tokens grow with
the number of ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def replica_token_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s token batch (rank 0 uses the workload's own seed)."""
    return seed if rank == 0 else seed + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """The largest value of `x` over all ranks (x itself without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(tokens_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Tokens per second of the whole job: all ranks' tokens over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return tokens_per_rank * steps * world / (max_ms / 1e3)

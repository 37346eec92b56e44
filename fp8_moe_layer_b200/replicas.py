"""Data-parallel replicas of the layer: one process per GPU, each with its own batch of tokens
and its own copy of the experts. The layer has no exchange step, so the only collectives are the
benchmark's bookkeeping (a barrier and the max over ranks of the device time)."""
from __future__ import annotations

import os
from typing import Sequence

import torch
import torch.distributed as dist


def rank_env():
    """(rank, world size, local rank) from the torchrun environment (1 process if absent)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own batch: the seed of rank r is base + r."""
    return int(base_seed) + int(rank)


def max_over_ranks(values: Sequence[float], device=None) -> list:
    """Elementwise maximum of per-rank timings (the slowest replica sets the step time)."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's device time."""
    return tokens_per_rank * world / (max_ms * 1e-3)

"""Replica bookkeeping for multi-GPU runs.

The decode path shards with no exchange: sequences, KV heads and layers are
independent. A run on N GPUs is N independent replicas (one process per GPU);
the only cross-rank traffic is the timing reduction below, done on the host
side of torch.distributed (nccl on GPUs, gloo on CPU).
"""

from __future__ import annotations

import os


def world():
    """(rank, world_size, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def _reduce(value: float, op: str) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def reduce_max(value: float) -> float:
    return _reduce(value, "max")


def reduce_sum(value: float) -> float:
    return _reduce(value, "sum")


def aggregate(units: float, elapsed_ms: float):
    """Whole-job throughput of independent replicas: units summed over ranks,
    divided by the slowest rank's time. Returns (total_units, max_ms, units_per_s)."""
    total = reduce_sum(units)
    slowest = reduce_max(elapsed_ms)
    return total, slowest, (total / (slowest / 1e3) if slowest > 0 else 0.0)


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()

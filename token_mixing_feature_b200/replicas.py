"""Data-parallel replicas: each rank runs the whole forward pass on its own
batch (samples are independent, so there is no exchange step); the job's
throughput is all ranks' samples over the slowest rank's time.

Works with any torch.distributed backend (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import Optional

import torch


def max_over_ranks(x: float, device: Optional[torch.device] = None) -> float:
    """All-reduce MAX of one float across the default process group (identity
    when torch.distributed is not initialised)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(samples_per_rank: int, steps: int, elapsed_ms_this_rank: float, world: int,
                   device: Optional[torch.device] = None) -> dict:
    """Whole-job samples/s: world * samples_per_rank * steps over the max time."""
    ms = max_over_ranks(elapsed_ms_this_rank, device)
    return {"elapsed_ms": ms, "samples": samples_per_rank * steps * world,
            "samples_per_s": samples_per_rank * steps * world / (ms / 1e3), "ms_per_step": ms / steps}

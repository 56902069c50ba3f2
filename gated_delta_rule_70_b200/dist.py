"""Multi-process plumbing of the benchmark: one process per GPU, each with its own batch
(weak scaling: the (sequence, head) units are independent, so there is no data-path
collective).  Only the timing is combined across ranks.  Nothing here touches CUDA
unless asked to (a CUDA device for the NCCL backend), so the same logic runs under
gloo on CPU.
"""

from __future__ import annotations

from typing import List, Optional, Sequence


def world_info(env) -> tuple:
    """(rank, world size, local rank) from a torchrun-style environment mapping."""
    return int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")), int(env.get("LOCAL_RANK", "0"))


def max_over_ranks(values: Sequence[float], device=None) -> List[float]:
    """Element-wise maximum of `values` over every rank of the default process group
    (every rank gets the result); the values themselves when there is no group."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu().tolist()]


def whole_job_rate(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Units per second of the whole job when each of `world` ranks processed
    `units_per_rank` per step and the slowest rank took `ms_per_step`."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def report_rank(rank: int) -> Optional[bool]:
    """Only rank 0 prints the benchmark line."""
    return rank == 0

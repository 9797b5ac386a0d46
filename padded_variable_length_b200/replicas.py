"""Host-side bookkeeping of a multi-GPU run of independent replicas.

The attention of one batch has no exchange step (every (batch entry, head) pair is
independent), so N GPUs run N independent replicas, one batch each.  Timing is taken on the
device per rank and combined as the maximum over ranks; the job's throughput counts the
work of all ranks.  The functions here hold that arithmetic and the one collective it
needs, so that it can be exercised on CPU ranks (gloo) as well as on NCCL ranks."""
from typing import Optional

import torch


def max_over_ranks(ms: float, device: Optional[torch.device] = None) -> float:
    """The largest of the ranks' times (every rank gets it); `ms` itself on one process."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(ms)
    if torch.distributed.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_step: float, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: the work of all `world` replicas over the slowest rank's time."""
    if max_ms <= 0.0:
        raise ValueError("time must be positive")
    return world * flops_per_step * steps / (max_ms / 1e3) / 1e12


def replica_seed(seed: int, rank: int) -> int:
    """Each replica draws its own data; the lengths and sizes stay those of the workload."""
    return seed + 7919 * rank

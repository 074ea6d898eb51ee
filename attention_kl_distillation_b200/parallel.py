"""Multi-GPU plumbing for the attention-KL path (host side only).

The path shards with no data exchange: every (batch, head) pair is an
independent problem in both the forward and the backward (dK reduces only
within a head).  One process per GPU takes a contiguous range of the B*H heads
(or, for weak-scaling benchmarks, a whole replica of the workload); the only
collectives are optional reductions of host-side scalars: a loss or a timing
taken as the maximum over ranks.  They go through torch.distributed, so the
same code runs over NCCL on GPUs and over gloo on CPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def head_shard(BH: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, stop) range of the BH heads owned by `rank`; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(BH, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _reduce(x: float, op, device) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, device="cpu") -> float:
    """Maximum of a host scalar over all ranks (the job's time is its slowest rank's)."""
    return _reduce(x, dist.ReduceOp.MAX, device)


def sum_over_ranks(x: float, device="cpu") -> float:
    return _reduce(x, dist.ReduceOp.SUM, device)

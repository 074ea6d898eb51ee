"""Multi-GPU plumbing for the attention-KL path (host side only).

The path shards with no data exchange: every (batch, head) pair is an
independent problem in both the forward and the backward (dK reduces only
within a head).  One process per GPU takes a contiguous range of the B*H heads
(``shard_heads``) and calls the library on it as a problem with B = 1 and H =
the range's length; the per-rank results are reassembled, where a caller
wants them whole, with ``all_gather_heads``.  For weak-scaling benchmarks a
rank may instead run a whole replica of the workload.  The only collectives
are optional and outside the library: reassembly of per-row results, and
reductions of host-side scalars (a loss, or a timing taken as the maximum over
ranks).  They go through torch.distributed, so the same code runs over NCCL on
GPUs and over gloo on CPU.
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


def shard_heads(t: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """The rank's heads of a [B, H, ...] tensor as a contiguous [1, h, ...] tensor.

    The heads are numbered b*H + h (batch-major), the order the library's
    [B][H] layout uses, so a slice of them is itself a valid problem with B = 1."""
    if t.dim() < 3:
        raise ValueError("expected a [B, H, ...] tensor")
    B, H = t.shape[:2]
    a, b = head_shard(B * H, world, rank)
    return t.reshape(B * H, *t.shape[2:])[a:b].unsqueeze(0).contiguous()


def all_gather_heads(local: torch.Tensor, B: int, H: int) -> torch.Tensor:
    """Reassemble [1, h_r, ...] shards from every rank into the full [B, H, ...] tensor.

    Shards differ in length by at most one head, so each is padded to the
    longest before the all-gather and trimmed after it.  Without an initialised
    process group (or with one rank) the local tensor is the whole result."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        if local.shape[1] != B * H:
            raise ValueError("a single rank must hold every head")
        return local.reshape(B, H, *local.shape[2:])
    world, rank = dist.get_world_size(), dist.get_rank()
    a, b = head_shard(B * H, world, rank)
    if local.shape[:2] != (1, b - a):
        raise ValueError(f"rank {rank} holds {tuple(local.shape[:2])}, expected (1, {b - a})")
    rest = local.shape[2:]
    longest = -(-B * H // world)
    pad = torch.zeros((longest, *rest), dtype=local.dtype, device=local.device)
    pad[: b - a] = local[0]
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    full = torch.cat([parts[r][: head_shard(B * H, world, r)[1] - head_shard(B * H, world, r)[0]]
                      for r in range(world)])
    return full.reshape(B, H, *rest)


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

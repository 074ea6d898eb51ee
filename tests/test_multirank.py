"""Multi-rank host logic on CPU (gloo, world sizes 2 and 4): head sharding covers
every head exactly once, each rank slices its heads as the bench's head-sharded
mode does, per-rank results on their shards reassemble into the unsharded
result (no exchange is needed before that), and timings reduce to the maximum."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from attention_kl_distillation_b200.parallel import head_shard


@pytest.mark.parametrize("BH,world", [(32, 2), (7, 3), (1, 2), (5, 8)])
def test_head_shard_partitions(BH, world):
    seen = []
    for r in range(world):
        a, b = head_shard(BH, world, r)
        assert 0 <= a <= b <= BH
        seen.extend(range(a, b))
    assert seen == list(range(BH))
    sizes = [head_shard(BH, world, r)[1] - head_shard(BH, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    from pathlib import Path
    root = Path(__file__).resolve().parent.parent
    sys.path.insert(0, str(root))
    import torch
    import torch.distributed as dist

    from attention_kl_distillation_b200.inputs import Workload, bf16_bits, make_inputs
    from attention_kl_distillation_b200.parallel import (all_gather_heads, head_shard,
                                                         max_over_ranks, shard_heads,
                                                         sum_over_ranks)
    from oracle import oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("mr", 2, 3, 48, 64, 16, 16, True, "perturb", 0.5, False, 77)
        # the slicing a GPU rank does before its library calls (B = 1, H = its heads)
        shards = [shard_heads(t, world, rank) for t in make_inputs(w)]
        a, b = head_shard(w.BH, world, rank)
        assert all(x.shape[:2] == (1, b - a) and x.is_contiguous() for x in shards)
        orc = O.default()
        L, A, Bv = orc.fwd_all(*[bf16_bits(x).reshape(b - a, *x.shape[2:]) for x in shards],
                               causal=True, nthreads=1)
        local = torch.from_numpy(L).reshape(1, b - a, -1)
        full = all_gather_heads(local, w.B, w.H)
        out[rank] = (a, b, full.numpy())
        out[f"t{rank}"] = max_over_ranks(10.0 + rank)
        out[f"s{rank}"] = sum_over_ranks(float(L.sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_heads_reassemble_unsharded_result(world):
    """Each rank slices its heads, computes them alone (the oracle stands in for the
    library on CPU), and all_gather_heads rebuilds the [B, H, NQ] result on every
    rank.  Six heads over four ranks gives shards of two and one head."""
    from attention_kl_distillation_b200.inputs import Workload, bf16_bits, make_inputs
    from oracle import oracle as O
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    w = Workload("mr", 2, 3, 48, 64, 16, 16, True, "perturb", 0.5, False, 77)
    ins = [bf16_bits(t).reshape(w.BH, -1, t.shape[-1]) for t in make_inputs(w)]
    full, _, _ = O.default().fwd_all(*ins, causal=True, nthreads=2)
    full = full.reshape(w.B, w.H, -1)
    for r in range(world):
        a, b, got = out[r]
        assert got.shape == full.shape
        assert np.array_equal(got, full)        # same rows, same arithmetic: bit-identical
    assert all(out[f"t{r}"] == 10.0 + world - 1 for r in range(world))   # max over ranks
    for r in range(world):
        assert abs(out[f"s{r}"] - float(full.sum())) <= 1e-9 * max(1.0, abs(float(full.sum())))


def test_shard_heads_single_process():
    """Without a process group, one rank's shard is the whole problem."""
    import torch

    from attention_kl_distillation_b200.parallel import all_gather_heads, shard_heads
    t = torch.arange(2 * 3 * 4 * 5, dtype=torch.float32).reshape(2, 3, 4, 5)
    parts = [shard_heads(t, 4, r) for r in range(4)]
    assert [p.shape[1] for p in parts] == [2, 2, 1, 1]
    assert torch.equal(torch.cat(parts, dim=1).reshape(2, 3, 4, 5), t)
    assert torch.equal(all_gather_heads(shard_heads(t, 1, 0), 2, 3), t)

"""Multi-rank host logic on CPU (gloo, world size 2): head sharding covers every
head exactly once, per-rank oracle results on their shards reassemble the
unsharded result (no exchange is needed), and timings reduce to the maximum."""
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
    import torch.distributed as dist

    from attention_kl_distillation_b200.inputs import Workload, bf16_bits, make_inputs
    from attention_kl_distillation_b200.parallel import head_shard, max_over_ranks, sum_over_ranks
    from oracle import oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("mr", 1, 5, 48, 64, 16, 16, True, "perturb", 0.5, False, 77)
        ins = [bf16_bits(t).reshape(w.BH, -1, t.shape[-1]) for t in make_inputs(w)]
        a, b = head_shard(w.BH, world, rank)
        orc = O.default()
        L, _, _ = orc.fwd_all(*[x[a:b] for x in ins], causal=True, nthreads=1)
        out[rank] = (a, b, L)
        t = max_over_ranks(10.0 + rank)
        s = sum_over_ranks(float(L.sum()))
        out[f"t{rank}"] = t
        out[f"s{rank}"] = s
    finally:
        dist.destroy_process_group()


def test_sharded_heads_reassemble_unsharded_result():
    from attention_kl_distillation_b200.inputs import Workload, bf16_bits, make_inputs
    from oracle import oracle as O
    world = 2
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
    w = Workload("mr", 1, 5, 48, 64, 16, 16, True, "perturb", 0.5, False, 77)
    ins = [bf16_bits(t).reshape(w.BH, -1, t.shape[-1]) for t in make_inputs(w)]
    full, _, _ = O.default().fwd_all(*ins, causal=True, nthreads=2)
    got = np.zeros_like(full)
    for r in range(world):
        a, b, L = out[r]
        got[a:b] = L
    assert np.array_equal(got, full)            # same rows, same arithmetic: bit-identical
    assert out["t0"] == out["t1"] == 11.0        # max over ranks
    assert abs(out["s0"] - float(full.sum())) <= 1e-9 * max(1.0, abs(float(full.sum())))

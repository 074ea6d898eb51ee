"""GPU parity of the forward (streamkl_fwd through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gpu_common import (all_rows, check_fwd, cuda_inputs, gpu_fwd, oracle_bits, workload)

pytestmark = pytest.mark.gpu

EDGE = [  # B, H, NQ, NK, d1, d2, causal
    (1, 1, 1, 1, 64, 64, False),
    (1, 1, 1, 1, 128, 128, True),
    (1, 2, 2, 2, 128, 128, True),
    (1, 1, 127, 127, 64, 64, True),
    (1, 1, 128, 128, 128, 128, True),
    (1, 1, 129, 129, 128, 64, True),
    (1, 2, 200, 200, 64, 128, False),
    (2, 1, 200, 333, 128, 128, False),
    (1, 1, 100, 300, 128, 128, True),
    (1, 1, 300, 100, 64, 64, False),
    (1, 3, 257, 513, 128, 64, True),
    (1, 1, 1, 1000, 128, 128, False),
    (1, 1, 5, 1000, 64, 64, True),
    (3, 50, 130, 130, 64, 64, True),     # more work units than SMs
]


@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "B{}H{}Q{}K{}d{}-{}{}".format(*s[:6], "c" if s[6] else ""))
def test_fwd_edge_shapes(orc, shape):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(*shape)
    ins = make_inputs(w)
    gpu = gpu_fwd(cuda_inputs(ins), w.causal)
    rows = all_rows(w.BH, w.NQ)
    if len(rows) > 4000:
        rows = rows[np.random.default_rng(0).choice(len(rows), 4000, replace=False)]
    ora = orc.fwd_rows(*oracle_bits(ins), rows, causal=w.causal)
    check_fwd(gpu, ora, rows, w.name)


def test_fwd_tiny_workload(orc):
    """The tiny non-causal workload (B1 H2 N256 d64), every row."""
    from attention_kl_distillation_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["tiny"]
    ins = make_inputs(w)
    gpu = gpu_fwd(cuda_inputs(ins), w.causal)
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, causal=w.causal), rows, w.name)


def test_fwd_explicit_scales(orc):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 150, 260, 128, 64, True)
    ins = make_inputs(w)
    gpu = gpu_fwd(cuda_inputs(ins), True, s1=0.31, s2=0.05)
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, causal=True, s1=0.31, s2=0.05), rows)


def test_fwd_large_logits(orc):
    """Logits spanning hundreds of nats: online rescaling must stay finite and exact enough."""
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 256, 384, 64, 64, False)
    ins = [t * 4 for t in make_inputs(w)]
    gpu = gpu_fwd(cuda_inputs(ins), False, s1=1.0, s2=0.7)
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, s1=1.0, s2=0.7), rows)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fwd_identical_inputs_give_exact_zero(causal, d):
    """S1 == S2 bit for bit, so acc == 0 and LSE1 == LSE2: L must be exactly 0."""
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 333, 333, d, d, causal)
    Q, K, _, _ = cuda_inputs(make_inputs(w))
    L, A, B = gpu_fwd([Q, K, Q, K], causal)
    assert np.all(L == 0.0)
    assert np.array_equal(A, B)


def test_fwd_key_permutation_invariance():
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 200, 640, 128, 128, False)
    Q1, K1, Q2, K2 = cuda_inputs(make_inputs(w))
    perm = torch.randperm(640, generator=torch.Generator().manual_seed(3)).cuda()
    L, A, B = gpu_fwd([Q1, K1, Q2, K2], False)
    Lp, Ap, Bp = gpu_fwd([Q1, K1[:, :, perm].contiguous(), Q2, K2[:, :, perm].contiguous()], False)
    assert np.abs(L - Lp).max() <= 1e-5
    assert np.abs(A - Ap).max() <= 1e-5 and np.abs(B - Bp).max() <= 1e-5


@pytest.mark.parametrize("name", ["causal4k", "sparse_student", "long64k", "fwdbwd16k"])
def test_fwd_full_size_sampled(orc, name):
    """Full-size workloads, >= 256 seeded rows per head plus the tile/causal edge rows."""
    from attention_kl_distillation_b200.inputs import WORKLOADS, make_inputs, sample_rows
    w = WORKLOADS[name]
    ins = make_inputs(w)
    dev = cuda_inputs(ins)
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    free0, _ = torch.cuda.mem_get_info()
    gpu = gpu_fwd(dev, w.causal)
    free1, _ = torch.cuda.mem_get_info()
    peak_extra = torch.cuda.max_memory_allocated() - base
    out_bytes = 3 * 4 * w.BH * w.NQ
    # nothing materialised: extra memory is the three fp32 row vectors (plus allocator rounding)
    assert peak_extra <= out_bytes + (8 << 20), peak_extra
    assert free0 - free1 <= out_bytes + (64 << 20)
    rows = sample_rows(w.BH, w.NQ, 256, seed=w.seed)
    ora = orc.fwd_rows(*oracle_bits(ins), rows, causal=w.causal)
    check_fwd(gpu, ora, rows, name)

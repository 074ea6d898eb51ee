"""GPU parity of the transposed forward (few query rows: keys on the UMMA M axis,
the ETAP page's S^T = K Q^T) against the fp64 oracle, and its agreement with the
128-row tile kernel, which serves the same rows when they are part of a larger
query set."""
import numpy as np
import pytest
import torch

from gpu_common import all_rows, check_fwd, cuda_inputs, gpu_fwd, oracle_bits, workload

pytestmark = pytest.mark.gpu

SHAPES = [  # B, H, NQ, NK, d1, d2, causal -- NQ <= 32 takes the transposed kernel
    (1, 1, 1, 1, 128, 128, False),
    (1, 2, 1, 129, 64, 64, True),
    (1, 1, 3, 3, 128, 64, True),
    (2, 1, 16, 16, 64, 128, True),
    (1, 3, 16, 700, 128, 128, False),
    (1, 1, 17, 128, 128, 128, True),
    (1, 2, 31, 257, 64, 64, True),
    (1, 1, 32, 32, 128, 128, True),
    (2, 2, 32, 1000, 128, 64, False),
    (1, 1, 33, 300, 128, 128, True),      # first size on the 128-row tile kernel
    (5, 40, 8, 384, 64, 64, True),        # more work units than SMs
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}Q{}K{}d{}-{}{}".format(*s[:6], "c" if s[6] else ""))
def test_transposed_matches_oracle(orc, shape):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(*shape)
    ins = make_inputs(w)
    gpu = gpu_fwd(cuda_inputs(ins), w.causal)
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, causal=w.causal), rows, w.name)


@pytest.mark.parametrize("nq", [1, 9, 16, 25, 32])
@pytest.mark.parametrize("dims", [(128, 128), (64, 128)])
def test_transposed_agrees_with_row_tile_kernel(nq, dims):
    """Without the causal mask a row's result does not depend on the other rows:
    the first nq rows computed alone (transposed kernel) and as part of 200 rows
    (128-row tile kernel) agree to fp32 rounding."""
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 3, 200, 900, dims[0], dims[1], False)
    Q1, K1, Q2, K2 = cuda_inputs(make_inputs(w))
    big = gpu_fwd([Q1, K1, Q2, K2], False)
    small = gpu_fwd([Q1[:, :, :nq].contiguous(), K1, Q2[:, :, :nq].contiguous(), K2], False)
    for b, s in zip(big, small):
        assert np.abs(b[:, :nq] - s).max() <= 2e-5 * max(1.0, np.abs(b[:, :nq]).max())


@pytest.mark.parametrize("causal", [False, True])
def test_transposed_identical_inputs_give_exact_zero(causal):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 20, 333, 128, 128, causal)
    Q, K, _, _ = cuda_inputs(make_inputs(w))
    L, A, B = gpu_fwd([Q, K, Q, K], causal)
    assert np.all(L == 0.0)
    assert np.array_equal(A, B)


def test_transposed_large_logits(orc):
    """Logits spanning hundreds of nats: the per-element rescaling of the
    per-lane states and the lane merge must stay finite and accurate."""
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 24, 500, 64, 64, False)
    ins = [t * 4 for t in make_inputs(w)]
    gpu = gpu_fwd(cuda_inputs(ins), False, s1=1.0, s2=0.7)
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, s1=1.0, s2=0.7), rows)


@pytest.mark.parametrize("nsplit", [2, 5, 64])
@pytest.mark.parametrize("shape", [(1, 3, 17, 3000, 128, 64, True), (2, 2, 32, 2000, 64, 64, False)],
                         ids=["Q17c", "Q32"])
def test_transposed_splitk(orc, shape, nsplit):
    from attention_kl_distillation_b200 import fwd_splitk, query_device_status
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(*shape)
    ins = make_inputs(w)
    dev = cuda_inputs(ins)
    L, A, B = fwd_splitk(*dev, causal=w.causal, nsplit=nsplit)
    torch.cuda.synchronize()
    assert query_device_status() == 0
    gpu = tuple(t.reshape(w.BH, -1).cpu().numpy().astype(np.float64) for t in (L, A, B))
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, causal=w.causal), rows, f"{w.name} split {nsplit}")


def test_unit_count_overflow_is_refused_before_launch():
    """2^30 heads split in two make 2^31 work units, more than the kernels count
    in int: the call returns EINVAL without launching (the pointers are never
    dereferenced, so placeholders serve)."""
    import ctypes
    from attention_kl_distillation_b200 import binding as B
    lib = B.lib()
    prob = B.problem(1, 1 << 30, 8, 512, 64, 64, False)
    v = ctypes.c_void_p
    ptrs = [v(1 << 20) for _ in range(7)]
    before = lib.streamkl_launch_count()
    st = lib.streamkl_fwd_splitk(ctypes.byref(prob), *ptrs, 2, v(1 << 20), ctypes.c_size_t(1 << 62), v(0))
    assert st == B.EINVAL
    assert lib.streamkl_launch_count() == before


@pytest.mark.parametrize("nq", [1, 20])
def test_transposed_unsplit_long_keys(orc, nq):
    """The unsplit transposed forward on the 64K key set (B1 H32 NK=65536 causal):
    one CTA streams all 512 key tiles of a head, every query row checked."""
    from attention_kl_distillation_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["long64k"].with_(NQ=nq)
    ins = make_inputs(w)
    gpu = gpu_fwd(cuda_inputs(ins), True)
    rows = all_rows(w.BH, w.NQ)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, causal=True), rows, f"long keys NQ={nq}")

"""GPU parity of the backward (streamkl_bwd through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gpu_common import TOL_GRAD, check_fwd, cuda_inputs, oracle_bits, rel_frobenius, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["fused_key_tiles", "fused_query_tiles", "fused_sides", "split"])
def bwd_algo(request):
    """Every backward test runs with each algorithm of streamkl_bwd: the fused kernel
    with key-tile units, with query-tile units, with query-tile units and one gradient
    side per pass, and the two split passes."""
    from attention_kl_distillation_b200 import set_bwd_algorithm
    set_bwd_algorithm(request.param)
    yield request.param
    set_bwd_algorithm("auto")

SHAPES = [  # B, H, NQ, NK, d1, d2, causal
    (1, 1, 64, 128, 64, 64, False),
    (1, 2, 130, 200, 128, 128, True),
    (1, 1, 100, 300, 128, 64, True),
    (1, 1, 257, 257, 64, 128, False),
    (2, 1, 1, 1, 128, 128, True),
    (1, 1, 200, 100, 64, 64, False),
    (1, 2, 384, 384, 128, 128, True),
    (3, 2, 70, 333, 64, 64, True),
]


def run_bwd(dev, dL, causal, need=(True, True, True, True), s1=None, s2=None, saved=False):
    """Forward then backward through the C ABI.  With saved=True also returns the
    forward's L, LSE1, LSE2 ([BH, NQ] float64), the state the backward consumed."""
    from attention_kl_distillation_b200 import bwd, fwd, query_device_status
    L, A, B = fwd(*dev, causal=causal, s1=s1, s2=s2)
    grads = bwd(dL, *dev, L, A, B, causal=causal, s1=s1, s2=s2, need=need)
    torch.cuda.synchronize()
    assert query_device_status() == 0
    out = [g.float().cpu().numpy().astype(np.float64) if g is not None else None for g in grads]
    if saved:
        BH = L.shape[0] * L.shape[1]
        return out, tuple(t.reshape(BH, -1).cpu().numpy().astype(np.float64) for t in (L, A, B))
    return out


_FWDBWD_ORACLE = {}


def fwdbwd16k_oracle(orc, bits, kind, key, g):
    """Oracle results on the forward+backward workload, computed once per session:
    every backward algorithm is checked against the same rows and heads."""
    if (kind, key) not in _FWDBWD_ORACLE:
        if kind == "rows":
            rows = np.asarray(key, dtype=np.int64).reshape(-1, 2)
            _FWDBWD_ORACLE[(kind, key)] = orc.bwd_rows(*bits, rows, np.full(len(rows), g),
                                                       causal=True)
        else:
            _FWDBWD_ORACLE[(kind, key)] = orc.bwd_heads(*bits, list(key),
                                                        np.full((len(key), bits[0].shape[2]), g),
                                                        causal=True)
    return _FWDBWD_ORACLE[(kind, key)]


def oracle_heads(orc, ins, dL, causal, heads, s1=None, s2=None):
    B, H, NQ = dL.shape
    g = dL.reshape(B * H, NQ).cpu().numpy().astype(np.float64)[heads]
    return orc.bwd_heads(*oracle_bits(ins), heads, g, causal=causal, s1=s1, s2=s2)


def check_grads(gpu, ora, heads, names=("dQ1", "dK1", "dQ2", "dK2"), what=""):
    for n, gval in zip(("dQ1", "dK1", "dQ2", "dK2"), gpu):
        if n not in names:
            continue
        G = gval.reshape(-1, *gval.shape[2:])[heads]
        assert np.all(np.isfinite(G)), f"{what} {n} not finite"
        if np.linalg.norm(ora[n]) == 0.0:
            # e.g. a single visible key: the exact gradient vanishes; allow fp32 rounding residue
            assert np.abs(G).max() <= 1e-6, f"{what} {n}: expected 0, max |g| {np.abs(G).max():.2e}"
            continue
        err = rel_frobenius(G, ora[n])
        assert err <= TOL_GRAD, f"{what} {n}: relative Frobenius error {err:.3e}"


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}Q{}K{}d{}-{}{}".format(*s[:6], "c" if s[6] else ""))
def test_bwd_small_shapes(orc, shape):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(*shape)
    ins = make_inputs(w)
    dL = torch.randn((w.B, w.H, w.NQ), generator=torch.Generator().manual_seed(11))
    gpu = run_bwd(cuda_inputs(ins), dL.cuda(), w.causal)
    heads = list(range(w.BH))
    check_grads(gpu, oracle_heads(orc, ins, dL, w.causal, heads), heads, what=w.name)


@pytest.mark.parametrize("config", ["teacher_fixed", "student_fixed"])
def test_bwd_gradient_configurations(orc, config):
    """NULL outputs skip work: teacher fixed returns only dQ2/dK2, student fixed only dQ1/dK1."""
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 192, 256, 128, 128, True)
    ins = make_inputs(w)
    dL = torch.randn((w.B, w.H, w.NQ), generator=torch.Generator().manual_seed(12))
    need = (False, False, True, True) if config == "teacher_fixed" else (True, True, False, False)
    gpu = run_bwd(cuda_inputs(ins), dL.cuda(), True, need=need)
    assert [g is None for g in gpu] == [not x for x in need]
    names = [n for n, x in zip(("dQ1", "dK1", "dQ2", "dK2"), need) if x]
    check_grads(gpu, oracle_heads(orc, ins, dL, True, [0, 1]), [0, 1], names=names)


def test_bwd_single_output(orc):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 1, 150, 150, 64, 128, False)
    ins = make_inputs(w)
    dL = torch.randn((1, 1, 150), generator=torch.Generator().manual_seed(13))
    gpu = run_bwd(cuda_inputs(ins), dL.cuda(), False, need=(False, True, False, False))
    check_grads(gpu, oracle_heads(orc, ins, dL, False, [0]), [0], names=["dK1"])


@pytest.mark.parametrize("need", ["1000", "0100", "0010", "0001", "1100", "0011", "1001", "0110"])
@pytest.mark.parametrize("dims", [(128, 64), (64, 128)])
def test_bwd_one_sided_and_partial_outputs(orc, need, dims):
    """Every single output and both one-sided configurations, with teacher and
    student head dimensions that differ (the one-sided kernels keep a dQ
    accumulator of one side's width), ragged non-causal tiles."""
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 136, 200, dims[0], dims[1], False)
    ins = make_inputs(w)
    dL = torch.randn((w.B, w.H, w.NQ), generator=torch.Generator().manual_seed(15))
    nd = tuple(c == "1" for c in need)
    gpu = run_bwd(cuda_inputs(ins), dL.cuda(), False, need=nd)
    assert [g is None for g in gpu] == [not x for x in nd]
    names = [n for n, x in zip(("dQ1", "dK1", "dQ2", "dK2"), nd) if x]
    check_grads(gpu, oracle_heads(orc, ins, dL, False, [0, 1]), [0, 1], names=names)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_one_sided_matches_full_kernel_bitwise(bwd_algo, causal):
    """The gradient a fused kernel keeps on chip (dK with key-tile units, dQ with
    query-tile units) is accumulated in TMEM in a fixed order, and a one-sided
    kernel forms its dS with the same arithmetic as the two-sided one, so that
    gradient is the same to the bit (the other goes through fp32 atomics and is
    not compared)."""
    if not bwd_algo.startswith("fused"):
        pytest.skip("the specialised kernels are the fused path")
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 192, 320, 128, 128, causal)
    dev = cuda_inputs(make_inputs(w))
    dL = torch.randn((1, 2, w.NQ), device="cuda")
    full = run_bwd(dev, dL, causal)
    i1, i2 = (1, 3) if bwd_algo == "fused_key_tiles" else (0, 2)
    teacher = run_bwd(dev, dL, causal, need=tuple(k == i1 for k in range(4)))
    student = run_bwd(dev, dL, causal, need=tuple(k == i2 for k in range(4)))
    assert np.array_equal(teacher[i1], full[i1])
    assert np.array_equal(student[i2], full[i2])


def test_bwd_explicit_scales(orc):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 1, 128, 192, 128, 128, True)
    ins = make_inputs(w)
    dL = torch.randn((1, 1, 128), generator=torch.Generator().manual_seed(14))
    gpu = run_bwd(cuda_inputs(ins), dL.cuda(), True, s1=0.2, s2=0.11)
    check_grads(gpu, oracle_heads(orc, ins, dL, True, [0], s1=0.2, s2=0.11), [0])


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_identical_inputs_give_exact_zero(causal):
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 200, 200, 128, 128, causal)
    Q, K, _, _ = cuda_inputs(make_inputs(w))
    dL = torch.randn((1, 2, 200), device="cuda")
    for g in run_bwd([Q, K, Q, K], dL, causal):
        assert np.all(g == 0.0)


def test_autograd_wrapper_matches_direct_call():
    from attention_kl_distillation_b200 import bwd, fwd, streamkl
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 130, 260, 128, 64, True)
    Q1, K1, Q2, K2 = cuda_inputs(make_inputs(w))
    ins = [t.clone().requires_grad_(True) for t in (Q1, K1, Q2, K2)]
    L = streamkl(*ins, causal=True)
    (L * 0.5).sum().backward()
    L0, A, B = fwd(Q1, K1, Q2, K2, causal=True)
    dL = torch.full_like(L0, 0.5)
    ref = bwd(dL, Q1, K1, Q2, K2, L0, A, B, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(L.detach(), L0)
    for t, r in zip(ins, ref):
        err = ((t.grad.float() - r.float()).norm() / r.float().norm()).item()
        assert err <= 1e-2   # fp32 atomics: not bitwise reproducible


@pytest.mark.parametrize("frozen", ["teacher", "student"])
def test_autograd_frozen_side_runs_one_sided(frozen):
    """Distillation with a frozen side through the autograd wrapper: only the
    trainable side gets gradients, equal to a direct one-sided call."""
    from attention_kl_distillation_b200 import bwd, fwd, streamkl
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, 160, 300, 128, 128, True)
    Q1, K1, Q2, K2 = cuda_inputs(make_inputs(w))
    train = (False, False, True, True) if frozen == "teacher" else (True, True, False, False)
    ins = [t.clone().requires_grad_(r) for t, r in zip((Q1, K1, Q2, K2), train)]
    L = streamkl(*ins, causal=True)
    L.sum().backward()
    L0, A, B = fwd(Q1, K1, Q2, K2, causal=True)
    ref = bwd(torch.ones_like(L0), Q1, K1, Q2, K2, L0, A, B, causal=True, need=train)
    torch.cuda.synchronize()
    for t, r, n in zip(ins, ref, train):
        if not n:
            assert t.grad is None and r is None
            continue
        err = ((t.grad.float() - r.float()).norm() / r.float().norm()).item()
        assert err <= 1e-2   # fp32 atomics: not bitwise reproducible


def test_bwd_full_size_workload(orc):
    """Forward+backward workload (B1 H32 N16384 d128 causal, dL = 1/(B*H*NQ)):
    the forward's L, LSE1, LSE2 and dQ on >= 256 sampled rows of every head,
    dK1/dK2 in full on head 0 and one seeded head."""
    from attention_kl_distillation_b200.inputs import WORKLOADS, make_inputs, sample_rows
    w = WORKLOADS["fwdbwd16k"]
    ins = make_inputs(w)
    dev = cuda_inputs(ins)
    g = 1.0 / (w.B * w.H * w.NQ)
    dL = torch.full((w.B, w.H, w.NQ), g, device="cuda")
    (dQ1, dK1, dQ2, dK2), fwd_out = run_bwd(dev, dL, True, saved=True)
    bits = oracle_bits(ins)
    rows = sample_rows(w.BH, w.NQ, 256, seed=w.seed)
    oL, oA, oB, oq1, oq2 = fwdbwd16k_oracle(orc, bits, "rows", tuple(rows.ravel().tolist()), g)
    # the saved state the backward consumed: L, LSE1, LSE2 of the same rows
    check_fwd(fwd_out, (oL, oA, oB), rows, "fwdbwd16k forward")
    gq1 = dQ1.reshape(w.BH, w.NQ, -1)[rows[:, 0], rows[:, 1]]
    gq2 = dQ2.reshape(w.BH, w.NQ, -1)[rows[:, 0], rows[:, 1]]
    assert rel_frobenius(gq1, oq1) <= TOL_GRAD
    assert rel_frobenius(gq2, oq2) <= TOL_GRAD
    heads = [0, int(np.random.default_rng(w.seed).integers(1, w.BH))]
    o = fwdbwd16k_oracle(orc, bits, "heads", tuple(heads), g)
    for n, G in (("dK1", dK1), ("dK2", dK2)):
        err = rel_frobenius(G.reshape(w.BH, w.NK, -1)[heads], o[n])
        assert err <= TOL_GRAD, f"{n} {err:.3e}"
    # every row of those two heads: the forward's saved state against the oracle's
    hrows = np.stack(np.meshgrid(heads, np.arange(w.NQ), indexing="ij"), -1).reshape(-1, 2)
    check_fwd(fwd_out, (o["L"].ravel(), o["LSE1"].ravel(), o["LSE2"].ravel()), hrows,
              "fwdbwd16k forward, whole heads")


@pytest.mark.parametrize("side", ["student", "teacher"])
def test_bwd_full_size_one_sided(orc, bwd_algo, side):
    """The one-sided kernels on the forward+backward workload (B1 H32 N16384 d128
    causal): the student side alone (the page's configuration 1, standard
    distillation) or the teacher side alone; dQ on sampled rows of every head,
    dK in full on head 0 and one seeded head.  Every algorithm has instances
    specialised to one side."""
    from attention_kl_distillation_b200.inputs import WORKLOADS, make_inputs, sample_rows
    w = WORKLOADS["fwdbwd16k"]
    ins = make_inputs(w)
    dev = cuda_inputs(ins)
    g = 1.0 / (w.B * w.H * w.NQ)
    dL = torch.full((w.B, w.H, w.NQ), g, device="cuda")
    need = (False, False, True, True) if side == "student" else (True, True, False, False)
    out = run_bwd(dev, dL, True, need=need)
    dQ, dK = (out[2], out[3]) if side == "student" else (out[0], out[1])
    assert all(out[i] is None for i in range(4) if not need[i])
    bits = oracle_bits(ins)
    rows = sample_rows(w.BH, w.NQ, 256, seed=w.seed + 1)
    _, _, _, oq1, oq2 = fwdbwd16k_oracle(orc, bits, "rows", tuple(rows.ravel().tolist()), g)
    gq = dQ.reshape(w.BH, w.NQ, -1)[rows[:, 0], rows[:, 1]]
    assert rel_frobenius(gq, oq2 if side == "student" else oq1) <= TOL_GRAD
    heads = [0, int(np.random.default_rng(w.seed + 1).integers(1, w.BH))]
    o = fwdbwd16k_oracle(orc, bits, "heads", tuple(heads), g)
    err = rel_frobenius(dK.reshape(w.BH, w.NK, -1)[heads], o["dK2" if side == "student" else "dK1"])
    assert err <= TOL_GRAD, f"{side} dK {err:.3e}"

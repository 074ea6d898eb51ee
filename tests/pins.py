"""Pins for the fp64 oracle: facts fixed by the StreamKL summary page and by
mathematics, not by the oracle's own formula.

Each ``pin_*`` function takes an oracle handle and raises AssertionError when
the oracle disagrees.  ``test_oracle_pins.py`` runs them against the oracle
and against builds with one planted mistake each, which must fail at least one.

What pins what:
* brute force (library softmax/logsumexp/entropy on full matrices): L, LSE,
  the causal mask, operand order;
* exact bf16 decode: the input path;
* Gibbs' inequality, identical distributions give 0, common key shift and key
  permutation invariances: the log-ratio and LSE bookkeeping;
* closed forms for one and two keys: L, LSE and every gradient;
* central finite differences of sum_i g_i L_i: the whole backward;
* zero column sums of the key gradients (softmax shift invariance): the
  "- L" term of dL/dx1 in its log-probability reading;
* the large-N_K limit (sigma1^2 + sigma2^2)/2 for independent Gaussian
  teacher and student: plausibility at the sparse-student shape.
"""
from __future__ import annotations

import numpy as np

from brute import brute_forward

RNG_SEED = 20260602


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.abs(a - b) / np.maximum(1.0, np.abs(b))
    if not np.all(err <= tol):
        raise AssertionError(f"{what}: max scaled error {err.max():.3e} > {tol:.1e}")


def _problem(rng, BH, NQ, NK, d1, d2, scale=1.0):
    return (_rand(rng, BH, NQ, d1, scale=scale), _rand(rng, BH, NK, d1, scale=scale),
            _rand(rng, BH, NQ, d2, scale=scale), _rand(rng, BH, NK, d2, scale=scale))


BRUTE_CASES = [  # (BH, NQ, NK, d1, d2, causal)
    (2, 16, 16, 8, 8, False),
    (2, 16, 16, 8, 8, True),
    (1, 33, 47, 16, 8, False),
    (1, 40, 64, 8, 16, True),
    (1, 1, 1, 4, 4, True),
    (1, 64, 64, 16, 16, True),
    (1, 5, 3, 4, 2, False),
]


def pin_brute_force(orc):
    rng = np.random.default_rng(RNG_SEED)
    for BH, NQ, NK, d1, d2, causal in BRUTE_CASES:
        Q1, K1, Q2, K2 = _problem(rng, BH, NQ, NK, d1, d2, scale=1.5)
        s1, s2 = 1.0 / np.sqrt(d1), 0.7 / np.sqrt(d2)
        L, A, B = orc.fwd_all(Q1, K1, Q2, K2, causal=causal, s1=s1, s2=s2, nthreads=2)
        bL, bA, bB = brute_forward(Q1, K1, Q2, K2, causal, s1, s2)
        tag = f"brute BH{BH} NQ{NQ} NK{NK} d{d1}/{d2} causal={causal}"
        _close(L, bL, 1e-12, tag + " L")
        _close(A, bA, 1e-12, tag + " LSE1")
        _close(B, bB, 1e-12, tag + " LSE2")


def pin_bf16_decode(orc):
    """bf16 bit patterns must give exactly the result of their float64 values."""
    rng = np.random.default_rng(RNG_SEED + 1)
    shape_q, shape_k = (2, 24, 16), (2, 40, 16)
    # values k/64 with |k| < 256 are exact in bf16 (8 significant bits)
    vals = [rng.integers(-255, 256, size=s).astype(np.float64) / 64.0
            for s in (shape_q, shape_k, shape_q, shape_k)]
    bits = [(v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16) for v in vals]
    for causal in (False, True):
        r64 = orc.fwd_all(*vals, causal=causal, nthreads=2)
        rbf = orc.fwd_all(*bits, causal=causal, nthreads=2)
        for a, b, n in zip(r64, rbf, ("L", "LSE1", "LSE2")):
            if not np.array_equal(a, b):
                raise AssertionError(f"bf16 decode changes {n}")


def pin_gibbs(orc):
    rng = np.random.default_rng(RNG_SEED + 2)
    for causal in (False, True):
        Q1, K1, Q2, K2 = _problem(rng, 3, 48, 48, 16, 16, scale=2.0)
        L, _, _ = orc.fwd_all(Q1, K1, Q2, K2, causal=causal, nthreads=2)
        if L.min() < -1e-12:
            raise AssertionError(f"KL below zero: {L.min():.3e}")
        if L.max() <= 0.0:
            raise AssertionError("KL of different distributions is not positive")


def pin_identical_zero(orc):
    rng = np.random.default_rng(RNG_SEED + 3)
    Q, K, _, _ = _problem(rng, 2, 20, 20, 8, 8)
    for causal in (False, True):
        L, A, B = orc.fwd_all(Q, K, Q, K, causal=causal, nthreads=2)
        if not (np.all(L == 0.0) and np.array_equal(A, B)):
            raise AssertionError("identical distributions must give L == 0 and LSE1 == LSE2")
        g = rng.standard_normal((2, 20))
        out = orc.bwd_heads(Q, K, Q, K, [0, 1], g, causal=causal, nthreads=2)
        for n in ("dQ1", "dK1", "dQ2", "dK2"):
            if not np.all(out[n] == 0.0):
                raise AssertionError(f"identical distributions must give {n} == 0")


def pin_key_shift(orc):
    """Adding v to every key of K2 shifts x2 by a per-row constant: L fixed, LSE2 += s2<Q2_i, v>."""
    rng = np.random.default_rng(RNG_SEED + 4)
    Q1, K1, Q2, K2 = _problem(rng, 2, 16, 24, 8, 8)
    v = rng.standard_normal(8)
    for causal in (False, True):
        L, A, B = orc.fwd_all(Q1, K1, Q2, K2, causal=causal, nthreads=2)
        Ls, As, Bs = orc.fwd_all(Q1, K1, Q2, K2 + v, causal=causal, nthreads=2)
        shift = (Q2 @ v) / np.sqrt(8)
        _close(Ls, L, 1e-12, "key shift: L")
        _close(As, A, 0.0, "key shift: LSE1")
        _close(Bs, B + shift, 1e-12, "key shift: LSE2")


def pin_key_permutation(orc):
    """Non-causal: permuting keys (K1 and K2 together) leaves L and LSE unchanged; dK permutes."""
    rng = np.random.default_rng(RNG_SEED + 5)
    Q1, K1, Q2, K2 = _problem(rng, 1, 12, 30, 8, 4)
    perm = rng.permutation(30)
    L, A, B = orc.fwd_all(Q1, K1, Q2, K2, nthreads=2)
    Lp, Ap, Bp = orc.fwd_all(Q1, K1[:, perm], Q2, K2[:, perm], nthreads=2)
    _close(Lp, L, 1e-12, "permutation: L")
    _close(Ap, A, 1e-12, "permutation: LSE1")
    _close(Bp, B, 1e-12, "permutation: LSE2")
    g = rng.standard_normal((1, 12))
    o = orc.bwd_heads(Q1, K1, Q2, K2, [0], g, nthreads=2)
    op = orc.bwd_heads(Q1, K1[:, perm], Q2, K2[:, perm], [0], g, nthreads=2)
    _close(op["dQ1"], o["dQ1"], 1e-12, "permutation: dQ1")
    _close(op["dK1"], o["dK1"][:, perm], 1e-12, "permutation: dK1")
    _close(op["dK2"], o["dK2"][:, perm], 1e-12, "permutation: dK2")


def _softplus(a):
    return np.logaddexp(0.0, a)


def _sigmoid(a):
    return np.exp(-_softplus(-a))


def pin_two_keys(orc):
    """N_K = 2: with a = x1_0 - x1_1, b = x2_0 - x2_1, p = sigmoid(a), q = sigmoid(b):
    L = p(a-b) - softplus(a) + softplus(b), LSE1 = x1_1 + softplus(a),
    dL/da = p(1-p)(a-b), dL/db = q - p."""
    rng = np.random.default_rng(RNG_SEED + 6)
    BH, NQ, d1, d2 = 2, 9, 6, 5
    Q1, K1, Q2, K2 = _problem(rng, BH, NQ, 2, d1, d2, scale=1.3)
    s1, s2 = 0.9, 0.6
    g = rng.standard_normal((BH, NQ))
    out = orc.bwd_heads(Q1, K1, Q2, K2, list(range(BH)), g, s1=s1, s2=s2, nthreads=2)
    L, A, B = orc.fwd_all(Q1, K1, Q2, K2, s1=s1, s2=s2, nthreads=2)
    for h in range(BH):
        x1 = s1 * Q1[h] @ K1[h].T
        x2 = s2 * Q2[h] @ K2[h].T
        a = x1[:, 0] - x1[:, 1]
        b = x2[:, 0] - x2[:, 1]
        p, q = _sigmoid(a), _sigmoid(b)
        _close(L[h], p * (a - b) - _softplus(a) + _softplus(b), 1e-12, "two keys: L")
        _close(A[h], x1[:, 1] + _softplus(a), 1e-12, "two keys: LSE1")
        _close(B[h], x2[:, 1] + _softplus(b), 1e-12, "two keys: LSE2")
        da = g[h] * p * (1 - p) * (a - b)     # dL/dx1_0 = -dL/dx1_1
        db = g[h] * (q - p)                   # dL/dx2_0 = -dL/dx2_1
        _close(out["dQ1"][h], s1 * da[:, None] * (K1[h, 0] - K1[h, 1])[None, :], 1e-12,
               "two keys: dQ1")
        _close(out["dQ2"][h], s2 * db[:, None] * (K2[h, 0] - K2[h, 1])[None, :], 1e-12,
               "two keys: dQ2")
        dk1 = s1 * (da[:, None] * Q1[h]).sum(0)
        dk2 = s2 * (db[:, None] * Q2[h]).sum(0)
        _close(out["dK1"][h], np.stack([dk1, -dk1]), 1e-12, "two keys: dK1")
        _close(out["dK2"][h], np.stack([dk2, -dk2]), 1e-12, "two keys: dK2")


def pin_one_key(orc):
    """N_K = 1: L = 0, LSE_t = x_t, every gradient 0."""
    rng = np.random.default_rng(RNG_SEED + 7)
    Q1, K1, Q2, K2 = _problem(rng, 1, 7, 1, 4, 3)
    L, A, B = orc.fwd_all(Q1, K1, Q2, K2, s1=1.0, s2=1.0, nthreads=2)
    _close(L, 0.0 * L, 0.0, "one key: L")
    _close(A, (Q1[0] @ K1[0].T)[:, 0][None], 1e-14, "one key: LSE1")
    _close(B, (Q2[0] @ K2[0].T)[:, 0][None], 1e-14, "one key: LSE2")
    out = orc.bwd_heads(Q1, K1, Q2, K2, [0], np.ones((1, 7)), s1=1.0, s2=1.0, nthreads=2)
    for n in ("dQ1", "dK1", "dQ2", "dK2"):
        if np.abs(out[n]).max() > 1e-15:
            raise AssertionError(f"one key: {n} must vanish")


FD_CASES = [  # (NQ, NK, d1, d2, causal)
    (6, 6, 4, 4, False),
    (8, 8, 4, 3, True),
    (5, 9, 3, 5, True),
    (7, 4, 4, 4, False),
]


def pin_finite_differences(orc):
    """Central differences of F = sum_i g_i L_i against every gradient element."""
    rng = np.random.default_rng(RNG_SEED + 8)
    for NQ, NK, d1, d2, causal in FD_CASES:
        Q1, K1, Q2, K2 = _problem(rng, 1, NQ, NK, d1, d2)
        s1, s2 = 1.0 / np.sqrt(d1), 1.0 / np.sqrt(d2)
        g = rng.standard_normal((1, NQ))
        out = orc.bwd_heads(Q1, K1, Q2, K2, [0], g, causal=causal, s1=s1, s2=s2, nthreads=1)
        ins = {"Q1": Q1, "K1": K1, "Q2": Q2, "K2": K2}

        def F(**over):
            a = {**ins, **over}
            L, _, _ = orc.fwd_all(a["Q1"], a["K1"], a["Q2"], a["K2"], causal=causal, s1=s1, s2=s2,
                                  nthreads=1)
            return float((g * L).sum())

        for name in ("Q1", "K1", "Q2", "K2"):
            base = ins[name]
            fd = np.zeros_like(base)
            for idx in np.ndindex(base.shape):
                h = 1e-6 * max(1.0, abs(base[idx]))
                up = base.copy(); up[idx] += h
                dn = base.copy(); dn[idx] -= h
                fd[idx] = (F(**{name: up}) - F(**{name: dn})) / (2 * h)
            an = out["d" + name]
            rel = np.linalg.norm(fd - an) / max(np.linalg.norm(an), 1e-30)
            if not (rel <= 1e-7 and np.abs(fd - an).max() <= 1e-8):
                raise AssertionError(
                    f"finite differences d{name} NQ{NQ} NK{NK} causal={causal}: rel {rel:.2e}")


def pin_key_gradient_sums(orc):
    """Softmax is shift invariant per row, so sum_j dS_t[i, j] = 0 and hence sum_j dK_t[j] = 0."""
    rng = np.random.default_rng(RNG_SEED + 9)
    for causal in (False, True):
        Q1, K1, Q2, K2 = _problem(rng, 1, 24, 24, 8, 8, scale=1.5)
        g = rng.standard_normal((1, 24))
        o = orc.bwd_heads(Q1, K1, Q2, K2, [0], g, causal=causal, nthreads=2)
        for n in ("dK1", "dK2"):
            s = np.abs(o[n].sum(axis=1)).max()
            scale = np.abs(o[n]).max()
            if s > 1e-12 * max(1.0, scale):
                raise AssertionError(f"{n} column sum {s:.2e} is not zero (causal={causal})")


def pin_independent_limit(orc):
    """Independent Gaussian teacher and student, large N_K: L_i -> (sigma1^2 + sigma2^2)/2 with
    sigma_t^2 = |Q_t,i|^2 / d_t.  Checked at N_K = 32768, d1 = 128, d2 = 64 (bf16 inputs)."""
    from attention_kl_distillation_b200.inputs import WORKLOADS, bf16_bits, make_inputs
    w = WORKLOADS["sparse_student"].with_(B=1, H=1, NQ=8)
    Q1, K1, Q2, K2 = make_inputs(w)
    bits = [bf16_bits(t) for t in (Q1, K1, Q2, K2)]
    rows = np.stack([np.zeros(8, np.int64), np.arange(8)], axis=1)
    L, _, _ = orc.fwd_rows(*bits, rows, nthreads=2)
    q1 = Q1.float().numpy()[0, 0].astype(np.float64)
    q2 = Q2.float().numpy()[0, 0].astype(np.float64)
    pred = 0.5 * ((q1 ** 2).sum(1) / w.d1 + (q2 ** 2).sum(1) / w.d2)
    if np.abs(L - pred).max() > 0.05:
        raise AssertionError(f"independent limit off by {np.abs(L - pred).max():.3f}")


ALL_PINS = [
    pin_brute_force, pin_bf16_decode, pin_gibbs, pin_identical_zero, pin_key_shift,
    pin_key_permutation, pin_two_keys, pin_one_key, pin_finite_differences,
    pin_key_gradient_sums, pin_independent_limit,
]

"""Helpers shared by the GPU parity tests (CUDA path through the C ABI vs the oracle)."""
from __future__ import annotations

import numpy as np
import torch

from attention_kl_distillation_b200.inputs import Workload, bf16_bits, make_inputs

# Forward tolerances: |dL| <= 2e-3 * max(1, |L|), |dLSE| <= 1e-3 (absolute).
TOL_L = 2e-3
TOL_LSE = 1e-3
# Gradients: relative Frobenius error per tensor over the checked subset.
TOL_GRAD = 2e-2


def workload(B, H, NQ, NK, d1, d2, causal, seed=7, sigma=0.5):
    student = "perturb" if d1 == d2 else "independent"
    return Workload(f"B{B}H{H}Q{NQ}K{NK}d{d1}/{d2}{'c' if causal else ''}", B, H, NQ, NK, d1, d2,
                    bool(causal), student, sigma, False, seed)


def cuda_inputs(cpu_inputs):
    return [t.cuda() for t in cpu_inputs]


def oracle_bits(cpu_inputs):
    return [bf16_bits(t) for t in cpu_inputs]


def gpu_fwd(dev_inputs, causal, s1=None, s2=None):
    from attention_kl_distillation_b200 import fwd, query_device_status
    L, A, B = fwd(*dev_inputs, causal=causal, s1=s1, s2=s2)
    torch.cuda.synchronize()
    assert query_device_status() == 0
    BH = L.shape[0] * L.shape[1]
    return tuple(t.reshape(BH, -1).cpu().numpy().astype(np.float64) for t in (L, A, B))


def check_fwd(gpu, ora_vals, rows, what=""):
    """gpu: (L, LSE1, LSE2) [BH, NQ]; ora_vals: oracle values for `rows` [n, 2]."""
    gL, gA, gB = (g[rows[:, 0], rows[:, 1]] for g in gpu)
    oL, oA, oB = ora_vals
    assert np.all(np.isfinite(gL)) and np.all(np.isfinite(gA)) and np.all(np.isfinite(gB)), what
    eL = np.abs(gL - oL) / np.maximum(1.0, np.abs(oL))
    eA = np.abs(gA - oA)
    eB = np.abs(gB - oB)
    assert eL.max() <= TOL_L, f"{what} L error {eL.max():.3e} at row {rows[eL.argmax()]}"
    assert eA.max() <= TOL_LSE, f"{what} LSE1 error {eA.max():.3e} at row {rows[eA.argmax()]}"
    assert eB.max() <= TOL_LSE, f"{what} LSE2 error {eB.max():.3e} at row {rows[eB.argmax()]}"
    return eL.max(), max(eA.max(), eB.max())


def all_rows(BH, NQ):
    bh, i = np.meshgrid(np.arange(BH), np.arange(NQ), indexing="ij")
    return np.stack([bh.ravel(), i.ravel()], axis=1).astype(np.int64)


def rel_frobenius(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))

"""Brute-force fp64 reference for tiny inputs, built from library routines.

Independent of the oracle: it materialises the full N_Q x N_K attention maps
with numpy, normalises them with ``scipy.special.softmax``, takes LSE from
``scipy.special.logsumexp`` and the divergence from ``scipy.stats.entropy``
(sum of p*log(p/q) with direct logs of probabilities).  Only for tiny shapes.
"""
from __future__ import annotations

import numpy as np
from scipy import special, stats


def visible_mask(NQ: int, NK: int, causal: bool) -> np.ndarray:
    """Boolean [NQ, NK]; causal visibility is bottom-right aligned (j <= i + NK - NQ)."""
    if not causal:
        return np.ones((NQ, NK), dtype=bool)
    i = np.arange(NQ)[:, None]
    j = np.arange(NK)[None, :]
    return j <= i + (NK - NQ)


def brute_forward(Q1, K1, Q2, K2, causal, s1, s2):
    """Q*/K* float64 [BH, N, d].  Returns L, LSE1, LSE2 as [BH, NQ]."""
    BH, NQ, _ = Q1.shape
    NK = K1.shape[1]
    mask = visible_mask(NQ, NK, causal)
    L = np.zeros((BH, NQ))
    A = np.zeros((BH, NQ))
    B = np.zeros((BH, NQ))
    for h in range(BH):
        x1 = s1 * (Q1[h] @ K1[h].T)
        x2 = s2 * (Q2[h] @ K2[h].T)
        for i in range(NQ):
            v = mask[i]
            P1 = special.softmax(x1[i, v])
            P2 = special.softmax(x2[i, v])
            L[h, i] = stats.entropy(P1, P2)
            A[h, i] = special.logsumexp(x1[i, v])
            B[h, i] = special.logsumexp(x2[i, v])
    return L, A, B

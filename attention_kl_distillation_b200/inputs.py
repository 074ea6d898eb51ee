"""Seeded synthetic inputs for the attention-KL path.

This module holds the input recipe only (shapes, value distributions, seeds,
row samples).  It contains none of the method's arithmetic, and it is the one
piece of code that both the CUDA path's callers and the CPU oracle's tests
use.

Recipe (the StreamKL summary page names no dataset; its workload is a context
length of 4K to 512K tokens, "Risultati Sperimentali"):

* Q1 and K1 are i.i.d. N(0, 1) in fp32.
* The student is either the teacher plus sigma * N(0, 1) noise (Q2 = Q1 +
  sigma*n, K2 = K1 + sigma*n', when d1 == d2), or independent N(0, 1) draws.
* Draw order from one seeded ``torch.Generator``: Q1, K1, then Q2's draw,
  then K2's draw.  Each tensor is rounded once to bf16 (round to nearest
  even).  Those bf16 bytes are the single source of truth for both sides.
* Layout: contiguous [B, H, N, d].
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    NQ: int
    NK: int
    d1: int
    d2: int
    causal: bool
    student: str          # "perturb" or "independent"
    sigma: float = 0.0    # noise scale for "perturb"
    backward: bool = False
    seed: int = 0

    @property
    def BH(self) -> int:
        return self.B * self.H

    def visible_pairs(self) -> int:
        """Query/key pairs that are visible (bottom-right aligned causal mask)."""
        if not self.causal:
            return self.BH * self.NQ * self.NK
        return self.BH * _causal_pairs(self.NQ, self.NK)

    def fwd_flops(self) -> int:
        """Algorithmic forward FLOPs: two QK^T products over visible pairs."""
        return 2 * (self.d1 + self.d2) * self.visible_pairs()

    def bwd_flops(self) -> int:
        """Algorithmic backward FLOPs: two recomputed products and four contractions."""
        return 6 * (self.d1 + self.d2) * self.visible_pairs()

    def input_bytes(self) -> int:
        return 2 * self.BH * (self.NQ * (self.d1 + self.d2) + self.NK * (self.d1 + self.d2))

    def materialised_bytes(self) -> int:
        """Bytes to hold both N_Q x N_K attention maps in bf16 (the materialising baseline)."""
        return 2 * self.BH * self.NQ * self.NK * 2

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _causal_pairs(NQ: int, NK: int) -> int:
    off = NK - NQ
    i = np.arange(NQ, dtype=np.int64)
    return int(np.clip(i + off + 1, 0, NK).sum())


# The five workloads: shapes, distributions and seeds (seed = 1000 + index).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 256, 64, 64, False, "perturb", 0.3, False, 1001),
    "causal4k": Workload("causal4k", 1, 32, 4096, 4096, 128, 128, True, "perturb", 0.5, False, 1002),
    "sparse_student": Workload("sparse_student", 2, 16, 2048, 32768, 128, 64, False, "independent",
                               0.0, False, 1003),
    "long64k": Workload("long64k", 1, 32, 65536, 65536, 128, 128, True, "perturb", 0.5, False, 1004),
    "fwdbwd16k": Workload("fwdbwd16k", 1, 32, 16384, 16384, 128, 128, True, "perturb", 0.5, True,
                          1005),
}


def make_inputs(w: Workload, seed: int | None = None):
    """Q1, K1, Q2, K2 as contiguous bf16 CPU tensors [B, H, N, d]."""
    g = torch.Generator().manual_seed(int(w.seed if seed is None else seed))
    B, H = w.B, w.H

    def draw(n, d):
        return torch.randn((B, H, n, d), generator=g, dtype=torch.float32)

    q1 = draw(w.NQ, w.d1)
    k1 = draw(w.NK, w.d1)
    Q1 = q1.to(torch.bfloat16)
    K1 = k1.to(torch.bfloat16)
    if w.student == "perturb":
        if w.d1 != w.d2:
            raise ValueError("a perturbed student needs d1 == d2")
        n = draw(w.NQ, w.d2)
        n.mul_(w.sigma).add_(q1)
        Q2 = n.to(torch.bfloat16)
        del n
        n = draw(w.NK, w.d2)
        n.mul_(w.sigma).add_(k1)
        K2 = n.to(torch.bfloat16)
        del n
    elif w.student == "independent":
        Q2 = draw(w.NQ, w.d2).to(torch.bfloat16)
        K2 = draw(w.NK, w.d2).to(torch.bfloat16)
    else:
        raise ValueError(f"unknown student recipe {w.student!r}")
    return Q1, K1, Q2, K2


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU bf16 tensor, as uint16 numpy (no copy of values)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def edge_rows(NQ: int) -> list[int]:
    """Rows that sit on tile and causal edges: 0, 1, 127, 128, 129 and NQ-1 (those that exist)."""
    return sorted({r for r in (0, 1, 127, 128, 129, NQ - 1) if 0 <= r < NQ})


def sample_rows(BH: int, NQ: int, per_head: int, seed: int, heads=None) -> np.ndarray:
    """A seeded sample of (bh, i) rows: per head, the edge rows plus per_head random rows."""
    rng = np.random.default_rng(seed)
    heads = range(BH) if heads is None else heads
    out = []
    for bh in heads:
        if per_head >= NQ:
            rows = np.arange(NQ)
        else:
            rows = np.union1d(rng.choice(NQ, size=per_head, replace=False), edge_rows(NQ))
        out.append(np.stack([np.full(rows.shape, bh), rows], axis=1))
    return np.concatenate(out, axis=0).astype(np.int64)

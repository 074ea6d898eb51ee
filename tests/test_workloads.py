"""The workload accounting behind every reported rate: visible pairs, FLOPs and bytes.

The pair counts are checked by brute force against the bottom-right causal mask
(key j visible from row i when j <= i + NK - NQ), and the recipes against their
closed forms: B*H*NQ*NK without a mask, B*H*N(N+1)/2 for square causal shapes.
FLOPs count only visible pairs: 2(d1+d2) per pair forward (the two QK^T products,
StreamKL summary page, "Metodologia" section 1) and 6(d1+d2) backward (two
recomputed products and four contractions, section 2).
"""
import itertools

import numpy as np
import pytest

from attention_kl_distillation_b200.inputs import WORKLOADS, Workload


def _brute_pairs(NQ, NK, causal):
    i = np.arange(NQ)[:, None]
    j = np.arange(NK)[None, :]
    visible = (j <= i + NK - NQ) if causal else np.ones((NQ, NK), bool)
    return int(visible.sum())


@pytest.mark.parametrize("NQ,NK,causal", [
    (nq, nk, c) for nq, nk, c in itertools.product([1, 2, 63, 64, 129, 300], [1, 2, 64, 128, 300], [False, True])
    if not (c and nq > nk)])
def test_visible_pairs_match_the_mask(NQ, NK, causal):
    w = Workload("t", B=2, H=3, NQ=NQ, NK=NK, d1=64, d2=128, causal=causal, student="independent")
    assert w.visible_pairs() == 6 * _brute_pairs(NQ, NK, causal)


def test_recipe_pairs_closed_forms():
    for w in WORKLOADS.values():
        if w.causal:
            assert w.NQ == w.NK, "every causal recipe is square"
            assert w.visible_pairs() == w.BH * w.NQ * (w.NQ + 1) // 2
        else:
            assert w.visible_pairs() == w.BH * w.NQ * w.NK


def test_recipe_flops_and_bytes():
    w = WORKLOADS["fwdbwd16k"]  # B1 H32 N16384 d128 causal
    pairs = 32 * 16384 * 16385 // 2
    assert w.visible_pairs() == pairs == 4_295_229_440
    assert w.fwd_flops() == 2 * 256 * pairs == 2_199_157_473_280
    assert w.bwd_flops() == 6 * 256 * pairs == 6_597_472_419_840
    assert w.input_bytes() == 2 * 32 * 16384 * 4 * 128 == 536_870_912
    s = WORKLOADS["sparse_student"]  # B2 H16 NQ2048 NK32768, d1 128, d2 64, no mask
    assert s.visible_pairs() == 2 * 16 * 2048 * 32768 == 2_147_483_648
    assert s.fwd_flops() == 2 * (128 + 64) * 2_147_483_648


def test_overrides_keep_the_accounting():
    w = WORKLOADS["long64k"].with_(NQ=1)
    assert w.visible_pairs() == w.BH * (w.NK - w.NQ + 1)  # the one row sees every key
    assert w.fwd_flops() == 2 * (w.d1 + w.d2) * w.visible_pairs()

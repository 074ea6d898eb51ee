"""CPU tests: the fp64 oracle against what the StreamKL page and mathematics fix.

Also plants one mistake at a time in the oracle (compile-time switch, CPU only)
and checks that at least one pin catches each of them.
"""
import json
from pathlib import Path

import numpy as np
import pytest

import pins
from oracle import oracle as O

GOLDEN = Path(__file__).resolve().parent / "golden"


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


# planted mistakes: 1 LSE2 dropped from the log ratio, 2 sign of dL/dx2,
# 3 transposed key operand, 4 causal frontier off by one, 5 raw-logit dL/dx1
@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5])
def test_pins_catch_planted_mistake(tmp_path, mutant):
    bad = O.Oracle(O.build(mutant, out_dir=tmp_path))
    assert bad.mutant == mutant
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(bad)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught planted mistake {mutant}"


def test_page_materialisation_number():
    """The page's worked number: both bf16 maps at 64K context and 32 heads are 512 GiB."""
    from attention_kl_distillation_b200.inputs import WORKLOADS
    g = json.loads((GOLDEN / "p1_materialisation.json").read_text())
    w = WORKLOADS["long64k"]
    assert (w.NQ, w.H) == (g["context_tokens"], g["heads"])
    assert w.materialised_bytes() == g["bytes_exact"] == g["gib"] * 2**30
    assert g["bytes_exact"] > g["h200_capacity_gb"] * 10**9


def test_bwd_rows_match_heads(orc):
    """The row-list backward and the whole-head backward agree on dQ."""
    rng = np.random.default_rng(5)
    Q1, K1, Q2, K2 = (rng.standard_normal(s) for s in [(2, 20, 8), (2, 28, 8), (2, 20, 4), (2, 28, 4)])
    g = rng.standard_normal((2, 20))
    for causal in (False, True):
        o = orc.bwd_heads(Q1, K1, Q2, K2, [0, 1], g, causal=causal)
        rows = np.array([[1, 0], [0, 7], [1, 19]])
        L, A, B, dq1, dq2 = orc.bwd_rows(Q1, K1, Q2, K2, rows, g[rows[:, 0], rows[:, 1]], causal=causal)
        for r, (h, i) in enumerate(rows):
            assert abs(L[r] - o["L"][h, i]) <= 1e-13
            np.testing.assert_allclose(dq1[r], o["dQ1"][h, i], rtol=0, atol=1e-13)
            np.testing.assert_allclose(dq2[r], o["dQ2"][h, i], rtol=0, atol=1e-13)


def test_rejects_bad_rows(orc):
    Q = np.zeros((1, 4, 2)); K = np.zeros((1, 4, 2))
    with pytest.raises(RuntimeError):
        orc.fwd_rows(Q, K, Q, K, np.array([[0, 4]]))
    with pytest.raises(RuntimeError):
        orc.fwd_rows(Q, K, Q, K, np.array([[1, 0]]))

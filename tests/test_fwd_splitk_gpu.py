"""GPU parity of the split-K forward (streamkl_fwd_splitk) against the oracle and
against the unsplit forward; the merge of partial states must reproduce the row
statistics for every split count."""
import numpy as np
import pytest
import torch

from gpu_common import all_rows, check_fwd, cuda_inputs, gpu_fwd, oracle_bits, workload

pytestmark = pytest.mark.gpu

SHAPES = [  # B, H, NQ, NK, d1, d2, causal
    (1, 4, 1, 5000, 128, 128, False),     # decode: one query row
    (1, 4, 1, 5000, 128, 128, True),
    (1, 2, 7, 300, 64, 64, True),
    (1, 2, 300, 2000, 128, 64, False),
    (2, 3, 129, 1000, 64, 128, True),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}Q{}K{}d{}-{}{}".format(*s[:6], "c" if s[6] else ""))
@pytest.mark.parametrize("nsplit", [1, 2, 3, 7, 10000])
def test_splitk_matches_oracle(orc, shape, nsplit):
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
    ref = gpu_fwd(dev, w.causal)
    assert np.abs(gpu[0] - ref[0]).max() <= 1e-4
    assert np.abs(gpu[1] - ref[1]).max() <= 1e-4 and np.abs(gpu[2] - ref[2]).max() <= 1e-4


def test_splitk_suggested_split_full_decode_workload(orc):
    """Decode-sized query count on the 64K long-context key set: B1 H32 NQ=1 NK=65536 causal."""
    from attention_kl_distillation_b200 import fwd_splitk
    from attention_kl_distillation_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["long64k"].with_(NQ=1)
    ins = make_inputs(w)
    dev = cuda_inputs(ins)
    L, A, B = fwd_splitk(*dev, causal=True)
    torch.cuda.synchronize()
    gpu = tuple(t.reshape(w.BH, -1).cpu().numpy().astype(np.float64) for t in (L, A, B))
    rows = all_rows(w.BH, 1)
    check_fwd(gpu, orc.fwd_rows(*oracle_bits(ins), rows, causal=True), rows, "decode 64K")

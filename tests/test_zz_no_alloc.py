"""The allocation-free backward entry point (streamkl_bwd_noalloc).

It exists for callers that cannot allocate device memory when they need the
gradient, such as a framework whose caching allocator already holds the free
memory, or code that must not call cudaMalloc because it may synchronise the
device.  It must give the same gradients as the ordinary entry point, which
takes a caller-allocated workspace, on two calls in a row, since every call
reuses the same static scratch.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from attention_kl_distillation_b200 import binding as B


def test_noalloc_rejects_problem_larger_than_scratch():
    """Rejected before any CUDA call when the needed scratch exceeds 64 MiB."""
    prob = B.problem(1, 32, 16384, 16384, 128, 128, causal=True)
    assert B.workspace_size(1, 32, 16384, 16384, 128, 128, True) > B.NOALLOC_SCRATCH_BYTES
    ptrs = [ctypes.c_void_p(256 * (k + 1)) for k in range(12)]  # dL, inputs, saved, outputs
    assert B.lib().streamkl_bwd_noalloc(ctypes.byref(prob), *ptrs, ctypes.c_void_p(0)) == B.EINVAL


def _cpu_args(NQ=40, NK=48, d1=64, d2=64):
    g = torch.Generator().manual_seed(5)
    Q1, K1, Q2, K2 = (torch.randn(1, 2, n, d, generator=g).to(torch.bfloat16)
                      for n, d in ((NQ, d1), (NK, d1), (NQ, d2), (NK, d2)))
    vec = [torch.zeros(1, 2, NQ) for _ in range(4)]     # dL, L, LSE1, LSE2
    out = [torch.empty_like(t) for t in (Q1, K1, Q2, K2)]
    return [vec[0], Q1, K1, Q2, K2, *vec[1:]], out


@pytest.mark.parametrize("case", ["short_out", "wrong_shape", "wrong_dtype", "strided",
                                  "bf16_dL", "wrong_L_shape", "no_output"])
def test_noalloc_refuses_bad_tensors_before_any_call(case):
    """The library receives raw pointers only, so the binding refuses anything that
    would make the kernels read or write out of bounds, on the host, before a call."""
    args, out = _cpu_args()
    if case == "short_out":
        out = out[:3]
    elif case == "wrong_shape":
        out[1] = torch.empty(1, 2, 47, 64, dtype=torch.bfloat16)
    elif case == "wrong_dtype":
        out[0] = out[0].float()
    elif case == "strided":
        out[2] = torch.empty(1, 2, 64, 40, dtype=torch.bfloat16).transpose(2, 3)
    elif case == "bf16_dL":
        args[0] = args[0].to(torch.bfloat16)
    elif case == "wrong_L_shape":
        args[5] = torch.zeros(1, 2, 41)
    elif case == "no_output":
        out = [None] * 4
    calls = B.launch_count()
    with pytest.raises(ValueError):
        B.bwd_noalloc(*args, out)
    assert B.launch_count() == calls


def test_noalloc_scratch_size_matches_header():
    import re
    text = B.HEADER.read_text()
    m = re.search(r"#define STREAMKL_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m, "macro not found in the header"
    assert B.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point():
    from gpu_common import TOL_GRAD, cuda_inputs, rel_frobenius, workload

    from attention_kl_distillation_b200 import bwd, fwd, query_device_status
    from attention_kl_distillation_b200.inputs import make_inputs

    w = workload(1, 3, 777, 777, 128, 64, True)
    assert B.workspace_size(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, True) <= B.NOALLOC_SCRATCH_BYTES
    Q1, K1, Q2, K2 = cuda_inputs(make_inputs(w))
    dL = torch.randn((w.B, w.H, w.NQ), generator=torch.Generator().manual_seed(21)).cuda()
    L, A, Bv = fwd(Q1, K1, Q2, K2, causal=True)
    ref = [g.float() for g in bwd(dL, Q1, K1, Q2, K2, L, A, Bv, causal=True)]
    for call in range(2):
        out = tuple(torch.full_like(t, float("nan")) for t in (Q1, K1, Q2, K2))
        B.bwd_noalloc(dL, Q1, K1, Q2, K2, L, A, Bv, out, causal=True)
        torch.cuda.synchronize()
        assert query_device_status() == 0
        for name, g, r in zip(("dQ1", "dK1", "dQ2", "dK2"), out, ref):
            g = g.float().cpu().numpy()
            assert np.all(np.isfinite(g)), f"call {call}: {name} not finite"
            err = rel_frobenius(g, r.cpu().numpy())
            assert err <= TOL_GRAD, f"call {call}: {name} differs by {err:.3e}"

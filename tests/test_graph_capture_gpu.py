"""The library's calls can be captured in a CUDA graph: no host synchronisation
and no allocation on the launch path.  A captured forward + backward replays
to the eager results (the forward bit for bit; gradients within fp32-atomic
rounding)."""
import pytest
import torch

from gpu_common import cuda_inputs, workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nq", [300, 20], ids=["row_tiles", "transposed"])
def test_forward_backward_in_a_cuda_graph(nq):
    from attention_kl_distillation_b200 import binding as B
    from attention_kl_distillation_b200 import bwd, fwd, workspace_size
    from attention_kl_distillation_b200.inputs import make_inputs
    w = workload(1, 2, nq, 400, 128, 128, True)
    Q1, K1, Q2, K2 = cuda_inputs(make_inputs(w))
    dL = torch.randn((1, 2, nq), device="cuda")
    L, A, Bv = (torch.empty((1, 2, nq), device="cuda") for _ in range(3))
    grads = tuple(torch.empty_like(t) for t in (Q1, K1, Q2, K2))
    ws = torch.empty(workspace_size(1, 2, nq, 400, 128, 128, True), dtype=torch.uint8, device="cuda")

    def step():
        fwd(Q1, K1, Q2, K2, causal=True, out=(L, A, Bv))
        bwd(dL, Q1, K1, Q2, K2, L, A, Bv, causal=True, workspace=ws, out=grads)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm-up outside the capture (first-call setup, kernel attributes)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (L, A, Bv) + grads]

    launches0 = B.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in (L, A, Bv) + grads:
        t.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert B.launch_count() > launches0  # the captured calls went through the library
    assert B.query_device_status() == 0
    for e, t in zip(eager[:3], (L, A, Bv)):
        assert torch.equal(e, t)
    for e, t in zip(eager[3:], grads):
        err = ((e.float() - t.float()).norm() / e.float().norm()).item()
        assert err <= 1e-2

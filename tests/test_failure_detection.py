"""Failure detection without a GPU fault: a kernel whose producer withholds its
key tiles must time out its bounded waits, record STREAMKL_ETIMEOUT, unwind and
leave the CUDA context usable."""
import pytest

from attention_kl_distillation_b200 import binding as B


def test_inject_argument_validation():
    with pytest.raises(B.StreamKLError):
        B.debug_inject(5)
    B.debug_inject(0)


@pytest.mark.gpu
@pytest.mark.parametrize("nq", [300, 20], ids=["row_tiles", "transposed"])
def test_stalled_producer_times_out_and_context_survives(nq):
    import numpy as np
    import torch

    from attention_kl_distillation_b200 import fwd, query_device_status
    from attention_kl_distillation_b200.inputs import make_inputs
    from gpu_common import cuda_inputs, workload

    w = workload(1, 2, nq, 300, 128, 128, True)
    dev = cuda_inputs(make_inputs(w))
    torch.cuda.synchronize()
    assert query_device_status() == B.OK
    B.set_wait_limit_ms(200)
    try:
        B.debug_inject(1)
        fwd(*dev, causal=True)                       # launches; waits run out on the device
        assert query_device_status() == B.ETIMEOUT   # recorded, then cleared by the query
        assert query_device_status() == B.OK
    finally:
        B.debug_inject(0)
        B.set_wait_limit_ms(2000)
    # the context is intact: a normal forward runs and matches a second run bit for bit
    L1, _, _ = fwd(*dev, causal=True)
    L2, _, _ = fwd(*dev, causal=True)
    torch.cuda.synchronize()
    assert query_device_status() == B.OK
    assert torch.equal(L1, L2) and bool(torch.isfinite(L1).all())
    assert np.isfinite(L1.cpu().numpy()).all()

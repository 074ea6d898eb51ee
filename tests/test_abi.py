"""CPU tests of the C ABI: the library loads, exports what the header declares,
and rejects bad arguments on the host before any CUDA call."""
import ctypes

import pytest

from attention_kl_distillation_b200 import binding as B


def test_exports_every_declared_function():
    names = B.header_functions()
    assert {"streamkl_fwd", "streamkl_bwd", "streamkl_bwd_workspace_size",
            "streamkl_status_string", "streamkl_query_device_status"} <= set(names)
    missing = [n for n in names if not hasattr(B.lib(), n)]
    assert not missing, f"declared but not exported: {missing}"


def test_status_strings_and_version():
    assert B.lib().streamkl_abi_version() == 1
    for code in range(6):
        assert B.status_string(code)
    assert B.status_string(B.OK) == "ok"
    assert "timed out" in B.status_string(B.ETIMEOUT)


def _fwd_raw(prob, ptrs=(16, 32, 48, 64), outs=(128, 256, 512)):
    lib = B.lib()
    return lib.streamkl_fwd(ctypes.byref(prob), *[ctypes.c_void_p(p) for p in ptrs],
                            *[ctypes.c_void_p(p) for p in outs], ctypes.c_void_p(0))


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(H=0), dict(NQ=0), dict(NK=0), dict(causal=2),
    dict(causal=1, NQ=129, NK=128),
])
def test_fwd_rejects_bad_sizes(bad):
    kw = dict(B=1, H=1, NQ=64, NK=64, d1=64, d2=64, causal=0)
    kw.update(bad)
    prob = B.Problem(kw["B"], kw["H"], kw["NQ"], kw["NK"], kw["d1"], kw["d2"], kw["causal"], 0.0, 0.0)
    assert _fwd_raw(prob) == B.EINVAL


@pytest.mark.parametrize("d1,d2", [(96, 64), (64, 32), (256, 128), (0, 64)])
def test_fwd_rejects_unsupported_head_dims(d1, d2):
    assert _fwd_raw(B.problem(1, 1, 64, 64, d1, d2)) == B.EUNSUPPORTED


def test_fwd_rejects_null_and_misaligned_pointers():
    prob = B.problem(1, 1, 64, 64, 64, 64)
    assert _fwd_raw(prob, ptrs=(0, 32, 48, 64)) == B.EINVAL
    assert _fwd_raw(prob, ptrs=(16, 32, 48, 72)) == B.EINVAL        # 8-byte aligned only
    assert _fwd_raw(prob, outs=(128, 0, 512)) == B.EINVAL
    assert _fwd_raw(prob, outs=(130, 256, 512)) == B.EINVAL
    assert B.lib().streamkl_fwd(None, *[ctypes.c_void_p(16)] * 7, None) == B.EINVAL


def test_fwd_rejects_nonfinite_scale():
    prob = B.problem(1, 1, 64, 64, 64, 64, s1=float("nan"))
    assert _fwd_raw(prob) == B.EINVAL


def test_workspace_size():
    ws = B.workspace_size(2, 3, 100, 50, 128, 64)
    need = 2 * 3 * 100 * (128 + 64) * 4
    assert ws >= need and ws % 256 == 0 and ws - need < 256 + 4096
    assert B.workspace_size(1, 1, 0, 5, 64, 64) == 0
    assert B.workspace_size(1, 1, 5, 5, 96, 64) == 0


def test_wait_limit_validation():
    with pytest.raises(B.StreamKLError):
        B.set_wait_limit_ms(0)
    B.set_wait_limit_ms(2000)

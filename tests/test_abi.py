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
    need = 2 * 3 * 100 * (128 + 64) * 4 + 2 * 3 * 128 * 8 * 4   # accumulator + row records
    assert ws >= need and ws % 256 == 0 and ws - need <= 768
    assert B.workspace_size(1, 1, 0, 5, 64, 64) == 0
    assert B.workspace_size(1, 1, 5, 5, 96, 64) == 0


def test_wait_limit_validation():
    with pytest.raises(B.StreamKLError):
        B.set_wait_limit_ms(0)
    B.set_wait_limit_ms(2000)


def _bwd_raw(prob, dL=256, ins=(16, 32, 48, 64), vecs=(512, 768, 1024), outs=(2048, 4096, 0, 0),
             ws=1 << 20, ws_bytes=1 << 40):
    lib = B.lib()
    v = ctypes.c_void_p
    return lib.streamkl_bwd(ctypes.byref(prob), v(dL), *[v(p) for p in ins], *[v(p) for p in vecs],
                            *[v(p) for p in outs], v(ws), ctypes.c_size_t(ws_bytes), v(0))


def test_bwd_rejects_bad_arguments():
    prob = B.problem(1, 2, 100, 100, 128, 64, causal=True)
    assert _bwd_raw(prob, dL=0) == B.EINVAL                          # missing dL
    assert _bwd_raw(prob, ins=(16, 32, 0, 64)) == B.EINVAL            # missing input
    assert _bwd_raw(prob, vecs=(512, 770, 1024)) == B.EINVAL          # misaligned LSE1
    assert _bwd_raw(prob, outs=(0, 0, 0, 0)) == B.EINVAL              # nothing requested
    assert _bwd_raw(prob, outs=(2056, 0, 0, 0)) == B.EINVAL           # misaligned output
    assert _bwd_raw(prob, ws=0) == B.EINVAL                           # no workspace
    assert _bwd_raw(prob, ws=(1 << 20) + 16) == B.EINVAL              # workspace not 256-aligned
    need = B.workspace_size(1, 2, 100, 100, 128, 64, True)
    assert _bwd_raw(prob, ws_bytes=need - 1) == B.EINVAL              # workspace too small
    assert _bwd_raw(B.problem(1, 2, 100, 100, 96, 64)) == B.EUNSUPPORTED
    assert _bwd_raw(B.problem(1, 2, 101, 100, 64, 64, causal=True)) == B.EINVAL


def test_binding_argtypes_match_header():
    """Each ctypes prototype has as many arguments as the header declares."""
    import re
    text = B.HEADER.read_text()
    for name in B.header_functions():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", text)
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        fn = getattr(B.lib(), name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == len(params), name


def test_bwd_algorithm_selection():
    """bwd_algorithm_for resolves AUTO and FUSED to a concrete algorithm.  Without a GPU
    the device is taken to have 148 SMs, as a B200 does."""
    lib = B.lib()
    assert lib.streamkl_set_bwd_algorithm(7) == B.EINVAL
    try:
        for name in ("split", "fused_key_tiles", "fused_query_tiles", "fused_sides"):
            B.set_bwd_algorithm(name)
            assert B.bwd_algorithm_for(1, 2, 256, 256, 64, 64) == name
        B.set_bwd_algorithm("fused")
        # query tiles once B*H*ceil(NQ/128) fills the SMs twice (296 units), else key tiles
        assert B.bwd_algorithm_for(1, 32, 16384, 16384, 128, 128, True) == "fused_query_tiles"
        assert B.bwd_algorithm_for(1, 32, 1024, 32768, 128, 128, True) == "fused_key_tiles"
        assert B.bwd_algorithm_for(1, 37, 1024, 1024, 128, 128) == "fused_query_tiles"
        assert B.bwd_algorithm_for(1, 36, 1024, 1024, 128, 128) == "fused_key_tiles"
        B.set_bwd_algorithm("auto")
        # AUTO is FUSED at every size: measured faster than split up to a 5 GiB fp32
        # accumulator (B1 H80 N65536 d128 causal: 357 against 400 ms)
        assert B.bwd_algorithm_for(1, 2, 256, 256, 64, 64) == "fused_key_tiles"
        assert B.bwd_algorithm_for(1, 32, 16384, 16384, 128, 128, True) == "fused_query_tiles"
        assert B.bwd_algorithm_for(1, 80, 65536, 65536, 128, 128, True) == "fused_query_tiles"
        assert B.bwd_algorithm_for(4, 32, 65536, 65536, 128, 128, True) == "fused_query_tiles"
    finally:
        B.set_bwd_algorithm("auto")


def test_splitk_workspace_and_validation():
    assert B.splitk_workspace_size(1, 2, 10, 640, 64, 64, 3) >= 3 * 5 * 2 * 10 * 4
    assert B.splitk_workspace_size(1, 2, 10, 640, 64, 64, 0) == 0
    # nsplit beyond the 5 key tiles of 128 is clamped
    assert B.splitk_workspace_size(1, 2, 10, 640, 64, 64, 50) == B.splitk_workspace_size(1, 2, 10, 640, 64, 64, 5)
    lib = B.lib()
    prob = B.problem(1, 2, 10, 640, 64, 64)
    v = ctypes.c_void_p
    args = [v(16 * (k + 1)) for k in range(7)]
    assert lib.streamkl_fwd_splitk(ctypes.byref(prob), *args, 0, v(1 << 20), 1 << 30, v(0)) == B.EINVAL
    assert lib.streamkl_fwd_splitk(ctypes.byref(prob), *args, 2, v(0), 1 << 30, v(0)) == B.EINVAL
    assert lib.streamkl_fwd_splitk(ctypes.byref(prob), *args, 2, v(1 << 20), 8, v(0)) == B.EINVAL

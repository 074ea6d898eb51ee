"""Python binding of libstreamkl (the C ABI in include/streamkl.h).

Argument marshalling only: tensors are checked for dtype, device, shape and
layout, and their pointers, sizes and the current CUDA stream are passed to
the library.  Every step of the computation runs in the library's sm_100a
kernels; there is no fallback.  Importing this module fails if the library
has not been built.
"""
from __future__ import annotations

import ctypes
import re
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libstreamkl.so"
HEADER = _PKG.parent / "include" / "streamkl.h"

if not LIB_PATH.exists():
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m attention_kl_distillation_b200.build` "
        "(the CUDA library is required; there is no fallback path)")

_lib = ctypes.CDLL(str(LIB_PATH))

OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT, EDEVICE = range(6)


class Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("NQ", ctypes.c_int),
                ("NK", ctypes.c_int), ("d1", ctypes.c_int), ("d2", ctypes.c_int),
                ("causal", ctypes.c_int), ("s1", ctypes.c_float), ("s2", ctypes.c_float)]


_vp = ctypes.c_void_p
_pp = ctypes.POINTER(Problem)
_lib.streamkl_fwd.argtypes = [_pp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.streamkl_fwd.restype = ctypes.c_int
_lib.streamkl_fwd_splitk.argtypes = [_pp] + [_vp] * 7 + [ctypes.c_int, _vp, ctypes.c_size_t, _vp]
_lib.streamkl_fwd_splitk.restype = ctypes.c_int
_lib.streamkl_fwd_splitk_workspace_size.argtypes = [_pp, ctypes.c_int]
_lib.streamkl_fwd_splitk_workspace_size.restype = ctypes.c_size_t
_lib.streamkl_fwd_splitk_suggest.argtypes = [_pp]
_lib.streamkl_fwd_splitk_suggest.restype = ctypes.c_int
_lib.streamkl_bwd_workspace_size.argtypes = [_pp]
_lib.streamkl_bwd_workspace_size.restype = ctypes.c_size_t
_lib.streamkl_bwd.argtypes = [_pp] + [_vp] * 13 + [ctypes.c_size_t, _vp]
_lib.streamkl_bwd.restype = ctypes.c_int
_lib.streamkl_bwd_noalloc.argtypes = [_pp] + [_vp] * 13
_lib.streamkl_bwd_noalloc.restype = ctypes.c_int
_lib.streamkl_bwd_noalloc_scratch_bytes.argtypes = []
_lib.streamkl_bwd_noalloc_scratch_bytes.restype = ctypes.c_size_t
_lib.streamkl_status_string.argtypes = [ctypes.c_int]
_lib.streamkl_status_string.restype = ctypes.c_char_p
_lib.streamkl_query_device_status.argtypes = [_vp]
_lib.streamkl_query_device_status.restype = ctypes.c_int
_lib.streamkl_set_wait_limit_ms.argtypes = [ctypes.c_int]
_lib.streamkl_set_wait_limit_ms.restype = ctypes.c_int
_lib.streamkl_abi_version.restype = ctypes.c_int
_lib.streamkl_debug_inject.argtypes = [ctypes.c_int]
_lib.streamkl_debug_inject.restype = ctypes.c_int
_lib.streamkl_set_bwd_algorithm.argtypes = [ctypes.c_int]
_lib.streamkl_set_bwd_algorithm.restype = ctypes.c_int
_lib.streamkl_bwd_algorithm_for.argtypes = [_pp]
_lib.streamkl_bwd_algorithm_for.restype = ctypes.c_int
_lib.streamkl_launch_count.restype = ctypes.c_uint64


class StreamKLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/streamkl.h declares."""
    text = HEADER.read_text()
    return sorted(set(re.findall(r"\b(streamkl_[a-z_0-9]+)\s*\(", text)))


def status_string(st: int) -> str:
    return _lib.streamkl_status_string(int(st)).decode()


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(_lib.streamkl_launch_count())


BWD_ALGOS = {"auto": 0, "fused": 1, "split": 2, "fused_key_tiles": 3, "fused_query_tiles": 4,
             "fused_sides": 5}


def set_bwd_algorithm(name: str) -> None:
    """Process-wide backward algorithm: "auto", "fused", "split", "fused_key_tiles",
    "fused_query_tiles" or "fused_sides" (see streamkl_bwd_algorithm in include/streamkl.h)."""
    st = _lib.streamkl_set_bwd_algorithm(BWD_ALGOS[name])
    if st != OK:
        raise StreamKLError(st, "streamkl_set_bwd_algorithm")


def bwd_algorithm_for(B, H, NQ, NK, d1, d2, causal=False) -> str:
    prob = problem(B, H, NQ, NK, d1, d2, causal)
    code = _lib.streamkl_bwd_algorithm_for(ctypes.byref(prob))
    return {v: k for k, v in BWD_ALGOS.items()}[code]


def debug_inject(mode: int) -> None:
    """Arm (1) or disarm (0) the one-shot stalled-producer fault of the next forward."""
    st = _lib.streamkl_debug_inject(int(mode))
    if st != OK:
        raise StreamKLError(st, "streamkl_debug_inject")


def set_wait_limit_ms(ms: int) -> None:
    st = _lib.streamkl_set_wait_limit_ms(int(ms))
    if st != OK:
        raise StreamKLError(st, "streamkl_set_wait_limit_ms")


def query_device_status(stream: torch.cuda.Stream | None = None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return _lib.streamkl_query_device_status(_vp(s.cuda_stream))


def problem(B, H, NQ, NK, d1, d2, causal=False, s1=None, s2=None) -> Problem:
    return Problem(int(B), int(H), int(NQ), int(NK), int(d1), int(d2), int(bool(causal)),
                   float(s1) if s1 is not None else 0.0, float(s2) if s2 is not None else 0.0)


def _ptr(t):
    return _vp(t.data_ptr()) if t is not None else _vp(0)


def _check_qk(Q1, K1, Q2, K2, require_cuda=True):
    for n, t in (("Q1", Q1), ("K1", K1), ("Q2", Q2), ("K2", K2)):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CUDA bf16 tensor [B, H, N, d]")
    B, H, NQ, d1 = Q1.shape
    NK = K1.shape[2]
    d2 = Q2.shape[3]
    if K1.shape != (B, H, NK, d1) or Q2.shape != (B, H, NQ, d2) or K2.shape != (B, H, NK, d2):
        raise ValueError("inconsistent shapes of Q1, K1, Q2, K2")
    if len({Q1.device, K1.device, Q2.device, K2.device}) != 1:
        raise ValueError("inputs must be on one device")
    if require_cuda and not Q1.is_cuda:
        raise ValueError("inputs must be CUDA tensors")
    return B, H, NQ, NK, d1, d2


def _check_bwd(dL, Q1, K1, Q2, K2, L, LSE1, LSE2, out, require_cuda=True):
    """Checks every tensor the backward entry points receive; the library sees only raw
    pointers, so a wrong dtype, shape, layout or device must be refused here.  `out`
    holds the four gradient tensors or None entries (None skips that gradient)."""
    dims = _check_qk(Q1, K1, Q2, K2, require_cuda=False)
    B, H, NQ = dims[:3]
    for n, t in (("dL", dL), ("L", L), ("LSE1", LSE1), ("LSE2", LSE2)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or t.shape != (B, H, NQ) \
                or not t.is_contiguous() or t.device != Q1.device:
            raise ValueError(f"{n} must be a contiguous fp32 tensor [B, H, NQ] on the inputs' device")
    if out is not None:
        if len(out) != 4:
            raise ValueError("out must hold four entries: dQ1, dK1, dQ2, dK2 (None skips one)")
        for n, o, t in zip(("dQ1", "dK1", "dQ2", "dK2"), out, (Q1, K1, Q2, K2)):
            if o is not None and (not isinstance(o, torch.Tensor) or o.shape != t.shape
                                  or o.dtype != torch.bfloat16 or not o.is_contiguous()
                                  or o.device != t.device):
                raise ValueError(f"gradient output {n} must match its input "
                                 f"(bf16, contiguous, shape {tuple(t.shape)}, same device)")
        if all(o is None for o in out):
            raise ValueError("out asks for no gradient")
    if require_cuda and not Q1.is_cuda:
        raise ValueError("inputs must be CUDA tensors")
    return dims


def _stream(device):
    return _vp(torch.cuda.current_stream(device).cuda_stream)


def fwd(Q1, K1, Q2, K2, causal=False, s1=None, s2=None, out=None):
    """L, LSE1, LSE2 (fp32 [B, H, NQ]) via streamkl_fwd on the current stream."""
    B, H, NQ, NK, d1, d2 = _check_qk(Q1, K1, Q2, K2)
    prob = problem(B, H, NQ, NK, d1, d2, causal, s1, s2)
    if out is None:
        out = tuple(torch.empty((B, H, NQ), dtype=torch.float32, device=Q1.device)
                    for _ in range(3))
    L, A, Bv = out
    with torch.cuda.device(Q1.device):
        st = _lib.streamkl_fwd(ctypes.byref(prob), _ptr(Q1), _ptr(K1), _ptr(Q2), _ptr(K2),
                               _ptr(L), _ptr(A), _ptr(Bv), _stream(Q1.device))
    if st != OK:
        raise StreamKLError(st, "streamkl_fwd")
    return L, A, Bv


def splitk_workspace_size(B, H, NQ, NK, d1, d2, nsplit, causal=False) -> int:
    prob = problem(B, H, NQ, NK, d1, d2, causal)
    return int(_lib.streamkl_fwd_splitk_workspace_size(ctypes.byref(prob), int(nsplit)))


def fwd_splitk(Q1, K1, Q2, K2, causal=False, s1=None, s2=None, nsplit=None, workspace=None,
               out=None):
    """streamkl_fwd_splitk: the forward with the keys split across CTAs (small N_Q).
    nsplit=None asks the library for a split that fills the device."""
    B, H, NQ, NK, d1, d2 = _check_qk(Q1, K1, Q2, K2)
    prob = problem(B, H, NQ, NK, d1, d2, causal, s1, s2)
    with torch.cuda.device(Q1.device):
        if nsplit is None:
            nsplit = int(_lib.streamkl_fwd_splitk_suggest(ctypes.byref(prob)))
            if nsplit < 1:
                raise StreamKLError(EINVAL, "streamkl_fwd_splitk_suggest")
        need = int(_lib.streamkl_fwd_splitk_workspace_size(ctypes.byref(prob), int(nsplit)))
        if workspace is None:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=Q1.device)
        if out is None:
            out = tuple(torch.empty((B, H, NQ), dtype=torch.float32, device=Q1.device)
                        for _ in range(3))
        L, A, Bv = out
        st = _lib.streamkl_fwd_splitk(ctypes.byref(prob), _ptr(Q1), _ptr(K1), _ptr(Q2), _ptr(K2),
                                      _ptr(L), _ptr(A), _ptr(Bv), int(nsplit), _ptr(workspace),
                                      ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                      _stream(Q1.device))
    if st != OK:
        raise StreamKLError(st, "streamkl_fwd_splitk")
    return L, A, Bv


def splitk_suggest(B, H, NQ, NK, d1, d2, causal=False) -> int:
    """streamkl_fwd_splitk_suggest for the current device."""
    prob = problem(B, H, NQ, NK, d1, d2, causal)
    n = int(_lib.streamkl_fwd_splitk_suggest(ctypes.byref(prob)))
    if n < 1:
        raise StreamKLError(EINVAL, "streamkl_fwd_splitk_suggest")
    return n


def workspace_size(B, H, NQ, NK, d1, d2, causal=False) -> int:
    prob = problem(B, H, NQ, NK, d1, d2, causal)
    return int(_lib.streamkl_bwd_workspace_size(ctypes.byref(prob)))


def bwd(dL, Q1, K1, Q2, K2, L, LSE1, LSE2, causal=False, s1=None, s2=None,
        need=(True, True, True, True), workspace=None, out=None):
    """dQ1, dK1, dQ2, dK2 (bf16, None where not needed) via streamkl_bwd.

    ``out`` may pass preallocated gradient tensors (None entries are skipped);
    ``workspace`` a preallocated device buffer of at least ``workspace_size`` bytes."""
    B, H, NQ, NK, d1, d2 = _check_bwd(dL, Q1, K1, Q2, K2, L, LSE1, LSE2, out)
    prob = problem(B, H, NQ, NK, d1, d2, causal, s1, s2)
    if out is not None:
        outs = list(out)
    else:
        outs = [torch.empty_like(t) if want else None
                for t, want in zip((Q1, K1, Q2, K2), need)]
    ws_bytes = int(_lib.streamkl_bwd_workspace_size(ctypes.byref(prob)))
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q1.device)
    elif workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small")
    with torch.cuda.device(Q1.device):
        st = _lib.streamkl_bwd(ctypes.byref(prob), _ptr(dL), _ptr(Q1), _ptr(K1), _ptr(Q2),
                               _ptr(K2), _ptr(L), _ptr(LSE1), _ptr(LSE2), *map(_ptr, outs),
                               _ptr(workspace), ctypes.c_size_t(workspace.numel()
                                                                * workspace.element_size()),
                               _stream(Q1.device))
    if st != OK:
        raise StreamKLError(st, "streamkl_bwd")
    return tuple(outs)


# Size of the static device scratch streamkl_bwd_noalloc uses, as the library reports it.
NOALLOC_SCRATCH_BYTES = int(_lib.streamkl_bwd_noalloc_scratch_bytes())


def bwd_noalloc(dL, Q1, K1, Q2, K2, L, LSE1, LSE2, out, causal=False, s1=None, s2=None):
    """streamkl_bwd_noalloc: the backward without a caller workspace, for callers that
    cannot allocate device memory.  ``out`` holds four preallocated bf16 gradients (None
    skips one); the library's own static scratch (NOALLOC_SCRATCH_BYTES per GPU) replaces
    the workspace.  Every tensor is checked as in ``bwd`` before the call."""
    if out is None:
        raise ValueError("bwd_noalloc needs preallocated gradient outputs")
    B, H, NQ, NK, d1, d2 = _check_bwd(dL, Q1, K1, Q2, K2, L, LSE1, LSE2, out)
    prob = problem(B, H, NQ, NK, d1, d2, causal, s1, s2)
    with torch.cuda.device(Q1.device):
        st = _lib.streamkl_bwd_noalloc(ctypes.byref(prob), _ptr(dL), _ptr(Q1), _ptr(K1), _ptr(Q2),
                                       _ptr(K2), _ptr(L), _ptr(LSE1), _ptr(LSE2), *map(_ptr, out),
                                       _stream(Q1.device))
    if st != OK:
        raise StreamKLError(st, "streamkl_bwd_noalloc")
    return tuple(out)


class _StreamKLFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, Q1, K1, Q2, K2, causal, s1, s2):
        L, LSE1, LSE2 = fwd(Q1, K1, Q2, K2, causal, s1, s2)
        ctx.save_for_backward(Q1, K1, Q2, K2, L, LSE1, LSE2)
        ctx.cfg = (causal, s1, s2)
        return L

    @staticmethod
    def backward(ctx, dL):
        Q1, K1, Q2, K2, L, LSE1, LSE2 = ctx.saved_tensors
        causal, s1, s2 = ctx.cfg
        need = tuple(bool(x) for x in ctx.needs_input_grad[:4])
        if not any(need):
            return (None,) * 7
        grads = bwd(dL.float().contiguous(), Q1, K1, Q2, K2, L, LSE1, LSE2, causal, s1, s2,
                    need=need)
        return (*grads, None, None, None)


def streamkl(Q1, K1, Q2, K2, causal=False, s1=None, s2=None):
    """Row-wise KL(P1 || P2) [B, H, NQ] (fp32) with autograd support."""
    return _StreamKLFunction.apply(Q1, K1, Q2, K2, causal, s1, s2)

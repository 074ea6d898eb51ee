"""fp64 CPU oracle for the row-wise attention KL divergence -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

This file is argument marshalling around ``streamkl_oracle.c`` (ctypes) plus
its build step.  The arithmetic, and the passages it follows on the StreamKL
summary page ("Metodologia" sections 1 and 2: the row-wise KL definition,
LSE_t = m_t + log l_t, regeneration P = exp(S - LSE), both gradient
configurations, and the stable log ratio of "Stabilita Numerica"), are
documented in the C file.

Inputs are numpy arrays shaped [B, H, N, d] (or [BH, N, d]), either ``uint16``
holding bf16 bit patterns (decoded exactly) or ``float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "streamkl_oracle.c"
_BUILD = _HERE / "_build"

_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double
_vp = ctypes.c_void_p


def lib_path(mutant: int = 0, out_dir: Path | None = None) -> Path:
    d = Path(out_dir) if out_dir is not None else _BUILD
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return d / name


def build(mutant: int = 0, out_dir: Path | None = None, force: bool = False) -> Path:
    """Compile the oracle with gcc.  ``mutant`` > 0 plants a known mistake."""
    out = lib_path(mutant, out_dir)
    if out.exists() and not force and out.stat().st_mtime >= _SRC.stat().st_mtime:
        return out
    out.parent.mkdir(parents=True, exist_ok=True)
    tmp = out.with_suffix(f".tmp{os.getpid()}.so")
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-pthread",
           f"-DORACLE_MUTANT={int(mutant)}", str(_SRC), "-o", str(tmp), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _as_input(x):
    a = np.asarray(x)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a), 1
    if a.dtype == np.float64:
        return np.ascontiguousarray(a), 0
    raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float64, got {a.dtype}")


def _shape(a):
    if a.ndim == 4:
        return a.shape[0] * a.shape[1], a.shape[2], a.shape[3]
    if a.ndim == 3:
        return a.shape
    raise ValueError("inputs must be [B,H,N,d] or [BH,N,d]")


class Oracle:
    """Handle on one build of the oracle library."""

    def __init__(self, path: Path | None = None, mutant: int = 0):
        if path is None:
            path = build(mutant)
        self.path = Path(path)
        lib = ctypes.CDLL(str(self.path))
        common = [_i64, _i64, _i64, _int, _int, _int, _dbl, _dbl, _int, _vp, _vp, _vp, _vp]
        lib.oracle_fwd_rows.argtypes = common + [_i64, _vp, _vp, _vp, _vp, _int]
        lib.oracle_fwd_rows.restype = _int
        lib.oracle_bwd_rows.argtypes = common + [_i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int]
        lib.oracle_bwd_rows.restype = _int
        lib.oracle_bwd_heads.argtypes = common + [_i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                  _vp, _int]
        lib.oracle_bwd_heads.restype = _int
        lib.oracle_mutant_id.restype = _int
        self.lib = lib
        self.mutant = lib.oracle_mutant_id()

    # -- helpers -----------------------------------------------------------
    def _prep(self, Q1, K1, Q2, K2, s1, s2):
        (q1, t1), (k1, t2), (q2, t3), (k2, t4) = map(_as_input, (Q1, K1, Q2, K2))
        if len({t1, t2, t3, t4}) != 1:
            raise TypeError("all four inputs must share one dtype")
        BH, NQ, d1 = _shape(q1)
        BHk, NK, d1k = _shape(k1)
        BH2, NQ2, d2 = _shape(q2)
        BHk2, NK2, d2k = _shape(k2)
        if not (BH == BHk == BH2 == BHk2 and NQ == NQ2 and NK == NK2 and d1 == d1k and d2 == d2k):
            raise ValueError("inconsistent input shapes")
        s1 = float(s1) if s1 is not None else 1.0 / np.sqrt(d1)
        s2 = float(s2) if s2 is not None else 1.0 / np.sqrt(d2)
        return (q1, k1, q2, k2), t1, (BH, NQ, NK, d1, d2), s1, s2

    @staticmethod
    def _ptr(a):
        return a.ctypes.data_as(_vp)

    # -- forward -------------------------------------------------------------
    def fwd_rows(self, Q1, K1, Q2, K2, rows, causal=False, s1=None, s2=None, nthreads=None):
        """L, LSE1, LSE2 (float64) for the listed rows; rows is an [n, 2] array of (bh, i)."""
        arrs, isbf, (BH, NQ, NK, d1, d2), s1, s2 = self._prep(Q1, K1, Q2, K2, s1, s2)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
        n = rows.shape[0]
        L = np.empty(n, np.float64)
        A = np.empty(n, np.float64)
        Bv = np.empty(n, np.float64)
        st = self.lib.oracle_fwd_rows(BH, NQ, NK, d1, d2, int(bool(causal)), s1, s2, isbf,
                                      *map(self._ptr, arrs), n, self._ptr(rows), self._ptr(L),
                                      self._ptr(A), self._ptr(Bv),
                                      nthreads or _host_threads())
        if st != 0:
            raise RuntimeError(f"oracle_fwd_rows failed with status {st}")
        return L, A, Bv

    def fwd_all(self, Q1, K1, Q2, K2, causal=False, s1=None, s2=None, nthreads=None):
        """Every row; outputs shaped [BH, NQ]."""
        q1 = np.asarray(Q1)
        BH, NQ, _ = _shape(q1)
        bh, i = np.meshgrid(np.arange(BH), np.arange(NQ), indexing="ij")
        rows = np.stack([bh.ravel(), i.ravel()], axis=1)
        L, A, Bv = self.fwd_rows(Q1, K1, Q2, K2, rows, causal, s1, s2, nthreads)
        return L.reshape(BH, NQ), A.reshape(BH, NQ), Bv.reshape(BH, NQ)

    # -- backward ------------------------------------------------------------
    def bwd_rows(self, Q1, K1, Q2, K2, rows, g, causal=False, s1=None, s2=None, nthreads=None):
        """L, LSE1, LSE2, dQ1 [n, d1], dQ2 [n, d2] for the listed rows with weights g [n]."""
        arrs, isbf, (BH, NQ, NK, d1, d2), s1, s2 = self._prep(Q1, K1, Q2, K2, s1, s2)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
        n = rows.shape[0]
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (n,)))
        L = np.empty(n); A = np.empty(n); Bv = np.empty(n)
        dq1 = np.empty((n, d1)); dq2 = np.empty((n, d2))
        st = self.lib.oracle_bwd_rows(BH, NQ, NK, d1, d2, int(bool(causal)), s1, s2, isbf,
                                      *map(self._ptr, arrs), n, self._ptr(rows), self._ptr(g),
                                      self._ptr(L), self._ptr(A), self._ptr(Bv), self._ptr(dq1),
                                      self._ptr(dq2), nthreads or _host_threads())
        if st != 0:
            raise RuntimeError(f"oracle_bwd_rows failed with status {st}")
        return L, A, Bv, dq1, dq2

    def bwd_heads(self, Q1, K1, Q2, K2, heads, g, causal=False, s1=None, s2=None, nthreads=None):
        """Whole-head backward.  g is [len(heads), NQ].  Returns a dict of float64 arrays."""
        arrs, isbf, (BH, NQ, NK, d1, d2), s1, s2 = self._prep(Q1, K1, Q2, K2, s1, s2)
        heads = np.ascontiguousarray(np.asarray(heads, dtype=np.int64).reshape(-1))
        nh = heads.shape[0]
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (nh, NQ)))
        out = {
            "L": np.empty((nh, NQ)), "LSE1": np.empty((nh, NQ)), "LSE2": np.empty((nh, NQ)),
            "dQ1": np.empty((nh, NQ, d1)), "dK1": np.empty((nh, NK, d1)),
            "dQ2": np.empty((nh, NQ, d2)), "dK2": np.empty((nh, NK, d2)),
        }
        st = self.lib.oracle_bwd_heads(
            BH, NQ, NK, d1, d2, int(bool(causal)), s1, s2, isbf, *map(self._ptr, arrs), nh,
            self._ptr(heads), self._ptr(g), self._ptr(out["L"]), self._ptr(out["LSE1"]),
            self._ptr(out["LSE2"]), self._ptr(out["dQ1"]), self._ptr(out["dK1"]),
            self._ptr(out["dQ2"]), self._ptr(out["dK2"]), nthreads or _host_threads())
        if st != 0:
            raise RuntimeError(f"oracle_bwd_heads failed with status {st}")
        return out


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The oracle (no planted mistake), built on first use."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle(build(0))
    return _DEFAULT


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bf16 bit patterns to float64 (for tests that perturb inputs)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)

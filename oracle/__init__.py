"""ctypes binding of the plain fp64 Muon oracle (``muon_oracle.cpp``), and the same method
with library matrix products for the largest shapes (``ns_blas.py``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The CUDA library never
loads it, and this module never loads the CUDA library.

``newton_schulz`` and ``muon_step`` take an optional ``lib``: a loaded C library (the plain-loop
oracle, or a deliberately broken copy of it in the mutation tests), or a Python oracle module
such as ``oracle.ns_blas`` (marked by ``PY_ORACLE = True``), which is then called directly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "muon_oracle.cpp")
LIB = os.path.join(HERE, "libmuon_oracle.so")

_lib = None


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Compile the oracle with g++ (-O3, portable x86-64 code, no -march)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["g++", "-O3", "-std=c++17", "-fPIC", "-shared", "-pthread", src, "-o", out]
        subprocess.check_call(cmd)
    return out


def load(path: Optional[str] = None):
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    dp = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_newton_schulz.restype = ctypes.c_int
    lib.oracle_newton_schulz.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, dp,
                                         ctypes.c_int, ctypes.c_double, ctypes.c_int]
    lib.oracle_muon_step.restype = ctypes.c_int
    lib.oracle_muon_step.argtypes = [ctypes.c_int, ctypes.POINTER(dp), ctypes.POINTER(dp),
                                     ctypes.POINTER(dp), i64p, i64p, ctypes.c_double, ctypes.c_double,
                                     ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int, dp,
                                     ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.POINTER(dp)]
    lib.oracle_adamw_step.restype = ctypes.c_int
    lib.oracle_adamw_step.argtypes = [ctypes.c_int, ctypes.POINTER(dp), ctypes.POINTER(dp), ctypes.POINTER(dp),
                                      ctypes.POINTER(dp), i64p, ctypes.c_int64, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_double, ctypes.c_double]
    if path is None:
        _lib = lib
    return lib


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _coeff_array(coeffs: Sequence[Tuple[float, float, float]]) -> np.ndarray:
    return np.ascontiguousarray(np.array(coeffs, dtype=np.float64).reshape(-1))


def newton_schulz(G: np.ndarray, coeffs: Sequence[Tuple[float, float, float]], zero_center: bool = False,
                  eps: float = 1e-7, nthreads: int = 0, lib=None) -> np.ndarray:
    """O = NewtonSchulz(G) in fp64; G is rows x cols."""
    if getattr(lib, "PY_ORACLE", False):
        return lib.newton_schulz(G, coeffs, zero_center=zero_center, eps=eps)
    lib = lib or load()
    G = np.ascontiguousarray(G, dtype=np.float64)
    O = np.empty_like(G)
    co = _coeff_array(coeffs) if len(coeffs) else np.zeros(3)
    rc = lib.oracle_newton_schulz(_dptr(G), _dptr(O), G.shape[0], G.shape[1], len(coeffs), _dptr(co),
                                  int(zero_center), eps, nthreads)
    if rc != 0:
        raise ValueError("oracle_newton_schulz rejected its arguments")
    return O


def muon_step(params: List[np.ndarray], grads: List[Optional[np.ndarray]], momentum: List[np.ndarray],
              lr: float, mu: float, nesterov: bool, weight_decay: float, rms_mode: int,
              coeffs: Sequence[Tuple[float, float, float]], zero_center: bool, eps: float,
              nthreads: int = 0, want_O: bool = False, lib=None):
    """One Muon step in fp64; params and momentum (float64, C-contiguous) are updated in place.
    Returns the list of O matrices when want_O."""
    if getattr(lib, "PY_ORACLE", False):
        return lib.muon_step(params, grads, momentum, lr=lr, mu=mu, nesterov=nesterov,
                             weight_decay=weight_decay, rms_mode=rms_mode, coeffs=coeffs,
                             zero_center=zero_center, eps=eps, want_O=want_O)
    lib = lib or load()
    n = len(params)
    for a in list(params) + list(momentum):
        assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    g64 = [None if g is None else np.ascontiguousarray(g, dtype=np.float64) for g in grads]
    dp = ctypes.POINTER(ctypes.c_double)
    P = (dp * n)(*[_dptr(p) for p in params])
    G = (dp * n)(*[(_dptr(g) if g is not None else dp()) for g in g64])
    M = (dp * n)(*[_dptr(m) for m in momentum])
    rows = np.array([p.shape[0] for p in params], dtype=np.int64)
    cols = np.array([p.shape[1] for p in params], dtype=np.int64)
    outs = [np.empty_like(p) for p in params] if want_O else None
    O = (dp * n)(*[_dptr(o) for o in outs]) if want_O else None
    co = _coeff_array(coeffs) if len(coeffs) else np.zeros(3)
    rc = lib.oracle_muon_step(n, P, G, M, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                              cols.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), lr, mu, int(nesterov),
                              weight_decay, rms_mode, len(coeffs), _dptr(co), int(zero_center), eps,
                              nthreads, O)
    if rc != 0:
        raise ValueError("oracle_muon_step rejected its arguments")
    return outs


def adamw_step(params: List[np.ndarray], grads: List[Optional[np.ndarray]], exp_avg: List[np.ndarray],
               exp_avg_sq: List[np.ndarray], step: int, lr: float, beta1: float, beta2: float, eps: float,
               weight_decay: float, lib=None) -> None:
    """One AdamW step in fp64 (any shapes; arrays are updated in place). `step` is the step count
    after this step (1 for the first)."""
    lib = lib or load()
    n = len(params)
    for a in list(params) + list(exp_avg) + list(exp_avg_sq):
        assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    g64 = [None if g is None else np.ascontiguousarray(g, dtype=np.float64) for g in grads]
    dp = ctypes.POINTER(ctypes.c_double)
    P = (dp * n)(*[_dptr(p) for p in params])
    G = (dp * n)(*[(_dptr(g) if g is not None else dp()) for g in g64])
    M = (dp * n)(*[_dptr(m) for m in exp_avg])
    V = (dp * n)(*[_dptr(v) for v in exp_avg_sq])
    numel = np.array([p.size for p in params], dtype=np.int64)
    rc = lib.oracle_adamw_step(n, P, G, M, V, numel.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), step, lr,
                               beta1, beta2, eps, weight_decay)
    if rc != 0:
        raise ValueError("oracle_adamw_step rejected its arguments")

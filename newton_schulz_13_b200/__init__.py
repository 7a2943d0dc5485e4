"""Python binding of libmuon.so, the sm_100a Muon optimizer step.

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
There is no CPU or PyTorch fallback; if the library is missing, importing this package raises.

    import newton_schulz_13_b200 as ns
    ns.muon_step(params, grads, momentum, lr=0.02, mu=0.95)     # lists of CUDA tensors
    X = ns.ns_orthogonalize(G, steps=5)                          # one matrix
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmuon.so")

BF16, FP32 = 0, 1
PREC_BF16, PREC_FP32 = 0, 1
RMS_ONE, RMS_SQRT_MAX1_ROWS_OVER_COLS = 0, 1
OK, WARN_NONFINITE = 0, 1
ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = -1, -2, -3, -4, -5
KC_CENTER, KC_PROLOGUE, KC_NORM, KC_GEMM, KC_EPILOGUE, KC_ADAMW = 0, 1, 2, 3, 4, 5
KC_GEMM_GRAM, KC_GEMM_POLY, KC_GEMM_UPDATE, KC_COUNT = 6, 7, 8, 9
KC_NAMES = ["center", "prologue", "norm", "gemm", "epilogue", "adamw", "gemm_gram", "gemm_poly", "gemm_update"]
MAX_NS_STEPS = 64

QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)

EXPORTS = ["muon_ns_orthogonalize", "muon_step", "muon_adamw_step", "muon_last_error",
           "muon_check_status", "muon_release_workspace", "muon_profile_enable", "muon_profile_read",
           "muon_launch_count", "muon_version", "muon_set_wave_elements", "muon_set_wait_limit_ns", "muon_set_chained_launch"]


class MuonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class Coeffs(ctypes.Structure):
    _fields_ = [("a", ctypes.c_float), ("b", ctypes.c_float), ("c", ctypes.c_float)]


def _load() -> ctypes.CDLL:
    # the library is built in-tree from csrc/ with nvcc when it is missing or older than its
    # sources; there is no fallback implementation if that fails
    from . import build as _build
    if _build.stale():
        try:
            _build.build()
        except Exception as e:  # noqa: BLE001
            raise ImportError(f"{LIB_PATH} is missing or out of date and building it failed ({e}); "
                              "there is no fallback implementation") from e
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing (there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i64p = ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)
    vpp = ctypes.POINTER(ctypes.c_void_p)
    lib.muon_ns_orthogonalize.restype = ctypes.c_int
    lib.muon_ns_orthogonalize.argtypes = [vp, ctypes.c_int, vp, ctypes.c_int, i64, i64, ctypes.c_int,
                                          ctypes.POINTER(Coeffs), ctypes.c_int, ctypes.c_float,
                                          ctypes.c_int, vp]
    lib.muon_step.restype = ctypes.c_int
    lib.muon_step.argtypes = [ctypes.c_int, vpp, vpp, ctypes.c_int, vpp, i64p, i64p, ctypes.c_float,
                              ctypes.c_float, ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                              ctypes.POINTER(Coeffs), ctypes.c_int, ctypes.c_float, ctypes.c_int, vp]
    lib.muon_adamw_step.restype = ctypes.c_int
    lib.muon_adamw_step.argtypes = [ctypes.c_int, vpp, vpp, ctypes.c_int, vpp, vpp, i64p, ctypes.c_int64,
                                    ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                    ctypes.c_float, vp]
    lib.muon_last_error.restype = ctypes.c_char_p
    lib.muon_last_error.argtypes = []
    lib.muon_check_status.restype = ctypes.c_int
    lib.muon_check_status.argtypes = [vp]
    lib.muon_release_workspace.restype = ctypes.c_int
    lib.muon_set_wave_elements.restype = ctypes.c_int
    lib.muon_set_wave_elements.argtypes = [ctypes.c_int64]
    lib.muon_set_wait_limit_ns.restype = ctypes.c_int
    lib.muon_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.muon_set_chained_launch.restype = ctypes.c_int
    lib.muon_set_chained_launch.argtypes = [ctypes.c_int]
    lib.muon_profile_enable.restype = ctypes.c_int
    lib.muon_profile_enable.argtypes = [ctypes.c_int]
    lib.muon_profile_read.restype = ctypes.c_int
    dp = ctypes.POINTER(ctypes.c_double)
    lib.muon_profile_read.argtypes = [i64p, dp, dp, dp]
    lib.muon_launch_count.restype = ctypes.c_int64
    lib.muon_version.restype = ctypes.c_int
    return lib


lib = _load()


def last_error() -> str:
    return lib.muon_last_error().decode()


def _check(rc: int) -> int:
    if rc < 0:
        raise MuonError(rc, last_error())
    return rc


def _coeff_array(steps: int, coeffs: Optional[Sequence[Tuple[float, float, float]]]):
    if coeffs is None:
        return None
    if len(coeffs) != steps:
        raise ValueError(f"need {steps} coefficient triples, got {len(coeffs)}")
    arr = (Coeffs * max(1, steps))()
    for k, (a, b, c) in enumerate(coeffs):
        arr[k] = Coeffs(a, b, c)
    return arr


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        if not torch.cuda.is_available():
            return None   # the library reports the missing device itself
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _prec_code(prec) -> int:
    if prec in ("bf16", PREC_BF16):
        return PREC_BF16
    if prec in ("fp32", PREC_FP32):
        return PREC_FP32
    raise ValueError(f"prec must be 'bf16' or 'fp32', got {prec!r}")


def ns_orthogonalize(G, X=None, steps: int = 5, coeffs=None, zero_center: bool = False,
                     eps: float = 1e-7, prec="bf16", stream=None, out_dtype=None):
    """X = NewtonSchulz(G) for one 2-D CUDA tensor G (bf16 or fp32, contiguous)."""
    import torch
    if G.dim() != 2 or not G.is_contiguous():
        raise ValueError("G must be a contiguous 2-D tensor")
    if X is None:
        X = torch.empty(G.shape, dtype=out_dtype or G.dtype, device=G.device)
    co = _coeff_array(steps, coeffs)
    _check(lib.muon_ns_orthogonalize(G.data_ptr(), _dtype_code(G), X.data_ptr(), _dtype_code(X),
                                     G.shape[0], G.shape[1], steps, co, int(zero_center), eps,
                                     _prec_code(prec), _stream_handle(stream)))
    return X


def muon_step(params: List, grads: List, momentum: List, lr: float = 0.02, mu: float = 0.95,
              nesterov: bool = True, weight_decay: float = 0.0, rms_scale: int = RMS_ONE,
              steps: int = 5, coeffs=None, zero_center: bool = False, eps: float = 1e-7,
              prec="bf16", stream=None) -> None:
    """One Muon step over lists of CUDA tensors (params and momentum fp32; grads bf16 or fp32,
    all of one dtype; a None grad skips its matrix)."""
    n = len(params)
    if not (len(grads) == len(momentum) == n):
        raise ValueError("params, grads and momentum must have the same length")
    g_dtype = None
    for g in grads:
        if g is not None:
            code = _dtype_code(g)
            if g_dtype is not None and code != g_dtype:
                raise TypeError("all gradients must share one dtype")
            g_dtype = code
    if g_dtype is None:
        return
    VP = ctypes.c_void_p * max(1, n)
    P = VP(*[p.data_ptr() for p in params])
    G = VP(*[(g.data_ptr() if g is not None else None) for g in grads])
    M = VP(*[m.data_ptr() for m in momentum])
    I64 = ctypes.c_int64 * max(1, n)
    rows = I64(*[p.shape[0] for p in params])
    cols = I64(*[p.shape[1] for p in params])
    co = _coeff_array(steps, coeffs)
    _check(lib.muon_step(n, ctypes.cast(P, ctypes.POINTER(ctypes.c_void_p)),
                         ctypes.cast(G, ctypes.POINTER(ctypes.c_void_p)), g_dtype,
                         ctypes.cast(M, ctypes.POINTER(ctypes.c_void_p)), rows, cols, lr, mu,
                         int(nesterov), weight_decay, int(rms_scale), steps, co, int(zero_center), eps,
                         _prec_code(prec), _stream_handle(stream)))


def adamw_step(params: List, grads: List, exp_avg: List, exp_avg_sq: List, step: int, lr: float = 1e-3,
               beta1: float = 0.9, beta2: float = 0.95, eps: float = 1e-8, weight_decay: float = 0.0,
               stream=None) -> None:
    """One AdamW step over lists of contiguous CUDA tensors of any shape (params and moments fp32;
    grads bf16 or fp32, all of one dtype; a None grad skips its tensor). `step` is the step count
    after this step (1 for the first)."""
    n = len(params)
    if not (len(grads) == len(exp_avg) == len(exp_avg_sq) == n):
        raise ValueError("params, grads, exp_avg and exp_avg_sq must have the same length")
    g_dtype = None
    for g in grads:
        if g is not None:
            code = _dtype_code(g)
            if g_dtype is not None and code != g_dtype:
                raise TypeError("all gradients must share one dtype")
            g_dtype = code
    if g_dtype is None:
        return
    VP = ctypes.c_void_p * max(1, n)
    cast = lambda a: ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))
    P = VP(*[p.data_ptr() for p in params])
    G = VP(*[(g.data_ptr() if g is not None else None) for g in grads])
    M = VP(*[m.data_ptr() for m in exp_avg])
    V = VP(*[v.data_ptr() for v in exp_avg_sq])
    N = (ctypes.c_int64 * max(1, n))(*[p.numel() for p in params])
    _check(lib.muon_adamw_step(n, cast(P), cast(G), g_dtype, cast(M), cast(V), N, step, lr, beta1, beta2,
                               eps, weight_decay, _stream_handle(stream)))


def check_status(stream=None) -> int:
    """Synchronises the stream and returns OK or WARN_NONFINITE; raises on a device timeout."""
    return _check(lib.muon_check_status(_stream_handle(stream)))


def release_workspace() -> None:
    _check(lib.muon_release_workspace())


def set_wave_elements(elements: int = 0) -> None:
    """Largest number of elements muon_step processes in one wave of launches (0: the default,
    2^29). Results do not depend on it; see muon_set_wave_elements in include/muon.h."""
    _check(lib.muon_set_wave_elements(int(elements)))


def set_chained_launch(mode: int = 1) -> None:
    """Chained launches of a wave's whole Newton-Schulz iteration: 0 never, 1 (default) for waves
    with at most 8 tiles per CTA pair per iteration, 2 for every wave of small matrices. Results
    are bit-identical; see muon_set_chained_launch in include/muon.h."""
    _check(lib.muon_set_chained_launch(int(mode)))


def set_wait_limit_ns(ns: int = 0) -> None:
    """Time limit of the waits inside the Newton-Schulz product kernels of later calls (0: the
    default, 2 s). A wait that runs out makes check_status() raise with ERR_TIMEOUT; a limit of a
    few nanoseconds exercises that path. See muon_set_wait_limit_ns in include/muon.h."""
    _check(lib.muon_set_wait_limit_ns(int(ns)))


def profile_enable(on: bool = True) -> None:
    _check(lib.muon_profile_enable(int(on)))


def profile_read():
    """Per kernel class: {name: (launches, ms, nominal_flops, executed_flops)} since the last read."""
    L = (ctypes.c_int64 * KC_COUNT)()
    T = (ctypes.c_double * KC_COUNT)()
    F = (ctypes.c_double * KC_COUNT)()
    E = (ctypes.c_double * KC_COUNT)()
    _check(lib.muon_profile_read(L, T, F, E))
    return {KC_NAMES[k]: (int(L[k]), float(T[k]), float(F[k]), float(E[k])) for k in range(KC_COUNT)}


def launch_count() -> int:
    return int(lib.muon_launch_count())


def version() -> int:
    return int(lib.muon_version())

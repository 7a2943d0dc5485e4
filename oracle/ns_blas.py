"""fp64 Newton-Schulz and Muon step with library matrix products: TEST INFRASTRUCTURE ONLY.

The same method as ``muon_oracle.cpp``, step for step in the pages' order, but every matrix
product is one numpy ``@`` (an fp64 BLAS GEMM) instead of a plain triple loop. That makes the
largest weight shapes of a Llama-8B-sized model (4096 x 14336: about 5.5e12 FLOP for five
quintic iterations) take seconds instead of hours, so the device path can be compared with an
fp64 result element by element at full size. Nothing here is blocked, fused or reordered beyond
what the library's own product does; only the order of each product's summation is the
library's.

Sources (cited by page title and section):
  * "Muon optimizer: matrix-aware LLM training", the `newtonschulz5` listing: divide by
    (||X||_F + eps), transpose when rows > cols, `steps` iterations of A = X X^T,
    B = b A + c A A, X = a X + B X, transpose back (this oracle keeps fp64 instead of the
    listing's bf16 working copy); the `Muon.step` listing: momentum buf = mu buf + (1 - mu) g,
    the Nesterov select, p -= lr * O.
  * "Muon meets Mamba" section 2.1 `zerocenter` (g minus its mean over dim 0, before the
    momentum buffer, section 4.2 order) and section 4.2 (decoupled decay p *= 1 - lr wd).
  * "AdamW vs Muon" part 3 "scaling and update": the RMS rescale by matrix shape, then lr.

Readings (the same as the C++ oracle's): Nesterov is u = mu m_t + (1 - mu) g_t; eps is added
to the norm; rows > cols is the transpose test; the RMS factor is sqrt(max(1, rows/cols)) when
requested, else 1.

Only the tests, the smoke check and the benchmark's CPU legs may import this module; it shares
no code with the CUDA library and never loads it.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

# Marks this module as an oracle implementation that the helpers in ``oracle`` (and the pins)
# call directly instead of through the C library.
PY_ORACLE = True


def center_columns(g: np.ndarray) -> np.ndarray:
    """g - 1 mean_dim0(g)^T ("Muon meets Mamba" 2.1: subtract each column's mean over dim 0)."""
    return g - g.mean(axis=0, keepdims=True)


def newton_schulz_update(u: np.ndarray, coeffs: Sequence[Tuple[float, float, float]], eps: float) -> np.ndarray:
    """The Newton-Schulz map of one update matrix u (rows x cols), in the `newtonschulz5` order."""
    X = u / (np.sqrt(np.sum(u * u)) + eps)      # X = u / (||u||_F + eps)
    tall = X.shape[0] > X.shape[1]
    if tall:                                    # iterate on the wide orientation
        X = X.T
    for a, b, c in coeffs:
        A = X @ X.T                             # A = X X^T
        B = b * A + c * (A @ A)                 # B = b A + c A A
        X = a * X + B @ X                       # X = a X + B X
    if tall:                                    # transpose back
        X = X.T
    return np.ascontiguousarray(X)


def newton_schulz(G: np.ndarray, coeffs: Sequence[Tuple[float, float, float]], zero_center: bool = False,
                  eps: float = 1e-7) -> np.ndarray:
    """O = NewtonSchulz(G) in fp64; G is rows x cols (any real dtype)."""
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2 or G.shape[0] <= 0 or G.shape[1] <= 0:
        raise ValueError("G must be a non-empty 2-D matrix")
    u = center_columns(G) if zero_center else G
    return newton_schulz_update(u, coeffs, eps)


def muon_step(params: List[np.ndarray], grads: List[Optional[np.ndarray]], momentum: List[np.ndarray],
              lr: float, mu: float, nesterov: bool, weight_decay: float, rms_mode: int,
              coeffs: Sequence[Tuple[float, float, float]], zero_center: bool, eps: float,
              want_O: bool = False):
    """One Muon step in fp64 over lists of matrices; params and momentum (float64, C-contiguous)
    are updated in place. A None gradient skips its matrix. Returns the O matrices when want_O."""
    outs = []
    for p, g, m in zip(params, grads, momentum):
        if g is None:
            outs.append(None)
            continue
        g = np.asarray(g, dtype=np.float64)
        if g.shape != p.shape or m.shape != p.shape:
            raise ValueError("params, grads and momentum must have one shape per matrix")
        if zero_center:
            g = center_columns(g)
        m *= mu                                         # m = mu m + (1 - mu) g
        m += (1.0 - mu) * g
        u = mu * m + (1.0 - mu) * g if nesterov else m  # Nesterov look-ahead, else the buffer
        O = newton_schulz_update(u, coeffs, eps)
        r, c = p.shape
        s = np.sqrt(max(1.0, r / c)) if rms_mode == 1 else 1.0
        p *= 1.0 - lr * weight_decay                    # decoupled decay, then the update
        p -= lr * s * O
        outs.append(O)
    return outs if want_O else None

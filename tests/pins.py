"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics,
computed without the oracle's own matrix iteration.

Each ``pin_*`` takes a loaded oracle library and raises AssertionError when
the oracle disagrees. They are run as tests (``test_oracle_pins.py``) and
against deliberately broken copies of the oracle source
(``test_oracle_mutants.py``), which shows that a plausible mistake anywhere in
the oracle trips at least one of them.
"""
from __future__ import annotations

import os
from typing import Dict, List, Sequence, Tuple

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> Dict[str, np.ndarray]:
    out: Dict[str, np.ndarray] = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = [s.strip() for s in line.split("=", 1)]
            rows = [[float(t) for t in r.split()] for r in val.split(";")]
            arr = np.array(rows, dtype=np.float64)
            out[key] = arr if len(rows) > 1 else arr.reshape(-1)
    return out


_COEF = read_golden("coefficients.txt")
QUINTIC = tuple(_COEF["quintic"])
CUBIC = tuple(_COEF["cubic"])
HYBRID = [tuple(_COEF["hybrid_stage1"])] * 8 + [tuple(_COEF["hybrid_stage2"])] * 2


def scalar_map(x: np.ndarray, coeffs: Sequence[Tuple[float, float, float]]) -> np.ndarray:
    """phi(x): the iteration's action on one singular value, p_k(x) = a x + b x^3 + c x^5
    composed over the iterations ("AdamW vs Muon", part 3: the iteration acts as a polynomial
    on every singular value and leaves U and V^T unchanged)."""
    x = np.asarray(x, dtype=np.float64).copy()
    for a, b, c in coeffs:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def spectral_reference(G: np.ndarray, coeffs, eps: float) -> np.ndarray:
    """U phi(Sigma / (||G||_F + eps)) V^T from LAPACK's SVD."""
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    scale = 1.0 / (np.linalg.norm(G) + eps)
    return (U * scalar_map(s * scale, coeffs)[None, :]) @ Vt


def rel(a: np.ndarray, b: np.ndarray) -> float:
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------

SHAPES = [(8, 12), (16, 40), (33, 17), (10, 10), (1, 7), (7, 1), (24, 5)]


def pin_spectral_map(lib) -> None:
    """Newton-Schulz equals U phi(Sigma) V^T for quintic, cubic and hybrid schedules."""
    for sched_name, coeffs in (("quintic", [QUINTIC] * 5), ("cubic", [CUBIC] * 5), ("hybrid", HYBRID),
                               ("quintic3", [QUINTIC] * 3)):
        for k, (r, c) in enumerate(SHAPES):
            G = rng(100 + k).standard_normal((r, c))
            got = oracle.newton_schulz(G, coeffs, eps=1e-7, lib=lib)
            want = spectral_reference(G, coeffs, 1e-7)
            assert rel(got, want) < 1e-10, (sched_name, r, c, rel(got, want))


def pin_rank_one(lib) -> None:
    """Rank-1 G = s u v^T: O = phi(s/(s+eps)) u v^T; the quintic chain from 1 is a closed form."""
    u = rng(1).standard_normal(9); u /= np.linalg.norm(u)
    v = rng(2).standard_normal(14); v /= np.linalg.norm(v)
    for s, eps in ((3.0, 0.0), (1e-7, 1e-7)):
        G = s * np.outer(u, v)
        got = oracle.newton_schulz(G, [QUINTIC] * 5, eps=eps, lib=lib)
        x0 = s / (s + eps)
        want = scalar_map(np.array([x0]), [QUINTIC] * 5)[0] * np.outer(u, v)
        assert rel(got, want) < 1e-12, (s, eps, rel(got, want))
    # the chain 1 -> 0.701 -> ... after 5 quintic iterations is 0.696436 (to 6 digits)
    G = np.outer(u, v)
    got = oracle.newton_schulz(G, [QUINTIC] * 5, eps=0.0, lib=lib)
    assert abs(float(u @ got @ v) - 0.696436) < 5e-7
    # eps = 1e-7 on a norm-1e-7 matrix halves the start value: x0 = 0.5
    G = 1e-7 * np.outer(u, v)
    got = oracle.newton_schulz(G, [QUINTIC], eps=1e-7, lib=lib)
    p = QUINTIC[0] * 0.5 + QUINTIC[1] * 0.125 + QUINTIC[2] * 0.03125
    assert abs(float(u @ got @ v) - p) < 1e-12


def pin_diagonal(lib) -> None:
    """diag(3, 4) normalises to diag(0.6, 0.8); the output is diag(phi(0.6), phi(0.8))."""
    G = np.diag([3.0, 4.0])
    for coeffs in ([QUINTIC] * 5, [CUBIC] * 5, [QUINTIC] * 1):
        got = oracle.newton_schulz(G, coeffs, eps=0.0, lib=lib)
        want = np.diag(scalar_map(np.array([0.6, 0.8]), coeffs))
        assert np.max(np.abs(got - want)) < 1e-13, (coeffs[0], got, want)
    # one quintic step on 0.6 by hand: 3.4445*0.6 - 4.775*0.216 + 2.0315*0.07776
    got = oracle.newton_schulz(G, [QUINTIC], eps=0.0, lib=lib)
    assert abs(got[0, 0] - (2.0667 - 1.0314 + 0.15796944)) < 1e-12


def pin_cubic_converges_to_polar(lib) -> None:
    """Run to convergence, the cubic iteration reaches U V^T, the orthogonal polar factor
    ("Muon meets Mamba" 2.2; "AdamW vs Muon" part 2)."""
    for k, (r, c) in enumerate([(6, 9), (9, 6), (5, 5), (12, 20)]):
        # well conditioned: singular values in [1, 2]
        Q1, _ = np.linalg.qr(rng(200 + k).standard_normal((r, r)))
        Q2, _ = np.linalg.qr(rng(300 + k).standard_normal((c, c)))
        m = min(r, c)
        S = np.zeros((r, c)); S[np.arange(m), np.arange(m)] = np.linspace(1.0, 2.0, m)
        G = Q1 @ S @ Q2.T
        got = oracle.newton_schulz(G, [CUBIC] * 60, eps=1e-7, lib=lib)
        U, _, Vt = np.linalg.svd(G, full_matrices=False)
        assert rel(got, U @ Vt) < 1e-10, (r, c, rel(got, U @ Vt))
        # the polar factor is a partial isometry: O O^T = I (wide) or O^T O = I (tall)
        gram = got @ got.T if r <= c else got.T @ got
        assert np.max(np.abs(gram - np.eye(m))) < 1e-10


def pin_quintic_band(lib) -> None:
    """Five quintic iterations push every normalised singular value above ~1.6e-3 into
    [0.68, 1.21]; smaller ones come out near 3.4445^5 x (their start)."""
    r, c = 30, 50
    Q1, _ = np.linalg.qr(rng(7).standard_normal((r, r)))
    Q2, _ = np.linalg.qr(rng(8).standard_normal((c, c)))
    sv = np.geomspace(4e-3, 1.0, r)
    assert (sv / np.linalg.norm(sv)).min() > 1.6e-3   # every normalised value above the threshold
    S = np.zeros((r, c)); S[np.arange(r), np.arange(r)] = sv
    G = Q1 @ S @ Q2.T
    O = oracle.newton_schulz(G, [QUINTIC] * 5, eps=0.0, lib=lib)
    out_sv = np.linalg.svd(O, compute_uv=False)
    assert out_sv.min() >= 0.68 and out_sv.max() <= 1.21, (out_sv.min(), out_sv.max())
    # a tiny singular value: x = 1e-6 after normalisation grows by about a^5
    S2 = S.copy(); S2[0, 0] = 1e-6 * np.linalg.norm(sv)
    G2 = Q1 @ S2 @ Q2.T
    x = 1e-6 * np.linalg.norm(sv) / np.linalg.norm(G2)
    O2 = oracle.newton_schulz(G2, [QUINTIC] * 5, eps=0.0, lib=lib)
    small = float(Q1[:, 0] @ O2 @ Q2[:, 0])
    assert abs(small / (x * QUINTIC[0] ** 5) - 1.0) < 1e-3


def pin_invariances(lib) -> None:
    """Scale, sign, transpose and orthogonal equivariance of the map."""
    co = [QUINTIC] * 5
    for k, (r, c) in enumerate([(8, 12), (12, 8), (9, 9)]):
        G = rng(400 + k).standard_normal((r, c))
        O = oracle.newton_schulz(G, co, eps=0.0, lib=lib)
        assert rel(oracle.newton_schulz(37.5 * G, co, eps=0.0, lib=lib), O) < 1e-12
        assert rel(oracle.newton_schulz(-G, co, eps=0.0, lib=lib), -O) < 1e-12
        assert rel(oracle.newton_schulz(np.ascontiguousarray(G.T), co, eps=0.0, lib=lib), O.T) < 1e-12
        Q, _ = np.linalg.qr(rng(500 + k).standard_normal((r, r)))
        R, _ = np.linalg.qr(rng(600 + k).standard_normal((c, c)))
        assert rel(oracle.newton_schulz(Q @ G @ R, co, eps=0.0, lib=lib), Q @ O @ R) < 1e-11


def pin_momentum_golden(lib) -> None:
    """Momentum, Nesterov and zero-centring against the hand-worked 2x2 example."""
    g = read_golden("momentum_2x2.txt")
    mu = float(g["mu"][0])
    for nesterov in (True, False):
        p = np.zeros((2, 2)); m = np.zeros((2, 2))
        # steps = 0 and eps = 0: O = u / ||u||_F, lr = 1: p = -O
        O1 = oracle.muon_step([p], [g["g1"]], [m], lr=1.0, mu=mu, nesterov=nesterov, weight_decay=0.0,
                              rms_mode=0, coeffs=[], zero_center=False, eps=0.0, want_O=True, lib=lib)[0]
        assert np.max(np.abs(m - g["buf1"])) < 1e-15
        u1 = g["u1_nesterov"] if nesterov else g["u1_plain"]
        assert np.max(np.abs(O1 * np.linalg.norm(u1) - u1)) < 1e-14
        assert np.max(np.abs(p + O1)) < 1e-15
        O2 = oracle.muon_step([p], [g["g2"]], [m], lr=1.0, mu=mu, nesterov=nesterov, weight_decay=0.0,
                              rms_mode=0, coeffs=[], zero_center=False, eps=0.0, want_O=True, lib=lib)[0]
        assert np.max(np.abs(m - g["buf2"])) < 1e-15
        u2 = g["u2_nesterov"] if nesterov else g["u2_plain"]
        assert np.max(np.abs(O2 * np.linalg.norm(u2) - u2)) < 1e-14
    p = np.zeros((2, 2)); m = np.zeros((2, 2))
    oracle.muon_step([p], [g["gz"]], [m], lr=1.0, mu=mu, nesterov=True, weight_decay=0.0, rms_mode=0,
                     coeffs=[], zero_center=True, eps=0.0, lib=lib)
    assert np.max(np.abs(m - g["bufz"])) < 1e-15


def pin_update_rule(lib) -> None:
    """p <- p (1 - lr wd) - lr s O, with s = sqrt(max(1, rows/cols)) in RMS mode."""
    for (r, c) in ((6, 4), (4, 6)):
        p0 = rng(9).standard_normal((r, c))
        grad = rng(10).standard_normal((r, c))
        for rms in (0, 1):
            p = p0.copy(); m = np.zeros((r, c))
            O = oracle.muon_step([p], [grad], [m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1,
                                 rms_mode=rms, coeffs=[QUINTIC] * 5, zero_center=False, eps=1e-7,
                                 want_O=True, lib=lib)[0]
            s = np.sqrt(max(1.0, r / c)) if rms else 1.0
            assert np.max(np.abs(p - (p0 * (1 - 0.02 * 0.1) - 0.02 * s * O))) < 1e-15
            # from a zero buffer, u = (mu (1 - mu) + (1 - mu)) g = 0.0975 g, so O = NS(g) with
            # eps seen at the scale of g
            assert rel(O, spectral_reference(grad, [QUINTIC] * 5, 1e-7 / 0.0975)) < 1e-10
    # a zero gradient from a zero buffer gives O = 0: the weights only decay
    p = p0.copy(); m = np.zeros_like(p0)
    O = oracle.muon_step([p], [np.zeros_like(p0)], [m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1,
                         rms_mode=0, coeffs=[QUINTIC] * 5, zero_center=False, eps=1e-7, want_O=True,
                         lib=lib)[0]
    assert np.all(O == 0.0) and np.all(np.isfinite(p))
    assert np.max(np.abs(p - p0 * (1 - 0.002))) < 1e-15


def pin_zero_center(lib) -> None:
    """With centring along dim 0, every column of O sums to zero (1^T u = 0 carries through
    the odd polynomial), and a gradient with all rows equal gives O = 0."""
    for (r, c) in ((9, 14), (14, 9)):
        G = rng(11).standard_normal((r, c)) + 3.0
        O = oracle.newton_schulz(G, [QUINTIC] * 5, zero_center=True, eps=1e-7, lib=lib)
        assert np.max(np.abs(O.sum(axis=0))) < 1e-11
        Gc = G - G.mean(axis=0, keepdims=True)
        assert rel(O, spectral_reference(Gc, [QUINTIC] * 5, 1e-7)) < 1e-10
        row = rng(12).standard_normal(c)
        Oz = oracle.newton_schulz(np.tile(row, (r, 1)), [QUINTIC] * 5, zero_center=True, eps=1e-7, lib=lib)
        # centring leaves only rounding residue (~1e-16), far below eps = 1e-7, so x0 <= ~1e-8
        # and O stays below a^5 x0 ~ 1e-5, against entries ~0.3 for a full-rank update
        assert np.max(np.abs(Oz)) < 1e-4


def pin_checkpoint_split(lib) -> None:
    """Five steps, then the state carried over, then five more, equals ten straight steps;
    a NULL gradient leaves its matrix untouched."""
    r, c = 7, 11
    grads = [rng(1000 + s).standard_normal((r, c)) for s in range(10)]
    p_a = rng(13).standard_normal((r, c)); m_a = np.zeros((r, c))
    p_b = p_a.copy(); m_b = m_a.copy()
    kw = dict(lr=0.02, mu=0.95, nesterov=True, weight_decay=0.01, rms_mode=0, coeffs=[QUINTIC] * 5,
              zero_center=False, eps=1e-7, lib=lib)
    for s in range(10):
        oracle.muon_step([p_a], [grads[s]], [m_a], **kw)
    for s in range(5):
        oracle.muon_step([p_b], [grads[s]], [m_b], **kw)
    p_b, m_b = p_b.copy(), m_b.copy()
    for s in range(5, 10):
        oracle.muon_step([p_b], [grads[s]], [m_b], **kw)
    assert np.array_equal(p_a, p_b) and np.array_equal(m_a, m_b)
    p_c = p_a.copy(); m_c = m_a.copy()
    oracle.muon_step([p_c], [None], [m_c], **kw)
    assert np.array_equal(p_c, p_a) and np.array_equal(m_c, m_a)


def _adamw(lib, p, g_list, lr, b1, b2, eps, wd, m=None, v=None, step0=0):
    m = np.zeros_like(p) if m is None else m
    v = np.zeros_like(p) if v is None else v
    for t, g in enumerate(g_list, start=step0 + 1):
        oracle.adamw_step([p], [g], [m], [v], step=t, lr=lr, beta1=b1, beta2=b2, eps=eps, weight_decay=wd,
                          lib=lib)
    return p, m, v


def pin_adamw_golden(lib) -> None:
    """AdamW against the hand-worked two-step example ("Muon meets Mamba" 4.2 `_step_adamw`)."""
    g = read_golden("adamw_2step.txt")
    p = g["p0"].copy(); m = np.zeros(2); v = np.zeros(2)
    kw = dict(lr=float(g["lr"][0]), beta1=float(g["b1"][0]), beta2=float(g["b2"][0]), eps=0.0,
              weight_decay=float(g["wd"][0]), lib=lib)
    oracle.adamw_step([p], [g["g1"]], [m], [v], step=1, **kw)
    assert np.max(np.abs(m - g["m1"])) < 1e-15 and np.max(np.abs(v - g["v1"])) < 1e-15
    assert np.max(np.abs(p - g["p1"])) < 1e-15
    oracle.adamw_step([p], [g["g2"]], [m], [v], step=2, **kw)
    assert np.max(np.abs(m - g["m2"])) < 1e-15 and np.max(np.abs(v - g["v2"])) < 1e-15
    assert np.max(np.abs(p - g["p2"])) < 1e-14
    _, m, v = _adamw(lib, np.zeros(2), [g["g1"], np.array([0.0, 3.0])], lr=0.0, b1=0.9, b2=0.99, eps=1e-8, wd=0.0)
    assert np.max(np.abs(m - g["bm2"])) < 1e-15 and np.max(np.abs(v - g["bv2"])) < 1e-15


def pin_adamw_closed_forms(lib) -> None:
    """With bias correction, a constant gradient g moves every weight by -lr g / (|g| + eps) at every
    step (the corrected moments are g and g^2 exactly); the first step from zero state is the same;
    a zero gradient leaves only the decoupled decay p (1 - lr wd)."""
    r = rng(21)
    g = r.standard_normal(40) * np.exp(r.uniform(-6, 2, 40))
    p0 = r.standard_normal(40)
    lr, eps = 1e-2, 1e-8
    for t_total in (1, 7):
        p, _, _ = _adamw(lib, p0.copy(), [g] * t_total, lr=lr, b1=0.9, b2=0.95, eps=eps, wd=0.0)
        want = p0 - t_total * lr * g / (np.abs(g) + eps)
        assert np.max(np.abs(p - want)) < 1e-12 * t_total, t_total
    p, m, v = _adamw(lib, p0.copy(), [np.zeros(40)] * 3, lr=lr, b1=0.9, b2=0.95, eps=eps, wd=0.1)
    assert np.max(np.abs(p - p0 * (1 - lr * 0.1) ** 3)) < 1e-15 and not m.any() and not v.any()


# the pins of the Muon step (Newton-Schulz, momentum, update); the AdamW pins follow
MUON_PINS = [pin_spectral_map, pin_rank_one, pin_diagonal, pin_cubic_converges_to_polar, pin_quintic_band,
             pin_invariances, pin_momentum_golden, pin_update_rule, pin_zero_center, pin_checkpoint_split]
ALL_PINS = MUON_PINS + [pin_adamw_golden, pin_adamw_closed_forms]


def failing_pins(lib, pins: Sequence = None) -> List[str]:
    bad = []
    for pin in (ALL_PINS if pins is None else pins):
        try:
            pin(lib)
        except (AssertionError, ValueError, FloatingPointError):
            bad.append(pin.__name__)
    return bad

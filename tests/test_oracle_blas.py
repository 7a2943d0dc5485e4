"""The fp64 oracle with library matrix products (``oracle/ns_blas.py``), which the full-size
parity tests use for the largest weight shapes, against the same pins as the plain-loop oracle
(facts fixed by the pages and the mathematics), against planted mistakes in copies of its own
source, and against the plain-loop oracle on shapes both finish quickly (CPU only)."""
import importlib.util

import numpy as np
import pytest

import oracle
from oracle import ns_blas
from tests import pins


@pytest.mark.parametrize("pin", pins.MUON_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(ns_blas)


@pytest.mark.parametrize("shape", [(64, 96), (96, 64), (80, 80), (1, 33), (33, 1), (130, 257)])
@pytest.mark.parametrize("sched", ["quintic", "cubic", "hybrid"])
def test_agrees_with_plain_loop_oracle(shape, sched):
    coeffs = {"quintic": [pins.QUINTIC] * 5, "cubic": [pins.CUBIC] * 5, "hybrid": pins.HYBRID}[sched]
    G = pins.rng(sum(shape)).standard_normal(shape) * np.exp(pins.rng(7).uniform(-4, 1, shape[1]))[None, :]
    a = oracle.newton_schulz(G, coeffs, eps=1e-7)
    b = ns_blas.newton_schulz(G, coeffs, eps=1e-7)
    assert pins.rel(b, a) < 1e-12


def test_step_agrees_with_plain_loop_oracle():
    """Three Muon steps with zero-centring, Nesterov, decay and the RMS factor."""
    shapes = [(40, 70), (70, 40)]
    r = pins.rng(77)
    p0 = [r.standard_normal(s) * 0.02 for s in shapes]
    kw = dict(lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1, rms_mode=1, coeffs=[pins.QUINTIC] * 5,
              zero_center=True, eps=1e-7, want_O=True)
    pa, ma = [p.copy() for p in p0], [np.zeros(s) for s in shapes]
    pb, mb = [p.copy() for p in p0], [np.zeros(s) for s in shapes]
    for step in range(3):
        g = [r.standard_normal(s) for s in shapes]
        Oa = oracle.muon_step(pa, g, ma, **kw)
        Ob = oracle.muon_step(pb, g, mb, lib=ns_blas, **kw)
        for j in range(len(shapes)):
            assert pins.rel(Ob[j], Oa[j]) < 1e-12
            assert pins.rel(pb[j], pa[j]) < 1e-14 and pins.rel(mb[j], ma[j]) < 1e-15


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        ns_blas.newton_schulz(np.zeros((0, 3)), [pins.QUINTIC])


# Plausible mistakes, each planted in a copy of the module source; every one must trip a pin.
MUTANTS = {
    "poly_sign": ("B = b * A + c * (A @ A)", "B = b * A - c * (A @ A)"),
    "dropped_aX": ("X = a * X + B @ X", "X = B @ X"),
    "dropped_BX": ("X = a * X + B @ X", "X = a * X"),
    "coeff_order": ("for a, b, c in coeffs:", "for a, c, b in coeffs:"),
    "gram_transposed": ("A = X @ X.T", "A = X.T @ X if X.shape[0] == X.shape[1] else X @ X.T"),
    "update_right_side": ("X = a * X + B @ X", "X = a * X + (X @ B if X.shape[0] == X.shape[1] else B @ X)"),
    "eps_dropped": ("(np.sqrt(np.sum(u * u)) + eps)", "np.sqrt(np.sum(u * u))"),
    "no_norm_sqrt": ("(np.sqrt(np.sum(u * u)) + eps)", "(np.sum(u * u) + eps)"),
    "no_transpose_back": ("    if tall:                                    # transpose back\n        X = X.T\n", ""),
    "momentum_coeff": ("m += (1.0 - mu) * g", "m += g"),
    "nesterov_ignored": ("u = mu * m + (1.0 - mu) * g if nesterov else m", "u = m"),
    "decay_sign": ("p *= 1.0 - lr * weight_decay", "p *= 1.0 + lr * weight_decay"),
    "rms_inverted": ("max(1.0, r / c)", "max(1.0, c / r)"),
    "center_wrong_axis": ("g.mean(axis=0, keepdims=True)", "g.mean(axis=1, keepdims=True)"),
    "center_skipped_in_step": ("        if zero_center:\n            g = center_columns(g)\n", ""),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(ns_blas.__file__).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    path = tmp_path / f"ns_blas_{name}.py"
    path.write_text(src.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location(f"ns_blas_{name}", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    bad = pins.failing_pins(mod, pins.MUON_PINS)
    assert bad, f"no pin caught mutant {name}"

"""Plant plausible mistakes in copies of the oracle source (on the CPU) and check that the
pins catch every one: a dropped term, a wrong sign, a wrong index, a transposed operand,
a misplaced eps, a forgotten transpose-back, a wrong momentum or decay coefficient."""
import os
import shutil
import subprocess

import pytest

import oracle
from tests import pins

MUTANTS = {
    "poly_sign": ("B[e] = b * A[e] + cc * AA[e];", "B[e] = b * A[e] - cc * AA[e];"),
    "dropped_aX": ("X[e] = a * X[e] + BX[e];", "X[e] = BX[e];"),
    "dropped_BX": ("X[e] = a * X[e] + BX[e];", "X[e] = a * X[e];"),
    "coeff_index": ("b = coeffs[3 * k + 1], cc = coeffs[3 * k + 2]",
                    "b = coeffs[3 * k + 2], cc = coeffs[3 * k + 1]"),
    "transposed_update": ("matmul(B.data(), X.data(), BX.data(), m, m, n, nthreads);",
                          "matmul(B.data(), X.data(), BX.data(), m, m, n, nthreads);"
                          " if (m == n) { std::vector<double> t(BX); matmul(X.data(), B.data(), t.data(), m, m, n, nthreads); BX = t; }"),
    "gram_not_transposed": ("matmul(X.data(), Xt.data(), A.data(), m, n, m, nthreads);   // A = X X^T",
                            "matmul(X.data(), Xt.data(), A.data(), m, n, m, nthreads); if (m == n) matmul(X.data(), X.data(), A.data(), m, m, m, nthreads);"),
    "eps_dropped": ("frobenius(u, n_el) + eps", "frobenius(u, n_el)"),
    "no_transpose_back": ("transpose(X.data(), O, m, n);", "std::memcpy(O, X.data(), sizeof(double) * n_el);"),
    "momentum_coeff": ("m[e] = mu * m[e] + (1.0 - mu) * g[e];", "m[e] = mu * m[e] + g[e];"),
    "nesterov_ignored": ("u[e] = nesterov ? mu * m[e] + (1.0 - mu) * g[e] : m[e];", "u[e] = m[e];"),
    "decay_sign": ("p[e] * (1.0 - lr * weight_decay)", "p[e] * (1.0 + lr * weight_decay)"),
    "rms_inverted": ("(double)r / (double)c", "(double)c / (double)r"),
    "center_wrong_divisor": ("mean[j] /= (double)r;", "mean[j] /= (double)c;"),
    "center_after_momentum": ("if (zero_center) zero_center_rows(g.data(), r, c);", ""),
    "matmul_accumulate_index": ("c[j] += a * b[j];", "c[j] += a * b[(j + 1) % N];"),
    "adamw_no_bias_corr1": ("const double step_size = lr / bias_corr1;", "const double step_size = lr;"),
    "adamw_no_bias_corr2": ("std::sqrt(v[e]) / std::sqrt(bias_corr2) + eps", "std::sqrt(v[e]) + eps"),
    "adamw_second_moment_not_squared": ("(1.0 - beta2) * g[e] * g[e]", "(1.0 - beta2) * g[e]"),
    "adamw_decay_after_update": ("if (weight_decay != 0.0) p[e] = p[e] * (1.0 - lr * weight_decay);",
                                 "if (weight_decay != 0.0) p[e] = p[e] * (1.0 - weight_decay);"),
    "adamw_momentum_coeff": ("m[e] = beta1 * m[e] + (1.0 - beta1) * g[e];", "m[e] = beta1 * m[e] + g[e];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mutant.cpp"
    path.write_text(mutated)
    so = str(tmp_path / f"libmutant_{name}.so")
    oracle.build(force=True, src=str(path), out=so)
    lib = oracle.load(so)
    bad = pins.failing_pins(lib)
    assert bad, f"no pin caught mutant {name}"

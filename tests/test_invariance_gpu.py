"""Invariances of the Newton-Schulz map on the CUDA path ("AdamW vs Muon" part 3: the iteration is
an odd polynomial acting on the singular values of G / ||G||_F, so it ignores the scale of G,
flips with its sign and commutes with transposition).

The device folds the normalisation into the first products (1/||u|| enters as alpha^2 on the
unnormalised Gram and as alpha on the first update), so very large or very small inputs meet
the fp32 accumulators before they are scaled, unlike the pages' normalise-first order. These
tests run the device path at extreme scales against the fp64 oracle, and check the exact
identities that follow from its arithmetic:
  - sign: every product is odd or even in G, and round-to-nearest is symmetric, so NS(-G) is
    exactly -NS(G);
  - powers of two with eps = 0: scaling G by 2^k scales every rounding of the unnormalised
    iterate and its Gram exactly, and alpha by exactly 2^-k, so the output is bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import TOL_O_BF16, TOL_O_FP32, host64, rel, to_dev

pytestmark = pytest.mark.gpu

Q5 = [synth.QUINTIC] * 5
PRECS = [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)]


def _gen(shape, seed):
    rng = np.random.default_rng(seed)
    G = rng.standard_normal(shape)
    return G * np.exp(rng.uniform(np.log(1e-2), 0.0, size=shape[1]))[None, :]


def _ns(G: np.ndarray, prec: str, eps: float = 1e-7) -> torch.Tensor:
    import newton_schulz_13_b200 as ns
    X = ns.ns_orthogonalize(to_dev(G, torch.float32), steps=5, coeffs=Q5, eps=eps, prec=prec,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    return X


@pytest.mark.parametrize("shape", [(700, 300), (300, 700)], ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("prec,tol", PRECS, ids=["bf16", "fp32"])
def test_scale_sign_transpose_against_oracle(shape, prec, tol):
    G0 = synth.round_to(_gen(shape, 51), "fp32")
    outs = {}
    for scale in (1e-6, 1.0, 1e6):
        G = synth.round_to(G0 * scale, "fp32")   # the oracle sees exactly the device's input
        X = host64(_ns(G, prec))
        assert np.all(np.isfinite(X))
        want = oracle.newton_schulz(G, Q5, eps=1e-7)
        assert rel(X, want) <= tol, (scale, rel(X, want))
        outs[scale] = X
    # sign: exactly the negated output
    Xn = host64(_ns(-G0, prec))
    assert np.array_equal(Xn, -outs[1.0])
    # transpose: the other orientation of the iterate, against the oracle and the device's own output
    Gt = np.ascontiguousarray(G0.T)
    Xt = host64(_ns(Gt, prec))
    want_t = oracle.newton_schulz(Gt, Q5, eps=1e-7)
    assert rel(Xt, want_t) <= tol, rel(Xt, want_t)
    assert rel(Xt, outs[1.0].T) <= 2 * tol


@pytest.mark.parametrize("shape", [(700, 300), (300, 700), (2100, 2600)], ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("prec", ["bf16", "fp32"])
def test_power_of_two_scale_is_bit_exact(shape, prec):
    G0 = synth.round_to(_gen(shape, 53), "fp32")
    ref = _ns(G0, prec, eps=0.0)
    # |k| <= 20 keeps every square and product of the input normal in fp32 (no subnormals, whose
    # rounding would not scale)
    for k in (-20, -7, 9, 20):
        Xk = _ns(G0 * 2.0 ** k, prec, eps=0.0)
        assert torch.equal(Xk, ref), k


@pytest.mark.parametrize("prec,tol", PRECS, ids=["bf16", "fp32"])
def test_step_invariant_to_gradient_scale(prec, tol):
    """The whole Muon step from a zero buffer: u is proportional to g, so the update O, and with it
    the new parameters, do not depend on the gradient's scale (eps aside); checked against the
    oracle at gradient scales 1e-6 and 1e6."""
    import newton_schulz_13_b200 as ns
    r, c = 300, 700
    rng = np.random.default_rng(57)
    p0 = synth.round_to(0.02 * rng.standard_normal((r, c)), "fp32")
    g0 = synth.round_to(_gen((r, c), 59), "fp32")
    for scale in (1e-6, 1e6):
        g = synth.round_to(g0 * scale, "fp32")
        p = to_dev(p0, torch.float32)
        m = torch.zeros((r, c), dtype=torch.float32, device="cuda")
        ns.muon_step([p], [to_dev(g, torch.float32)], [m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.01,
                     steps=5, coeffs=Q5, eps=1e-7, prec=prec)
        torch.cuda.synchronize()
        assert ns.check_status() == ns.OK
        o_p, o_m = p0.astype(np.float64).copy(), np.zeros((r, c))
        O_ref = oracle.muon_step([o_p], [g], [o_m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.01,
                                 rms_mode=0, coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
        decay = np.float64(np.float32(1.0 - np.float32(0.02) * np.float32(0.01)))
        O_gpu = (p0 * decay - host64(p)) / np.float64(np.float32(0.02))
        assert rel(O_gpu, O_ref) <= tol, (scale, rel(O_gpu, O_ref))
        assert rel(host64(p), o_p) <= 1e-3

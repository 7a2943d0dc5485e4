"""Bounds of every write the library makes, checked with guard bands.

Each buffer the caller passes (parameters, momentum, gradients, the orthogonalised output) is
placed inside a larger allocation whose other bytes hold a sentinel bit pattern (a NaN); after
the call the sentinel must be bit-identical, and the gradients (read only) must be unchanged
everywhere. The parameter update writes the caller's parameters through TMA stores clipped by
the tensor map's bounds (bf16 mode) or through plain stores (fp32 mode), so ragged shapes, the
256 x 512 tiles, odd offsets and single rows or columns are covered in both precisions. The
values are also checked against the fp64 oracle (its library-product form, for speed).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ns_blas
from tests.gpu_util import TOL_O_BF16, TOL_O_FP32, TOL_P, host64, rel

pytestmark = pytest.mark.gpu

Q5 = [synth.QUINTIC] * 5
BAND = 4096                      # elements on each side of the buffer
SENT32 = 0x7FC0DEAD              # a quiet-NaN bit pattern for 32-bit buffers
SENT16 = 0x7FDE                  # and for bf16 buffers


class Banded:
    """A (rows x cols) view inside a flat allocation of BAND + offset + rows * cols + BAND
    elements whose surrounding elements hold a sentinel."""

    def __init__(self, values: np.ndarray, dtype, offset: int = 0):
        self.shape = values.shape
        n = values.size
        self.lo = BAND + offset
        self.store = torch.empty(self.lo + n + BAND, dtype=dtype, device="cuda")
        ints = self.store.view(torch.int32 if dtype == torch.float32 else torch.int16)
        ints.fill_(SENT32 if dtype == torch.float32 else SENT16)
        self.view = self.store[self.lo:self.lo + n].view(self.shape)
        self.view.copy_(torch.from_numpy(np.ascontiguousarray(values)).to(dtype))
        self.snapshot = self.store.clone()

    def _ints(self, t):
        return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)

    def bands_intact(self) -> bool:
        n = self.view.numel()
        a, b = self._ints(self.store), self._ints(self.snapshot)
        return torch.equal(a[:self.lo], b[:self.lo]) and torch.equal(a[self.lo + n:], b[self.lo + n:])

    def unchanged(self) -> bool:
        return torch.equal(self._ints(self.store), self._ints(self.snapshot))


SHAPES = [(33, 17), (2100, 2600), (2600, 2100), (1, 7), (7, 1), (300, 701), (520, 520)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("prec,tol", [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)], ids=["bf16", "fp32"])
@pytest.mark.parametrize("offset", [0, 1, 4], ids=["aligned", "offset1", "offset4"])
def test_step_writes_stay_inside_their_buffers(shape, prec, tol, offset):
    import newton_schulz_13_b200 as ns
    r, c = shape
    rng = np.random.default_rng(61 + r + c)
    p0 = synth.round_to(0.02 * rng.standard_normal((r, c)), "fp32")
    g = synth.round_to(rng.standard_normal((r, c)) * np.exp(rng.uniform(-2, 0, c))[None, :], "bf16")
    P = Banded(p0, torch.float32, offset)
    M = Banded(np.zeros((r, c)), torch.float32, offset)
    G = Banded(g, torch.bfloat16, offset)
    ns.muon_step([P.view], [G.view], [M.view], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1, rms_scale=1,
                 steps=5, coeffs=Q5, eps=1e-7, prec=prec)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    assert P.bands_intact(), "parameter guard band overwritten"
    assert M.bands_intact(), "momentum guard band overwritten"
    assert G.unchanged(), "gradient buffer or its guard band changed"
    o_p, o_m = p0.astype(np.float64).copy(), np.zeros((r, c))
    O_ref = ns_blas.muon_step([o_p], [g], [o_m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1, rms_mode=1,
                              coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
    s = np.sqrt(max(1.0, r / c))
    decay = np.float64(np.float32(1.0 - np.float32(0.02) * np.float32(0.1)))
    O_gpu = (p0 * decay - host64(P.view)) / (np.float64(np.float32(0.02)) * s)
    assert rel(O_gpu, O_ref) <= tol, rel(O_gpu, O_ref)
    # The parameter bound needs a step small against the weights: lr ||O|| / ||p|| is about
    # 0.9 / sqrt(max(r, c)) here (O has min(r, c) singular values near 0.9, p entries N(0, 0.02)),
    # 16-26 % for the tiny shapes, where an O error within its tolerance moves p by more than 1e-3.
    if max(r, c) >= 256:
        assert rel(host64(P.view), o_p) <= TOL_P


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("prec,tol", [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)], ids=["bf16", "fp32"])
@pytest.mark.parametrize("out", ["fp32", "bf16"])
def test_orthogonalize_writes_stay_inside_the_output(shape, prec, tol, out):
    import newton_schulz_13_b200 as ns
    r, c = shape
    rng = np.random.default_rng(67 + r * c)
    g = synth.round_to(rng.standard_normal((r, c)), "fp32")
    G = Banded(g, torch.float32, 1)
    X = Banded(np.zeros((r, c)), torch.float32 if out == "fp32" else torch.bfloat16, 3)
    ns.ns_orthogonalize(G.view, X.view, steps=5, coeffs=Q5, eps=1e-7, prec=prec)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    assert X.bands_intact(), "output guard band overwritten"
    assert G.unchanged(), "input buffer or its guard band changed"
    want = ns_blas.newton_schulz(g, Q5, eps=1e-7)
    got = host64(X.view)
    # a bf16 output adds one rounding (2^-9 relative) to the bf16 or fp32 working precision
    assert rel(got, want) <= (tol if out == "fp32" else tol + 4e-3), rel(got, want)


@pytest.mark.parametrize("prec,tol", [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)], ids=["bf16", "fp32"])
def test_mixed_wave_on_wide_tiles(prec, tol):
    """One call whose wave runs on 256 x 512 tiles (the 2100 x 2600 matrix carries its FLOPs) and
    also holds matrices whose contraction is a single K slice or a few (1 x 7, 7 x 1, 33 x 17,
    300 x 64): their tiles start and end inside the ring's first stages. Each matrix in its own
    guard bands, values against the oracle."""
    import newton_schulz_13_b200 as ns
    shapes = [(7, 1), (2100, 2600), (33, 17), (1, 7), (300, 64)]
    rng = np.random.default_rng(71)
    p0s, gs, Ps, Ms, Gs = [], [], [], [], []
    for k, (r, c) in enumerate(shapes):
        p0 = synth.round_to(0.02 * rng.standard_normal((r, c)), "fp32")
        g = synth.round_to(rng.standard_normal((r, c)), "bf16")
        p0s.append(p0)
        gs.append(g)
        Ps.append(Banded(p0, torch.float32, k % 3))
        Ms.append(Banded(np.zeros((r, c)), torch.float32, 1))
        Gs.append(Banded(g, torch.bfloat16, 2))
    ns.muon_step([P.view for P in Ps], [G.view for G in Gs], [M.view for M in Ms], lr=0.02, mu=0.95,
                 nesterov=True, weight_decay=0.1, rms_scale=1, steps=5, coeffs=Q5, eps=1e-7, prec=prec)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    for k, (r, c) in enumerate(shapes):
        assert Ps[k].bands_intact() and Ms[k].bands_intact() and Gs[k].unchanged(), shapes[k]
        o_p, o_m = p0s[k].astype(np.float64).copy(), np.zeros((r, c))
        O_ref = ns_blas.muon_step([o_p], [gs[k]], [o_m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1,
                                  rms_mode=1, coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
        s = np.sqrt(max(1.0, r / c))
        decay = np.float64(np.float32(1.0 - np.float32(0.02) * np.float32(0.1)))
        O_gpu = (p0s[k] * decay - host64(Ps[k].view)) / (np.float64(np.float32(0.02)) * s)
        assert rel(O_gpu, O_ref) <= tol, (shapes[k], rel(O_gpu, O_ref))

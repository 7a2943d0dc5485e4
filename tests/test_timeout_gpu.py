"""The failure path of the bounded waits inside the Newton-Schulz product kernels.

Every wait of those kernels has a time limit; when one runs out, the kernel raises the abort flag
of both CTAs of its pair, drains the copies and tensor-core work still in flight (settling the two
producers' stage counts, which can then differ), frees its tensor memory, sets the timeout bit of
the device status word and returns. These tests make the waits run out on purpose, with a limit
of a few nanoseconds set through muon_set_wait_limit_ns, so that the first wait that is not already
complete gives up. Nothing waits on a flag that is never set and nothing faults: the check is that
the call reports MUON_ERR_TIMEOUT through muon_check_status, and that the device stays usable, with
the next call at the default limit correct against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import TOL_O_BF16, TOL_O_FP32, TOL_P, host64, rel, to_dev

pytestmark = pytest.mark.gpu

Q5 = [synth.QUINTIC] * 5


@pytest.fixture
def short_waits():
    import newton_schulz_13_b200 as ns
    ns.check_status()            # start from a clear status word
    yield ns.set_wait_limit_ns
    ns.set_wait_limit_ns(0)


def _inputs(shape, seed):
    rng = np.random.default_rng(seed)
    p0 = synth.round_to(0.02 * rng.standard_normal(shape), "fp32")
    g = synth.round_to(rng.standard_normal(shape), "bf16")
    return p0, g


def _step(ns, p0, g, prec):
    p = to_dev(p0, torch.float32)
    m = torch.zeros(p0.shape, dtype=torch.float32, device="cuda")
    ns.muon_step([p], [to_dev(g, torch.bfloat16)], [m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.01,
                 steps=5, coeffs=Q5, eps=1e-7, prec=prec)
    return p


# 256 x 512: the 256 x 256 CTA-pair tiles, in one chained launch (chain 1, the default for a single
# small matrix) or in one launch per phase with eight epilogue warps (chain 0); 2100 x 2600: the
# 256 x 512 tiles; fp32: the 3xTF32 kernel
@pytest.mark.parametrize("shape,prec,tol,chain", [((256, 512), "bf16", TOL_O_BF16, 1), ((256, 512), "bf16", TOL_O_BF16, 0),
                                                  ((2100, 2600), "bf16", TOL_O_BF16, 1),
                                                  ((256, 512), "fp32", TOL_O_FP32, 1), ((700, 300), "fp32", TOL_O_FP32, 1)],
                         ids=["bf16-256x512-chained", "bf16-256x512-per-phase", "bf16-wide-2100x2600", "fp32-256x512",
                              "fp32-tall-700x300"])
def test_wait_that_runs_out_is_reported_and_the_device_recovers(short_waits, shape, prec, tol, chain):
    import newton_schulz_13_b200 as ns
    ns.set_chained_launch(chain)
    try:
        _timeout_then_recover(ns, shape, prec, tol)
    finally:
        ns.set_chained_launch(1)


def _timeout_then_recover(ns, shape, prec, tol):
    p0, g = _inputs(shape, 71)
    short_waits = ns.set_wait_limit_ns
    short_waits(4)                                    # 4 ns: the first incomplete wait gives up
    _step(ns, p0, g, prec)
    with pytest.raises(ns.MuonError) as ei:
        ns.check_status()
    assert ei.value.code == ns.ERR_TIMEOUT
    assert ns.check_status() == ns.OK                 # the status word was cleared
    short_waits(0)                                    # the default limit again
    p = _step(ns, p0, g, prec)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    o_p, o_m = p0.astype(np.float64).copy(), np.zeros(shape)
    O_ref = oracle.muon_step([o_p], [g], [o_m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.01, rms_mode=0,
                             coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
    decay = np.float64(np.float32(1.0 - np.float32(0.02) * np.float32(0.01)))
    O_gpu = (p0 * decay - host64(p)) / np.float64(np.float32(0.02))
    assert rel(O_gpu, O_ref) <= tol
    assert rel(host64(p), o_p) <= TOL_P


def test_timed_out_orthogonalize_then_many_normal_calls(short_waits):
    """Several timed-out calls in a row (wide and tall iterates), then normal ones: no state of the
    library or the device is left behind by the early exits."""
    import newton_schulz_13_b200 as ns
    rng = np.random.default_rng(73)
    Gs = [synth.round_to(rng.standard_normal(s), "fp32") for s in ((300, 700), (700, 300), (1000, 96))]
    short_waits(4)
    for G in Gs:
        ns.ns_orthogonalize(to_dev(G, torch.float32), steps=5, coeffs=Q5, prec="bf16", out_dtype=torch.float32)
    with pytest.raises(ns.MuonError) as ei:
        ns.check_status()
    assert ei.value.code == ns.ERR_TIMEOUT
    short_waits(0)
    for _ in range(2):
        for G in Gs:
            X = ns.ns_orthogonalize(to_dev(G, torch.float32), steps=5, coeffs=Q5, prec="bf16",
                                    out_dtype=torch.float32)
            assert rel(host64(X), oracle.newton_schulz(G, Q5, eps=1e-7)) <= TOL_O_BF16
    assert ns.check_status() == ns.OK

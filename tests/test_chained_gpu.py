"""Chained launches: the whole Newton-Schulz iteration of a wave of small matrices in one launch,
tiles claimed in order and each phase waiting per matrix for the phase whose results it reads.

The chained launch runs the same tiles with the same arithmetic as one launch per phase, so the
results must be bit-identical; every workload whose waves use 256 x 256 tiles is checked both
ways over two steps (the quintic, cubic with zero-centring, where the update waits on the Gram
product directly, and the 8 + 2 hybrid schedule), and against the fp64 oracle through the
workload tests, which run chained by default.
"""
import pytest
import torch

import synth
from tests.gpu_util import StepCase

pytestmark = pytest.mark.gpu


@pytest.fixture
def chain_switch():
    import newton_schulz_13_b200 as ns
    yield ns.set_chained_launch
    ns.set_chained_launch(True)


def _run(wl, chained, coeffs=None, prec="bf16"):
    import newton_schulz_13_b200 as ns
    ns.set_chained_launch(chained)
    case = StepCase(wl, sample=[], device_fill=True)
    for k in range(2):
        case.step(k, prec=prec, coeffs=coeffs)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    return [p.clone() for p in case.params] + [m.clone() for m in case.momentum]


@pytest.mark.parametrize("name,sched", [("gpt2_small", None), ("mamba_24", None), ("cubic_zero_center_12", None),
                                        ("single_256x512", None), ("gpt2_small", "hybrid")])
def test_chained_launch_is_bit_identical_to_per_phase_launches(chain_switch, name, sched):
    wl = synth.WORKLOADS[name]
    coeffs = synth.HYBRID if sched == "hybrid" else None
    a = _run(wl, True, coeffs)
    b = _run(wl, False, coeffs)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_chained_launch_counts_one_product_launch_per_wave(chain_switch):
    """GPT-2-small is one wave: one chained launch replaces the fifteen per-phase launches."""
    import newton_schulz_13_b200 as ns
    wl = synth.WORKLOADS["gpt2_small"]
    case = StepCase(wl, sample=[], device_fill=True)
    case.step(0)                      # builds the plan and writes the tables
    torch.cuda.synchronize()
    ns.profile_read()
    ns.profile_enable(True)
    try:
        case.step(1)
        torch.cuda.synchronize()
        rec = ns.profile_read()
    finally:
        ns.profile_enable(False)
    assert rec["gemm"][0] == 1, rec["gemm"]
    assert ns.check_status() == ns.OK

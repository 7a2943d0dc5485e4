"""Chained launches: the whole Newton-Schulz iteration of a wave of small matrices in one launch,
tiles claimed in order and each phase waiting per matrix for the phase whose results it reads.

The chained launch runs the same tiles with the same arithmetic as one launch per phase, so the
results must be bit-identical; every workload whose waves use 256 x 256 tiles is checked both
ways over two steps (the quintic, cubic with zero-centring, where the update waits on the Gram
product directly, and the 8 + 2 hybrid schedule). The automatic mode's choice per workload is
checked by counting product launches; the workload tests check both paths against the fp64
oracle (single_256x512 and the cubic set chain by default, the others do not).
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
    ns.set_chained_launch(1)


def _run(wl, mode, coeffs=None, prec="bf16"):
    import newton_schulz_13_b200 as ns
    ns.set_chained_launch(mode)
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
    a = _run(wl, 2, coeffs)   # chained
    b = _run(wl, 0, coeffs)   # one launch per phase
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _product_launches(wl):
    import newton_schulz_13_b200 as ns
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
    assert ns.check_status() == ns.OK
    return rec["gemm"][0]


@pytest.mark.parametrize("name,mode,launches", [
    ("gpt2_small", 2, 1),        # forced: one chained launch replaces the fifteen per-phase ones
    ("gpt2_small", 1, 15),       # automatic: about 25 tiles per CTA pair per iteration, per phase
    ("gpt2_small", 0, 15),
    ("single_256x512", 1, 1),    # automatic: a handful of tiles, chained
    ("cubic_zero_center_12", 1, 1),
    ("cubic_zero_center_12", 0, 10)])   # cubic: no polynomial product, two launches per step
def test_chained_launch_choice(chain_switch, name, mode, launches):
    chain_switch(mode)
    assert _product_launches(synth.WORKLOADS[name]) == launches


def test_chain_mode_rejects_other_values():
    import newton_schulz_13_b200 as ns
    with pytest.raises(ns.MuonError):
        ns.set_chained_launch(3)

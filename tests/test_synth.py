"""The seeded input generator: the numpy and torch backends draw the same stream, matrices are
independent of one another, and the workloads have the stated shapes and sizes."""
import math

import numpy as np
import pytest
import torch

import synth


def test_splitmix_reference_values():
    # splitmix64 from state 0: the first outputs of the published generator
    z = 0
    outs = []
    for _ in range(3):
        z = (z + synth.GAMMA) & ((1 << 64) - 1)
        outs.append(synth._mix_int(z))
    assert outs[0] == 0xE220A8397B1DCDAF
    assert outs[1] == 0x6E789E6AA1B965F4
    assert outs[2] == 0x06C45D188009454F


@pytest.mark.parametrize("key", [0, 1, 0xFFFFFFFFFFFFFFFF, synth.matrix_key(5, 3, 1, 0)])
def test_numpy_and_torch_backends_agree(key):
    n = 4097
    u_np = synth._uniform_np(key, n, 0)
    u_t = synth._uniform_t(key, n, 0, "cpu").numpy()
    assert np.array_equal(u_np, u_t)
    z_np = synth.standard_normal(key, n)
    z_t = synth.standard_normal_torch(key, n, "cpu").numpy()
    assert np.allclose(z_np, z_t, rtol=0, atol=1e-12)


def test_uniform_range_and_moments():
    u = synth._uniform_np(synth.matrix_key(0, 0, 1, 0), 200000, 0)
    assert u.min() > 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 5e-3
    z = synth.standard_normal(synth.matrix_key(0, 0, 1, 0), 200000)
    assert abs(z.mean()) < 1e-2 and abs(z.std() - 1.0) < 1e-2


def test_keys_separate_matrices_kinds_and_steps():
    keys = {synth.matrix_key(s, m, k, t) for s in range(3) for m in range(5) for k in (1, 2, 3) for t in range(4)}
    assert len(keys) == 3 * 5 * 3 * 4


def test_workload_sizes():
    w = synth.WORKLOADS
    assert w["single_256x512"].shapes == [(256, 512)]
    assert len(w["cubic_zero_center_12"].shapes) == 12
    assert len(w["gpt2_small"].shapes) == 48 and w["gpt2_small"].n_steps == 10
    assert len(w["mamba_24"].shapes) == 96
    ll = w["llama8b"]
    assert ll.count == 224 and ll.elements() == 6979321856
    assert math.isclose(ll.ns_flops(), 6.66e14, rel_tol=5e-3)
    assert w["cubic_zero_center_12"].ns_flops() == pytest.approx(2.72e11, rel=5e-3)


def test_column_scales_log_uniform():
    wl = synth.WORKLOADS["llama8b"]
    s = synth.log_uniform(synth.matrix_key(wl.seed, 1, synth.KIND_COLSCALE, 0), 4096, 1e-4, 1e-1)
    assert s.min() >= 1e-4 and s.max() <= 1e-1
    assert abs(np.log10(s).mean() - (-2.5)) < 0.05


def test_grad_is_reproducible_and_rounded_once():
    wl = synth.WORKLOADS["mamba_24"]
    a, b = wl.grad(5, 2), wl.grad(5, 2)
    assert np.array_equal(a, b)
    assert not np.array_equal(wl.grad(5, 2), wl.grad(5, 1))
    r = synth.round_to(a, "bf16")
    assert np.array_equal(r, torch.from_numpy(a).to(torch.bfloat16).double().numpy())

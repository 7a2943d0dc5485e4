"""AdamW step of the parameters that do not go to Muon: the CUDA path (through the C ABI) against
the fp64 oracle, on the GPT-2-small non-Muon parameters and on edge cases (ragged lengths,
misaligned views, skipped tensors). Arithmetic is fp32 on the device; the tolerance is 1e-5
relative (per tensor) on parameters and both moments."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import host64, rel, tdtype, to_dev

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _run(wl, steps, gdt_override=None):
    import newton_schulz_13_b200 as ns
    gdt = gdt_override or wl.grad_dtype
    ps = [to_dev(wl.param(i), torch.float32) for i in range(wl.count)]
    ms = [torch.zeros(n, device="cuda") for n in wl.sizes]
    vs = [torch.zeros(n, device="cuda") for n in wl.sizes]
    o_p = [host64(p) for p in ps]
    o_m = [np.zeros(n) for n in wl.sizes]
    o_v = [np.zeros(n) for n in wl.sizes]
    worst = 0.0
    for t in range(1, steps + 1):
        gs = [to_dev(wl.grad(i, t), tdtype(gdt)) for i in range(wl.count)]
        ns.adamw_step(ps, gs, ms, vs, step=t, lr=wl.lr, beta1=wl.beta1, beta2=wl.beta2, eps=wl.eps,
                      weight_decay=wl.weight_decay)
        oracle.adamw_step(o_p, [host64(g) for g in gs], o_m, o_v, step=t, lr=wl.lr, beta1=wl.beta1,
                          beta2=wl.beta2, eps=wl.eps, weight_decay=wl.weight_decay)
        torch.cuda.synchronize()
        for i in range(wl.count):
            for dev, ref in ((ps[i], o_p[i]), (ms[i], o_m[i]), (vs[i], o_v[i])):
                e = rel(host64(dev), ref)
                worst = max(worst, e)
                assert e <= TOL, (t, i, e)
    assert ns.check_status() == ns.OK
    return worst


@pytest.mark.parametrize("gdt", ["bf16", "fp32"])
def test_gpt2_small_non_muon_params(gdt):
    wl = synth.ADAM_WORKLOADS["gpt2_small_adamw"]
    print("worst", _run(wl, wl.n_steps, gdt))


def test_edge_cases_ragged_misaligned_skipped():
    import newton_schulz_13_b200 as ns
    rng = np.random.default_rng(3)
    sizes = [1, 7, 9, 8191, 8192, 8193, 40001]
    base = torch.zeros(sum(sizes) + 64, device="cuda")
    # tensors packed at odd float offsets: the vector path is off for the misaligned ones
    offs, o = [], 1
    for n in sizes:
        offs.append(o)
        o += n + 3
    big_p = torch.zeros(o + 8, device="cuda")
    big_m = torch.zeros(o + 8, device="cuda")
    big_v = torch.zeros(o + 8, device="cuda")
    p0 = [rng.standard_normal(n) for n in sizes]
    for off, n, p in zip(offs, sizes, p0):
        big_p[off:off + n] = torch.from_numpy(p).float().cuda()
    ps = [big_p[off:off + n] for off, n in zip(offs, sizes)]
    ms = [big_m[off:off + n] for off, n in zip(offs, sizes)]
    vs = [big_v[off:off + n] for off, n in zip(offs, sizes)]
    o_p = [host64(p) for p in ps]
    o_m = [np.zeros(n) for n in sizes]
    o_v = [np.zeros(n) for n in sizes]
    for t in (1, 2):
        gs = [torch.from_numpy(rng.standard_normal(n)).float().cuda() for n in sizes]
        gs[2] = None   # skipped tensor
        ns.adamw_step(ps, gs, ms, vs, step=t, lr=1e-2, weight_decay=0.1)
        oracle.adamw_step([o_p[i] for i in range(len(sizes)) if i != 2],
                          [host64(g) for i, g in enumerate(gs) if i != 2],
                          [o_m[i] for i in range(len(sizes)) if i != 2],
                          [o_v[i] for i in range(len(sizes)) if i != 2], step=t, lr=1e-2, beta1=0.9,
                          beta2=0.95, eps=1e-8, weight_decay=0.1)
        torch.cuda.synchronize()
    for i in range(len(sizes)):
        assert rel(host64(ps[i]), o_p[i]) <= TOL, i
        assert rel(host64(ms[i]), o_m[i]) <= TOL or not o_m[i].any()
    assert torch.equal(ms[2], torch.zeros_like(ms[2]))
    assert np.array_equal(host64(ps[2]), p0[2].astype(np.float32).astype(np.float64))


def test_many_tensors_multi_chunk_table():
    """1,000 tensors: the AdamW tensor table exceeds one 32,000-byte kernel-parameter chunk and is
    written in several launches; every tensor is checked."""
    import newton_schulz_13_b200 as ns
    rng = np.random.default_rng(5)
    sizes = [1 + 37 * (i % 11) for i in range(1000)]
    p0 = [rng.standard_normal(n).astype(np.float32) for n in sizes]
    g = [rng.standard_normal(n).astype(np.float32) for n in sizes]
    ps = [to_dev(x, torch.float32) for x in p0]
    ms = [torch.zeros(n, device="cuda") for n in sizes]
    vs = [torch.zeros(n, device="cuda") for n in sizes]
    # the C ABI takes the hyper-parameters as floats: the oracle gets the same fp32 values (with
    # beta2 = 0.999, 1 - fp32(beta2) differs from 0.001 by 1.3e-5 relative, and so does v)
    hp = {k: float(np.float32(v)) for k, v in
          dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01).items()}
    ns.adamw_step(ps, [to_dev(x, torch.float32) for x in g], ms, vs, step=1, **hp)
    o_p = [x.astype(np.float64) for x in p0]
    o_m = [np.zeros(n) for n in sizes]
    o_v = [np.zeros(n) for n in sizes]
    oracle.adamw_step(o_p, [x.astype(np.float64) for x in g], o_m, o_v, step=1, **hp)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    for i in range(len(sizes)):
        for dev, ref in ((ps[i], o_p[i]), (ms[i], o_m[i]), (vs[i], o_v[i])):
            assert rel(host64(dev), ref) <= TOL, i

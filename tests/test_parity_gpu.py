"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, element by element, on
seeded inputs: Newton-Schulz alone over many shapes and schedules, and the whole Muon step on
the small workloads."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import (TOL_M, TOL_O_BF16, TOL_O_FP32, TOL_P, StepCase, host64, rel, tdtype,
                            to_dev)

pytestmark = pytest.mark.gpu

Q5 = [synth.QUINTIC] * 5
C5 = [synth.CUBIC] * 5

# wide, tall, square, ragged tails, single row/column, several tiles in every dimension
NS_SHAPES = [(256, 512), (512, 256), (300, 700), (700, 300), (129, 129), (1, 7), (7, 1),
             (33, 17), (80, 1536), (1536, 48), (640, 640), (384, 1000)]
SCHEDULES = {"quintic5": Q5, "cubic5": C5, "hybrid10": synth.HYBRID, "quintic1": Q5[:1],
             "steps0": [], "a_only": [(2.0, 0.0, 0.0)], "b_only": [(0.0, 1.0, 0.0)],
             "c_only": [(0.0, 0.0, 1.0)]}


def _gen(shape, seed, scale=None):
    rng = np.random.default_rng(seed)
    G = rng.standard_normal(shape)
    if scale:
        G *= np.exp(rng.uniform(np.log(scale[0]), np.log(scale[1]), size=shape[1]))[None, :]
    return G


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import newton_schulz_13_b200  # noqa: F401  (fails loudly if the library is missing)
    yield


@pytest.mark.parametrize("shape", NS_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("sched", list(SCHEDULES), ids=str)
@pytest.mark.parametrize("gdt", ["fp32", "bf16"])
def test_ns_orthogonalize_bf16(shape, sched, gdt):
    import newton_schulz_13_b200 as ns
    co = SCHEDULES[sched]
    G = synth.round_to(_gen(shape, 7, (1e-2, 1.0)), gdt)
    Gd = to_dev(G, tdtype(gdt))
    X = ns.ns_orthogonalize(Gd, steps=len(co), coeffs=co, eps=1e-7, prec="bf16", out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    want = oracle.newton_schulz(G, co, eps=1e-7)
    got = host64(X)
    assert np.all(np.isfinite(got))
    assert rel(got, want) <= TOL_O_BF16, rel(got, want)


@pytest.mark.parametrize("shape", NS_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("sched", ["quintic5", "cubic5", "steps0", "c_only"], ids=str)
def test_ns_orthogonalize_fp32(shape, sched):
    import newton_schulz_13_b200 as ns
    co = SCHEDULES[sched]
    G = synth.round_to(_gen(shape, 11), "fp32")
    X = ns.ns_orthogonalize(to_dev(G, torch.float32), steps=len(co), coeffs=co, eps=1e-7, prec="fp32")
    want = oracle.newton_schulz(G, co, eps=1e-7)
    assert rel(host64(X), want) <= TOL_O_FP32, rel(host64(X), want)


@pytest.mark.parametrize("shape", [(1 << 20, 16), (16, 1 << 20), (2, 1 << 20)], ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("sched", ["quintic5", "cubic5"], ids=str)
@pytest.mark.parametrize("prec,tol", [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)], ids=["bf16", "fp32"])
def test_ns_largest_single_dimension(shape, sched, prec, tol):
    """The largest row or column count the C ABI accepts (2^20), on thin matrices the oracle still
    finishes in a second: Gram contractions over a million-long K, 4096 row tiles of the update."""
    import newton_schulz_13_b200 as ns
    co = SCHEDULES[sched]
    G = synth.round_to(_gen(shape, 17), "bf16")
    X = ns.ns_orthogonalize(to_dev(G, torch.bfloat16), steps=len(co), coeffs=co, eps=1e-7, prec=prec,
                            out_dtype=torch.float32)
    assert ns.check_status() == ns.OK
    want = oracle.newton_schulz(G, co, eps=1e-7)
    assert rel(host64(X), want) <= tol, rel(host64(X), want)


@pytest.mark.parametrize("shape", [(33, 17), (300, 701), (701, 300), (520, 520)], ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("offset", [0, 1], ids=["aligned", "offset1"])
def test_step_fp32_mode_ragged_and_unaligned_params(shape, offset):
    """fp32 mode fuses the parameter update into the last Newton-Schulz product with plain loads and
    stores: rows whose length is not a multiple of 4 floats, and parameter matrices that start one
    float past a 16-byte boundary, take the scalar path of that epilogue."""
    import newton_schulz_13_b200 as ns
    r, c = shape
    rng = np.random.default_rng(23)
    p0 = synth.round_to(0.02 * rng.standard_normal((r, c)), "fp32")
    g = synth.round_to(rng.standard_normal((r, c)), "fp32")
    store = torch.zeros(r * c + offset, dtype=torch.float32, device="cuda")
    p = store[offset:].view(r, c)
    p.copy_(torch.from_numpy(p0))
    m = torch.zeros((r, c), dtype=torch.float32, device="cuda")
    lr, wd = 0.02, 0.1
    ns.muon_step([p], [to_dev(g, torch.float32)], [m], lr=lr, mu=0.95, nesterov=True, weight_decay=wd,
                 rms_scale=1, steps=5, coeffs=Q5, eps=1e-7, prec="fp32")
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    o_p, o_m = p0.astype(np.float64).copy(), np.zeros((r, c))
    O_ref = oracle.muon_step([o_p], [g], [o_m], lr=lr, mu=0.95, nesterov=True, weight_decay=wd,
                             rms_mode=1, coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
    s = np.sqrt(max(1.0, r / c))
    decay = np.float64(np.float32(1.0 - np.float32(lr) * np.float32(wd)))
    O_gpu = (p0 * decay - host64(p)) / (np.float64(np.float32(lr)) * s)
    assert rel(O_gpu, O_ref) <= TOL_O_FP32, rel(O_gpu, O_ref)
    assert rel(host64(p), o_p) <= TOL_P
    assert rel(host64(m), o_m) <= TOL_M


@pytest.mark.parametrize("shape", [(96, 200), (200, 96), (64, 64)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_ns_zero_center(shape):
    import newton_schulz_13_b200 as ns
    G = synth.round_to(_gen(shape, 3) + 2.0, "fp32")
    for prec, tol in (("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)):
        X = ns.ns_orthogonalize(to_dev(G, torch.float32), steps=5, coeffs=Q5, zero_center=True, prec=prec,
                                out_dtype=torch.float32)
        want = oracle.newton_schulz(G, Q5, zero_center=True, eps=1e-7)
        assert rel(host64(X), want) <= tol


def _check_step(case: StepCase, step: int, prec: str, tol_o: float):
    wl = case.wl
    p_prev = {j: host64(case.params[j]) for j in case.sample}
    _, O_ref = case.step(step, prec=prec)
    torch.cuda.synchronize()
    decay = 1.0 - np.float32(wl.lr) * np.float32(wl.weight_decay)
    for j in case.sample:
        p_new = host64(case.params[j])
        assert np.all(np.isfinite(p_new))
        e_p = rel(p_new, case.o_params[j])
        e_m = rel(host64(case.momentum[j]), case.o_mom[j])
        O_gpu = (p_prev[j] * np.float64(np.float32(decay)) - p_new) / (np.float64(np.float32(wl.lr)) * case.rms(j))
        e_o = rel(O_gpu, O_ref[j])
        assert e_m <= TOL_M, (j, "momentum", e_m)
        assert e_o <= tol_o, (j, "O", e_o)
        assert e_p <= TOL_P, (j, "params", e_p)
        # keep the oracle on the device's trajectory only through its own state: no resync


@pytest.mark.parametrize("prec,tol", [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)])
def test_step_single_256x512(prec, tol):
    wl = synth.WORKLOADS["single_256x512"]
    case = StepCase(wl, sample=[0])
    _check_step(case, 0, prec, tol)


def test_step_zero_gradient_only_decays():
    import newton_schulz_13_b200 as ns
    p = torch.randn(64, 96, device="cuda")
    p0 = p.clone()
    g = torch.zeros(64, 96, device="cuda")
    m = torch.zeros(64, 96, device="cuda")
    ns.muon_step([p], [g], [m], lr=0.02, mu=0.95, weight_decay=0.1)
    assert ns.check_status() == ns.OK
    assert torch.isfinite(p).all()
    torch.testing.assert_close(p, p0 * (1 - 0.02 * 0.1), rtol=1e-6, atol=0)


def test_step_nonfinite_is_reported():
    import newton_schulz_13_b200 as ns
    p = torch.randn(32, 48, device="cuda")
    g = torch.randn(32, 48, device="cuda")
    g[3, 5] = float("nan")
    m = torch.zeros_like(p)
    ns.muon_step([p], [g], [m])
    assert ns.check_status() == ns.WARN_NONFINITE
    assert ns.check_status() == ns.OK   # the status word was cleared


def test_step_is_deterministic():
    import newton_schulz_13_b200 as ns
    wl = synth.WORKLOADS["mamba_24"]
    shapes = wl.shapes[:8]
    outs = []
    for _ in range(2):
        ps = [to_dev(wl.param(j), torch.float32) for j in range(8)]
        ms = [torch.zeros(s, device="cuda") for s in shapes]
        gs = [to_dev(wl.grad(j, 0), torch.bfloat16) for j in range(8)]
        for _s in range(2):
            ns.muon_step(ps, gs, ms, lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        outs.append([p.cpu() for p in ps] + [m.cpu() for m in ms])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_null_grad_skips_matrix():
    import newton_schulz_13_b200 as ns
    ps = [torch.randn(40, 70, device="cuda") for _ in range(3)]
    ms = [torch.zeros(40, 70, device="cuda") for _ in range(3)]
    before = [p.clone() for p in ps]
    gs = [torch.randn(40, 70, device="cuda"), None, torch.randn(40, 70, device="cuda")]
    ns.muon_step(ps, gs, ms)
    torch.cuda.synchronize()
    assert torch.equal(ps[1], before[1]) and torch.equal(ms[1], torch.zeros_like(ms[1]))
    assert not torch.equal(ps[0], before[0]) and not torch.equal(ps[2], before[2])


@pytest.mark.parametrize("prec,tol", [("bf16", TOL_O_BF16), ("fp32", TOL_O_FP32)], ids=["bf16", "fp32"])
def test_step_many_matrices_multi_chunk_tables(prec, tol):
    """600 small matrices: the per-call tables (matrix records, fused-update problems and, in bf16
    mode, the parameters' TMA views) exceed one 32,000-byte kernel-parameter chunk and are written
    in several launches. Every matrix is checked, so a chunk written to the wrong place shows."""
    import newton_schulz_13_b200 as ns
    rng = np.random.default_rng(31)
    shapes = [(16 + 8 * (j % 5), 24 + 8 * (j % 7)) for j in range(600)]
    p0 = [synth.round_to(0.02 * rng.standard_normal(s), "fp32") for s in shapes]
    g = [synth.round_to(rng.standard_normal(s), "fp32") for s in shapes]
    ps = [to_dev(x, torch.float32) for x in p0]
    ms = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    ns.muon_step(ps, [to_dev(x, torch.float32) for x in g], ms, lr=0.02, mu=0.95, nesterov=True,
                 weight_decay=0.0, steps=5, coeffs=Q5, eps=1e-7, prec=prec)
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    for j, s in enumerate(shapes):
        o_p, o_m = p0[j].astype(np.float64).copy(), np.zeros(s)
        O_ref = oracle.muon_step([o_p], [g[j]], [o_m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.0,
                                 rms_mode=0, coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
        O_gpu = (p0[j].astype(np.float64) - host64(ps[j])) / np.float64(np.float32(0.02))
        assert rel(O_gpu, O_ref) <= tol, (j, rel(O_gpu, O_ref))
        assert rel(host64(ms[j]), o_m) <= TOL_M, j


@pytest.mark.parametrize("shape", [(2100, 3000), (3000, 2100), (2304, 2344)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_ns_wide_tiles_ragged(shape):
    """Matrices with min(rows, cols) >= 2048 run their Gram and update products on 256 x 512 tiles:
    ragged row and column counts (not multiples of 256 or 512), wide and tall, against the oracle."""
    import newton_schulz_13_b200 as ns
    G = synth.round_to(_gen(shape, 41, (1e-2, 1.0)), "bf16")
    X = ns.ns_orthogonalize(to_dev(G, torch.bfloat16), steps=5, coeffs=Q5, eps=1e-7, prec="bf16",
                            out_dtype=torch.float32)
    assert ns.check_status() == ns.OK
    want = oracle.newton_schulz(G, Q5, eps=1e-7)
    assert rel(host64(X), want) <= TOL_O_BF16, rel(host64(X), want)


def test_step_wide_tiles_fused_update_ragged():
    """The fused parameter update on 256 x 512 tiles with ragged edges (2100 x 2600, tall 2600 x 2100)."""
    import newton_schulz_13_b200 as ns
    shapes = [(2100, 2600), (2600, 2100)]
    rng = np.random.default_rng(43)
    p0 = [synth.round_to(0.02 * rng.standard_normal(s), "fp32") for s in shapes]
    g = [synth.round_to(rng.standard_normal(s), "bf16") for s in shapes]
    ps = [to_dev(x, torch.float32) for x in p0]
    ms = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    ns.muon_step(ps, [to_dev(x, torch.bfloat16) for x in g], ms, lr=0.02, mu=0.95, nesterov=True,
                 weight_decay=0.1, rms_scale=1, steps=5, coeffs=Q5, eps=1e-7, prec="bf16")
    torch.cuda.synchronize()
    assert ns.check_status() == ns.OK
    decay = np.float64(np.float32(1.0 - np.float32(0.02) * np.float32(0.1)))
    for j, s in enumerate(shapes):
        o_p, o_m = p0[j].astype(np.float64).copy(), np.zeros(s)
        O_ref = oracle.muon_step([o_p], [g[j]], [o_m], lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1,
                                 rms_mode=1, coeffs=Q5, zero_center=False, eps=1e-7, want_O=True)[0]
        rms = np.sqrt(max(1.0, s[0] / s[1]))
        O_gpu = (p0[j] * decay - host64(ps[j])) / (np.float64(np.float32(0.02)) * rms)
        assert rel(O_gpu, O_ref) <= TOL_O_BF16, (j, rel(O_gpu, O_ref))
        assert rel(host64(ps[j]), o_p) <= TOL_P, j

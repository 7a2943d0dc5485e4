"""The no-allocation Newton-Schulz entry point, muon_ns_orthogonalize_noalloc.

It exists for callers that cannot allocate device memory while they run (a plugin or custom-call
hook whose framework owns every allocation, or a service that reserves its memory at start-up):
it works in a fixed scratch array compiled into the library instead of a cudaMalloc'd
workspace. These tests call it through the C ABI and compare it with the allocating
muon_ns_orthogonalize on two calls in a row, and with the fp64 oracle, within the bf16
tolerance the other parity tests use, including matrices at the limits of the scratch layout.
This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import ns_blas

pytestmark = pytest.mark.gpu

TOL_O_BF16 = 3e-2
QUINTIC5 = [(3.4445, -4.7750, 2.0315)] * 5


def _entry():
    import newton_schulz_13_b200 as ns
    f = ns.lib.muon_ns_orthogonalize_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ns.Coeffs), ctypes.c_float,
                  ctypes.c_void_p, ctypes.c_void_p]
    return ns, f


def _coeffs(ns, co):
    arr = (ns.Coeffs * len(co))()
    for k, (a, b, c) in enumerate(co):
        arr[k] = ns.Coeffs(a, b, c)
    return arr


def _rel(a: torch.Tensor, b: torch.Tensor) -> float:
    a64, b64 = a.double(), b.double()
    return float((a64 - b64).norm() / b64.norm())


def test_noalloc_matches_allocating_entry_point_on_two_calls():
    assert torch.cuda.is_available()
    ns, f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(1234)
    # two calls in a row: a wide fp32 input, then a tall bf16 input with a cubic tail
    cases = [((300, 700), torch.float32, QUINTIC5),
             ((1000, 96), torch.bfloat16, QUINTIC5[:3] + [(1.5, -0.5, 0.0)] * 2)]
    for (r, c), dt, co in cases:
        G = (torch.randn(r, c, device="cuda", generator=gen) *
             torch.rand(1, c, device="cuda", generator=gen)).to(dt).contiguous()
        X_na = torch.empty(r, c, dtype=torch.float32, device="cuda")
        rc = f(G.data_ptr(), ns.BF16 if dt == torch.bfloat16 else ns.FP32, X_na.data_ptr(), ns.FP32, r, c,
               len(co), _coeffs(ns, co), 1e-7, status.data_ptr(), stream)
        assert rc == ns.OK, ns.last_error()
        X_ref = ns.ns_orthogonalize(G, steps=len(co), coeffs=co, eps=1e-7, prec="bf16",
                                    out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        assert torch.isfinite(X_na).all()
        assert _rel(X_na, X_ref) <= TOL_O_BF16
        want = ns_blas.newton_schulz(G.double().cpu().numpy(), co, eps=1e-7)
        assert _rel(X_na.cpu(), torch.from_numpy(want)) <= TOL_O_BF16


def test_noalloc_call_does_not_grow_device_memory_and_rejects_oversize():
    assert torch.cuda.is_available()
    ns, f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    G = torch.randn(256, 512, device="cuda")
    X = torch.empty_like(G)
    co = _coeffs(ns, QUINTIC5)
    assert f(G.data_ptr(), ns.FP32, X.data_ptr(), ns.FP32, 256, 512, 5, co, 1e-7, None, stream) == ns.OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert f(G.data_ptr(), ns.FP32, X.data_ptr(), ns.FP32, 256, 512, 5, co, 1e-7, None, stream) == ns.OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    big = torch.empty(1100, 1100, device="cuda")
    out = torch.empty_like(big)
    rc = f(big.data_ptr(), ns.FP32, out.data_ptr(), ns.FP32, 1100, 1100, 5, co, 1e-7, None, stream)
    assert rc == ns.ERR_INVALID_ARG and "scratch" in ns.last_error()


# the largest accepted sizes in both orientations (min(m, n) = 1024, m * round_up(n, 8) = 2^21),
# a ragged one just under the limit (1016 * 2056 = 2,088,896 elements), a bf16 output and steps = 0
LIMIT_CASES = [((1024, 2048), torch.float32, torch.float32, 5),
               ((2048, 1024), torch.bfloat16, torch.bfloat16, 5),
               ((1016, 2050), torch.float32, torch.bfloat16, 5),
               ((2050, 1016), torch.bfloat16, torch.float32, 5),
               ((300, 700), torch.float32, torch.float32, 0)]


@pytest.mark.parametrize("shape,gdt,xdt,steps", LIMIT_CASES,
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_noalloc_at_the_scratch_limits(shape, gdt, xdt, steps):
    ns, f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    r, c = shape
    gen = torch.Generator(device="cuda").manual_seed(r * 7 + c)
    G = (torch.randn(r, c, device="cuda", generator=gen) *
         torch.rand(1, c, device="cuda", generator=gen)).to(gdt).contiguous()
    co = QUINTIC5[:steps]
    # the output sits between guard bands that must stay untouched
    band = 2048
    store = torch.full((band + r * c + band,), -7.0, dtype=xdt, device="cuda")
    X_na = store[band:band + r * c].view(r, c)
    rc = f(G.data_ptr(), ns.BF16 if gdt == torch.bfloat16 else ns.FP32, X_na.data_ptr(),
           ns.BF16 if xdt == torch.bfloat16 else ns.FP32, r, c, steps, _coeffs(ns, co) if steps else None, 1e-7,
           status.data_ptr(), stream)
    assert rc == ns.OK, ns.last_error()
    X_ref = ns.ns_orthogonalize(G, steps=steps, coeffs=co if steps else None, eps=1e-7, prec="bf16",
                                out_dtype=xdt)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    assert torch.all(store[:band] == -7.0) and torch.all(store[band + r * c:] == -7.0)
    assert torch.isfinite(X_na).all()
    # a bf16 output adds one rounding (2^-9 relative) on top of the bf16 working precision
    tol = TOL_O_BF16 + (4e-3 if xdt == torch.bfloat16 else 0.0)
    assert _rel(X_na, X_ref) <= tol
    want = ns_blas.newton_schulz(G.double().cpu().numpy(), co, eps=1e-7)
    assert _rel(X_na.cpu(), torch.from_numpy(want)) <= tol

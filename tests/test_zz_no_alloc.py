"""The no-allocation Newton-Schulz entry point, muon_ns_orthogonalize_noalloc.

It exists for callers that cannot allocate device memory while they run (a plugin or custom-call
hook whose framework owns every allocation, or a service that reserves its memory at start-up):
it works in a fixed scratch array compiled into the library instead of a cudaMalloc'd
workspace. These tests call it through the C ABI and compare it with the allocating
muon_ns_orthogonalize on two calls in a row, within the bf16 tolerance the other parity tests
use. This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

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

"""The C ABI without a GPU: the library loads, exports every symbol the header declares, rejects
bad arguments before touching a device, and fails loudly (no fallback) when no sm_100 device
is present."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("muon_ns_orthogonalize", "muon_step", "muon_last_error", "muon_check_status",
              "muon_release_workspace", "muon_profile_enable", "muon_profile_read", "muon_launch_count",
              "muon_version", "muon_ns_orthogonalize_noalloc", "muon_adamw_step"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import newton_schulz_13_b200 as ns
    out = subprocess.run(["nm", "-D", "--defined-only", ns.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(muon_\w+)$", out, flags=re.M))
    for n in declared_symbols():
        assert n in exported, n
        assert getattr(ns.lib, n) is not None
    # nothing else leaks out of the library
    assert exported == set(declared_symbols())


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "muon.h"\nint main(void){ return muon_version() > 0 ? 0 : 1; }\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-c", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(tmp_path / "use.o")])


def _step(ns, count=1, params=None, grads=None, mom=None, rows=None, cols=None, lr=0.02, mu=0.95,
          wd=0.0, steps=5, eps=1e-7, gdt=0, prec=0, rms=0):
    VP = ctypes.c_void_p * max(count, 1)
    I64 = ctypes.c_int64 * max(count, 1)
    P = VP(*(params or [0x10000 * (i + 1) for i in range(count)]))
    G = VP(*(grads or [0x90000000 + 0x10000 * i for i in range(count)]))
    M = VP(*(mom or [0x50000000 + 0x10000 * i for i in range(count)]))
    R = I64(*(rows or [4] * count))
    C = I64(*(cols or [4] * count))
    cast = lambda a: ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))
    return ns.lib.muon_step(count, cast(P), cast(G), gdt, cast(M), R, C, lr, mu, 1, wd, rms, steps, None, 0,
                            eps, prec, None)


@pytest.mark.parametrize("kw,needle", [
    (dict(count=-1), "count"),
    (dict(mu=1.0), "mu"),
    (dict(mu=-0.1), "mu"),
    (dict(eps=-1.0), "eps"),
    (dict(eps=float("nan")), "eps"),
    (dict(lr=float("inf")), "lr"),
    (dict(steps=-1), "steps"),
    (dict(steps=65), "steps"),
    (dict(gdt=7), "grad_dtype"),
    (dict(prec=9), "prec"),
    (dict(rms=5), "rms_scale"),
    (dict(rows=[0]), "positive"),
    (dict(cols=[-3]), "positive"),
    (dict(rows=[1 << 21]), "too large"),
    (dict(params=[0x1000], mom=[0x1008]), "overlap"),
    (dict(count=2, params=[0x1000, 0x2000], mom=[0x3000, 0x1004]), "overlap"),
])
def test_step_rejects_bad_arguments(kw, needle):
    import newton_schulz_13_b200 as ns
    assert _step(ns, **kw) == ns.ERR_INVALID_ARG
    assert needle in ns.last_error()


def test_null_arrays_rejected():
    import newton_schulz_13_b200 as ns
    rc = ns.lib.muon_step(1, None, None, 0, None, None, None, 0.02, 0.95, 1, 0.0, 0, 5, None, 0, 1e-7, 0, None)
    assert rc == ns.ERR_INVALID_ARG


def test_orthogonalize_rejects_bad_arguments():
    import newton_schulz_13_b200 as ns
    f = ns.lib.muon_ns_orthogonalize
    assert f(None, 0, 0x1000, 0, 4, 4, 5, None, 0, 1e-7, 0, None) == ns.ERR_INVALID_ARG
    assert f(0x1000, 0, 0x1010, 0, 4, 4, 5, None, 0, 1e-7, 0, None) == ns.ERR_INVALID_ARG   # overlap
    assert "overlap" in ns.last_error()
    assert f(0x1000, 3, 0x9000, 0, 4, 4, 5, None, 0, 1e-7, 0, None) == ns.ERR_INVALID_ARG
    assert f(0x1000, 0, 0x9000, 0, 0, 4, 5, None, 0, 1e-7, 0, None) == ns.ERR_INVALID_ARG
    bad = (ns.Coeffs * 1)(ns.Coeffs(float("nan"), 0, 0))
    assert f(0x1000, 0, 0x9000, 0, 4, 4, 1, bad, 0, 1e-7, 0, None) == ns.ERR_INVALID_ARG
    assert "finite" in ns.last_error()


def test_noalloc_rejects_oversize_before_device_work():
    import newton_schulz_13_b200 as ns
    f = ns.lib.muon_ns_orthogonalize_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_int, ctypes.POINTER(ns.Coeffs), ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    assert f(0x1000, 1, 0x100000000, 1, 1025, 1025, 5, None, 1e-7, None, None) == ns.ERR_INVALID_ARG
    assert "scratch" in ns.last_error()
    assert f(0x1000, 1, 0x100000000, 1, 8, 1 << 20, 5, None, 1e-7, None, None) == ns.ERR_INVALID_ARG
    # sizes whose products would overflow 64 bits are bounded before any product is formed
    for m, n in ((8, 1 << 62), (1 << 62, 8), (8, (1 << 63) - 1), ((1 << 63) - 1, (1 << 63) - 1)):
        assert f(0x1000, 1, 0x100000000, 1, m, n, 5, None, 1e-7, None, None) == ns.ERR_INVALID_ARG, (m, n)
        assert "scratch" in ns.last_error()


PER_DEVICE_ONCE_CHECK = r"""
#include <cstdio>
#include "device_once.h"
int main() {
  muon::PerDeviceOnce once;
  int calls = 0, fail_next = 0;
  auto fn = [&] { ++calls; if (fail_next) { fail_next = 0; return 7; } return 0; };
  if (once.run(0, fn) != 0 || calls != 1 || !once.done(0)) return 1;
  if (once.run(0, fn) != 0 || calls != 1) return 2;            // device 0: done, skipped
  if (once.done(1) || once.run(1, fn) != 0 || calls != 2) return 3;   // a second device runs it
  fail_next = 1;
  if (once.run(70, fn) != 7 || calls != 3 || once.done(70)) return 4;  // a failure is not kept
  if (once.run(70, fn) != 0 || calls != 4 || !once.done(70)) return 5; // and is retried
  if (once.run(-1, fn) != 0 || once.run(-1, fn) != 0 || calls != 6) return 6;   // untracked: always
  if (once.run(muon::PerDeviceOnce::kTracked, fn) != 0 || calls != 7) return 7;
  if (!once.done(0) || !once.done(1) || once.done(2)) return 8;
  std::puts("ok");
  return 0;
}
"""


def test_kernel_attributes_are_set_once_per_device(tmp_path):
    """The bookkeeping behind the kernels' shared-memory limit (an attribute of one device's
    context): set once per device, again on every other device, retried after a failure."""
    src = tmp_path / "once.cpp"
    src.write_text(PER_DEVICE_ONCE_CHECK)
    exe = tmp_path / "once"
    subprocess.check_call(["g++", "-std=c++17", "-Wall", "-Werror", "-I",
                           os.path.join(ROOT, "newton_schulz_13_b200", "csrc"), str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.returncode


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="checks the no-device path")
def test_no_device_fails_loudly():
    import newton_schulz_13_b200 as ns
    assert _step(ns) == ns.ERR_UNSUPPORTED
    assert ns.lib.muon_ns_orthogonalize(0x1000, 0, 0x9000, 0, 4, 4, 5, None, 0, 1e-7, 0, None) == ns.ERR_UNSUPPORTED
    import torch
    with pytest.raises(ns.MuonError) as ei:
        ns.muon_step([torch.zeros(4, 4)], [torch.zeros(4, 4)], [torch.zeros(4, 4)])
    assert ei.value.code == ns.ERR_UNSUPPORTED


def test_empty_step_is_a_noop():
    import newton_schulz_13_b200 as ns
    assert ns.lib.muon_step(0, None, None, 0, None, None, None, 0.02, 0.95, 1, 0.0, 0, 5, None, 0, 1e-7, 0, None) == ns.OK


def test_profile_read_without_launches():
    import newton_schulz_13_b200 as ns
    ns.profile_enable(False)
    rec = ns.profile_read()
    assert set(rec) == set(ns.KC_NAMES) and all(v[0] == 0 for v in rec.values())
    assert ns.version() >= 100


def _adam(ns, count=1, params=None, grads=None, m=None, v=None, numel=None, step=1, lr=1e-3, b1=0.9,
          b2=0.95, eps=1e-8, wd=0.0, gdt=0):
    VP = ctypes.c_void_p * max(count, 1)
    cast = lambda a: ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))
    P = VP(*(params or [0x100000 * (i + 1) for i in range(count)]))
    G = VP(*(grads or [0x90000000 + 0x100000 * i for i in range(count)]))
    M = VP(*(m or [0x50000000 + 0x100000 * i for i in range(count)]))
    V = VP(*(v or [0x70000000 + 0x100000 * i for i in range(count)]))
    N = (ctypes.c_int64 * max(count, 1))(*(numel or [16] * count))
    return ns.lib.muon_adamw_step(count, cast(P), cast(G), gdt, cast(M), cast(V), N, step, lr, b1, b2, eps, wd, None)


@pytest.mark.parametrize("kw,needle", [
    (dict(count=-1), "count"),
    (dict(step=0), "step"),
    (dict(b1=1.0), "beta"),
    (dict(b2=-0.5), "beta"),
    (dict(eps=-1e-8), "eps"),
    (dict(lr=float("nan")), "lr"),
    (dict(gdt=5), "grad_dtype"),
    (dict(numel=[-3]), "numel"),
    (dict(params=[0x1000], m=[0x1010]), "overlap"),
    (dict(count=2, params=[0x1000, 0x9000], v=[0x20000, 0x9020]), "overlap"),
])
def test_adamw_rejects_bad_arguments(kw, needle):
    import newton_schulz_13_b200 as ns
    assert _adam(ns, **kw) == ns.ERR_INVALID_ARG
    assert needle in ns.last_error()


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="checks the no-device path")
def test_adamw_no_device_fails_loudly():
    import newton_schulz_13_b200 as ns
    assert _adam(ns) == ns.ERR_UNSUPPORTED
    assert _adam(ns, numel=[0]) == ns.OK   # nothing to do: no device needed


def test_set_wave_elements_rejects_negative_values():
    import newton_schulz_13_b200 as ns
    with pytest.raises(ns.MuonError):
        ns.set_wave_elements(-1)
    ns.set_wave_elements(1 << 20)
    ns.set_wave_elements(0)

"""Benchmark of the Muon optimizer step on B200.

One step = one call of muon_step over the whole weight set of the workload (momentum,
Nesterov, Frobenius norm, quintic Newton-Schulz x5 on the tensor cores, decoupled decay and
update) with inputs resident in HBM. Default workload: the Llama-8B hidden-weight set
(32 layers x {Wq, Wk, Wv, Wo, gate, up, down}, 224 matrices, 6.98e9 elements).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own weight set (weak scaling:
the matrices are independent problems, so there is no data-path collective); timing is the
max over ranks. Rank 0 prints one JSON line.

--impl reference times the fp64 oracle on the host cores instead (a bounded sample of the same
workload per step, scaled to matrices/s).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "Muon step matrices/s and NS TFLOP/s (bf16) vs B200 dense tensor peak, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "ns_gemm_tc_llama8b_traffic.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "newton_schulz_13_b200", "csrc", f)
                  for f in ("ns_gemm.cu", "ptx.cuh", "tile_sched.cuh", "pair_pipe.cuh")]
KERNEL_HEADER = os.path.join(ROOT, "newton_schulz_13_b200", "csrc", "muon_internal.h")


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """Hash of the bf16 tensor-core kernel's source: its .cu file, the PTX helpers, the tile
    schedule and, from the shared header, the two structures it reads (GemmProblem, EpiScalars);
    other declarations there do not count."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p) as f:
            h.update(_code_only(f.read()).encode())
    text = open(KERNEL_HEADER).read()
    for name in ("struct GemmProblem {", "struct EpiScalars {"):
        start = text.index(name)
        h.update(_code_only(text[start:text.index("};", start) + 2]).encode())
    return h.hexdigest()[:16]


def _code_only(src: str) -> str:
    """C++ source without comments and with whitespace collapsed: edits to comments or layout do
    not change the kernel, so they do not invalidate a recorded profile."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def recorded_traffic():
    """DRAM bytes per launch of the tensor-core kernel from a committed ncu summary, if it was
    taken on the current kernel source; None otherwise."""
    try:
        text = open(PROFILE_TRAFFIC).read()
    except OSError:
        return None
    src = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    val = re.search(r"dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", text)
    if not src or not val or src.group(1) != kernel_source_hash():
        return None
    return float(val.group(1))


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "200", "-i", str(self.gpu)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                mx.append(float(parts[2].split()[0]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of x over ranks (identity when world == 1)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks_ok(ok: bool, world: int, device=None) -> bool:
    """True on every rank when ok is true on every rank (one collective, taken by all ranks)."""
    return reduce_max(0.0 if ok else 1.0, world, device) == 0.0


def barrier(world: int, device=None):
    if world == 1:
        return
    import torch
    import torch.distributed as dist
    t = torch.zeros(1, device=device)
    dist.all_reduce(t)


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample_seconds(wl: synth.Workload, sample, nthreads: int):
    """Times one fp64 oracle Muon step on the sampled matrices (host-generated inputs)."""
    import numpy as np
    import oracle
    params = [synth.round_to(wl.param(j), "fp32") for j in sample]
    grads = [synth.round_to(wl.grad(j, 0), wl.grad_dtype) for j in sample]
    mom = [np.zeros(wl.shapes[j]) for j in sample]
    t0 = time.perf_counter()
    oracle.muon_step(params, grads, mom, lr=wl.lr, mu=wl.mu, nesterov=wl.nesterov,
                     weight_decay=wl.weight_decay, rms_mode=wl.rms_scale, coeffs=wl.coeffs,
                     zero_center=wl.zero_center, eps=wl.eps, nthreads=nthreads)
    return time.perf_counter() - t0


def mat_flops(shape, coeffs):
    r, c = shape
    m, n = min(r, c), max(r, c)
    return sum(4.0 * m * m * n + (2.0 * m ** 3 if cc != 0 else 0.0) for (_, _, cc) in coeffs)


def cpu_sample_for(wl: synth.Workload, budget: float = 3.0e11):
    """Matrices timed for the CPU leg: the smallest-FLOP shapes of the first layer, up to
    `budget` Newton-Schulz FLOPs (3e11 is roughly 10 s of fp64 work on a 16-core host)."""
    order = sorted(range(min(wl.count, max(wl.layer_size, 1))), key=lambda j: mat_flops(wl.shapes[j], wl.coeffs))
    out, tot = [], 0.0
    for j in order:
        f = mat_flops(wl.shapes[j], wl.coeffs)
        if out and tot + f > budget:
            break
        out.append(j)
        tot += f
    return out


def cpu_baseline(wl: synth.Workload, nthreads: int):
    sample = cpu_sample_for(wl)
    secs = oracle_sample_seconds(wl, sample, nthreads)
    f_sample = sum(mat_flops(wl.shapes[j], wl.coeffs) for j in sample)
    f_all = sum(mat_flops(s, wl.coeffs) for s in wl.shapes)
    step_secs = secs * f_all / f_sample
    desc = (f"fp64 oracle step on matrices {sample} ({', '.join('%dx%d' % wl.shapes[j] for j in sample)}) of "
            f"layer 0 in {secs:.2f} s; whole-step time extrapolated by Newton-Schulz FLOPs "
            f"({f_sample:.3g} of {f_all:.3g}) to all {wl.count} matrices")
    # the single 256 x 512 matrix (quintic x5, one step) on one host thread: the oracle in seconds
    one = synth.WORKLOADS["single_256x512"]
    one_secs = min(oracle_sample_seconds(one, [0], 1) for _ in range(3))
    return {"value": wl.count / step_secs, "unit": "matrices/s", "cores": nthreads, "kind": "oracle",
            "sample": desc, "sample_seconds": secs, "extrapolated_step_seconds": step_secs,
            "single_256x512_one_thread": {"seconds": one_secs, "threads": 1,
                                          "sample": "one fp64 oracle Muon step of the single 256x512 "
                                                    "matrix on one host thread (best of 3)"}}


# ----------------------------------------------------------------------------- ours
def run_ours(args, world, rank, local):
    import torch
    import newton_schulz_13_b200 as ns

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    ns.set_wave_elements(args.wave_elements)
    ns.set_chained_launch(args.chained_launch)
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)
    wl = synth.WORKLOADS[args.workload]
    if not args.sharded:
        # every rank owns an independent weight set of the same shapes (weak scaling)
        wl = synth.Workload(**{**wl.__dict__, "seed": wl.seed + 1000 * rank})
        owner = [rank] * wl.count
    else:
        # one weight set replicated on every rank; each rank updates its share of the matrices
        # and the updated parameters are all-gathered, group by group, overlapping the compute
        # (strong scaling); the parameters are views of the sharded layout's flat buffer
        from newton_schulz_13_b200 import sharded
        sm = sharded.ShardedMuon(wl.shapes, device)
        owner = sm.owner
    gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
    params, grads, mom = [], [], []
    for j in range(wl.count):
        if args.sharded:
            sm.params[j].copy_(wl.param_torch(j, device))
            params.append(sm.params[j])
        else:
            params.append(wl.param_torch(j, device).to(torch.float32))
        grads.append(wl.grad_torch(j, 0, device).to(gdt))
        mom.append(torch.zeros(wl.shapes[j], dtype=torch.float32, device=device) if owner[j] == rank else None)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    hp = dict(lr=wl.lr, mu=wl.mu, nesterov=wl.nesterov, weight_decay=wl.weight_decay, rms_scale=wl.rms_scale,
              steps=len(wl.coeffs), coeffs=wl.coeffs, zero_center=wl.zero_center, eps=wl.eps, prec=args.prec,
              stream=stream)

    # the step as one muon_step call over all matrices, or as one call per group of whole layers
    per_call = max(1, wl.layer_size) * args.step_group_layers if args.step_group_layers > 0 else wl.count
    call_groups = [list(range(j, min(wl.count, j + per_call))) for j in range(0, wl.count, per_call)]

    def step():
        if args.sharded:
            sm.step(grads, mom, **hp)
        elif len(call_groups) == 1:
            ns.muon_step(params, grads, mom, **hp)
        else:
            for grp in call_groups:
                ns.muon_step([params[j] for j in grp], [grads[j] for j in grp], [mom[j] for j in grp], **hp)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = ns.check_status()
    ns.profile_read()
    ns.profile_enable(True)
    launches0 = ns.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(device)
    gpu_id = ("GPU-" + str(props.uuid)) if getattr(props, "uuid", None) else str(local)
    with ClockSampler(gpu_id) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world, device)
    launches = ns.launch_count() - launches0
    ms_total = reduce_max(ev0.elapsed_time(ev1), world, device)
    prof = ns.profile_read()
    ns.profile_enable(False)
    status = max(status, ns.check_status())
    ms_step = ms_total / args.steps
    value = (1 if args.sharded else world) * wl.count / (ms_step / 1e3)

    peaks, peak_src = load_peaks()
    g_launch, g_ms, g_fl, g_ex = prof["gemm"]
    achieved = g_fl / (g_ms * 1e-3) / 1e12          # TFLOP/s, algorithmic (nominal) FLOPs
    executed = g_ex / (g_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    traffic = recorded_traffic()
    fp32 = args.prec == "fp32"
    if fp32:
        # 3xTF32: three tf32 tensor-core products per fp32 product; the tf32 peak is the measured
        # bf16 peak times the nominal dense ratio (1.1 / 2.25 PFLOP/s)
        tf32_ratio = 1.1 / 2.25
        tf32_achieved = 3.0 * achieved
        tf32_peak = peak * tf32_ratio
        tf32_burst = burst * tf32_ratio
    elements = wl.elements()
    gbytes = 1 if wl.grad_dtype == "bf16" else 2
    # prologue: grad + m read + m write + bf16 U write; a separate epilogue kernel (used when the
    # parameter update is not fused into the last Newton-Schulz launch): bf16 O + p read + p write
    fused_update = prof["epilogue"][0] == 0
    xbytes = 8 if fp32 else 2   # the first iterate U: bf16, or fp32 as hi and lo tf32 planes
    ew_bytes = elements * ((2 * gbytes + 4 + 4 + xbytes) + (0 if fused_update else (xbytes + 4 + 4)))
    ew_ms = prof["prologue"][1] + prof["epilogue"][1] + prof["norm"][1] + prof["center"][1]
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    ew_achieved = ew_bytes * args.steps / (ew_ms * 1e-3) / 1e9 if ew_ms > 0 else None

    result = {
        "metric": METRIC, "value": value, "unit": "matrices/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.sharded else "weak",
        "vs_baseline": None, "dtype": "f32" if fp32 else "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "matrices_per_gpu": wl.count, "elements_per_gpu": elements,
                   "grad_dtype": wl.grad_dtype, "param_dtype": "fp32", "momentum_dtype": "fp32",
                   "ns": "quintic (3.4445, -4.7750, 2.0315) x5", "lr": wl.lr, "mu": wl.mu,
                   "ns_precision": ("fp32: 3xTF32 tensor-core products (hi/lo tf32 split), fp32 iterate"
                                    if fp32 else "bf16 operands, fp32 accumulation"),
                   "weight_decay": wl.weight_decay, "rms_scale": "sqrt(max(1, rows/cols))",
                   "l2": "no flush: inputs (params+grads+momentum, %.0f GB per GPU) are larger than the "
                         "126 MB L2" % (elements * (4 + 4 + 2 * gbytes) / 1e9),
                   "muon_step_calls_per_step": len(call_groups),
                   "wave_elements": args.wave_elements or (1 << 29),
                   "chained_launch": ("off", "auto (waves with <= 8 tiles per CTA pair per iteration)",
                                      "every wave")[args.chained_launch],
                   "parallelism": ("one weight set split across GPUs by Newton-Schulz FLOPs, updated parameters "
                                   "all-gathered (strong scaling)") if args.sharded else
                                  "independent weight set per GPU (weak scaling, no collective)"},
        "ns_tflops": achieved,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "ns_gemm_tc_kernel (all Newton-Schulz products)",
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                     "launches": g_launch, "avg_launch_ms": g_ms / max(g_launch, 1),
                     "flops_per_launch": g_fl / max(g_launch, 1),
                     "flops_definition": "nominal 4 m^2 n + 2 m^3 per quintic iteration, m = min dim",
                     "executed_tflops": executed, "frac_of_burst_peak": achieved / burst,
                     "executed_frac": executed / peak},
        "roofline_elementwise": {"bound": "hbm", "achieved": ew_achieved, "peak": hbm_peak, "unit": "GB/s",
                                 "frac": (ew_achieved / hbm_peak) if ew_achieved else None,
                                 "bytes_per_step": ew_bytes,
                                 "bytes_definition": "per element: grad + m read + m write + U write "
                                                     "(bf16, or fp32 hi and lo planes) (prologue)" + ("; the parameter update is fused into the "
                                                     "last Newton-Schulz launch" if fused_update else
                                                     ", bf16 O read + p read + p write (epilogue)"),
                                 "ms_per_step": ew_ms / args.steps},
        "kernels_ms_per_step": {k: v[1] / args.steps for k, v in prof.items()},
        "ns_phases": {ph: {"ms_per_step": prof[k][1] / args.steps,
                           "nominal_tflops": prof[k][2] / (prof[k][1] * 1e-3) / 1e12 if prof[k][1] else None,
                           "executed_tflops": prof[k][3] / (prof[k][1] * 1e-3) / 1e12 if prof[k][1] else None}
                      for ph, k in (("gram", "gemm_gram"), ("poly", "gemm_poly"), ("update", "gemm_update"))},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "status": status,
    }

    if fp32:
        result["roofline"] = {
            "bound": "tensor", "achieved": tf32_achieved, "peak": tf32_peak, "unit": "TFLOP/s",
            "frac": tf32_achieved / tf32_peak, "traffic": None,
            "kernel": "ns_gemm_x3_kernel (all Newton-Schulz products, 3xTF32)",
            "peak_source": f"{peak_src} bf16_tflops_sustained x 1.1/2.25 (nominal dense tf32/bf16 ratio)",
            "launches": g_launch, "avg_launch_ms": g_ms / max(g_launch, 1),
            "flops_per_launch": 3.0 * g_fl / max(g_launch, 1),
            "flops_definition": "3 tf32 products per fp32 product: 3 x (4 m^2 n + 2 m^3) per quintic "
                                "iteration, m = min dim",
            "fp32_equivalent_tflops": achieved, "executed_tflops": executed,
            "frac_of_burst_peak": tf32_achieved / tf32_burst, "executed_frac": executed / tf32_peak}
    if args.library_baseline:
        result["library_baseline"] = run_library_baseline(args, wl, grads, stream, world, device, prof)
    if args.e2e:
        result["e2e"] = run_e2e(args, wl, step, params, grads, mom, hp, stream, world, device)
    if args.adamw:
        result["adamw"] = run_adamw(args, ns, stream, world, device, hbm_peak, peak_src)
    if args.cpu_baseline and rank == 0 and world == 1:
        result["cpu_baseline"] = cpu_baseline(synth.WORKLOADS[args.workload], os.cpu_count() or 1)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, wl, step, params, grads, mom, hp, stream, world, device):
    """The step through the public API with host buffers: every step copies the gradients from
    pinned host memory to the device and the updated parameters back, inside the timed region.

    The copies are pipelined with the compute: the matrices are processed in groups of whole
    layers (one muon_step call per group, on the compute stream), the gradients of a group go up
    on a copy stream ahead of its call, and its updated parameters come down on a second copy
    stream as soon as its call has finished. With --sharded the whole step is one call."""
    import torch
    import newton_schulz_13_b200 as ns
    # pinned host copies of the step's inputs and results (42 GB per rank for Llama-8B); every rank
    # learns whether all of them got theirs before any collective of the measurement
    why = None
    try:
        h_grads = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in grads]
        h_params = [torch.empty(p.shape, dtype=p.dtype, pin_memory=True) for p in params]
    except RuntimeError as e:
        h_grads = h_params = None
        why = f"pinned host allocation failed: {str(e).splitlines()[0][:200]}"
    if not all_ranks_ok(why is None, world, device):
        return {"value": None, "unit": "matrices/s",
                "unavailable": why or "pinned host allocation failed on another rank"}
    for hg, g in zip(h_grads, grads):
        hg.copy_(g)
    bi = sum(g.numel() * g.element_size() for g in grads)
    bo = sum(p.numel() * p.element_size() for p in params)
    per = max(1, wl.layer_size) * max(1, args.e2e_group_layers)
    groups = [list(range(j, min(wl.count, j + per))) for j in range(0, wl.count, per)]
    if args.sharded:
        groups = [list(range(wl.count))]
    up = torch.cuda.Stream(device=device)
    down = torch.cuda.Stream(device=device)

    def e2e_step():
        ev_up = []
        for grp in groups:
            with torch.cuda.stream(up):
                for j in grp:
                    grads[j].copy_(h_grads[j], non_blocking=True)
                e = torch.cuda.Event()
                e.record(up)
                ev_up.append(e)
        for grp, e in zip(groups, ev_up):
            stream.wait_event(e)
            if args.sharded:
                step()
            else:
                ns.muon_step([params[j] for j in grp], [grads[j] for j in grp], [mom[j] for j in grp], **hp)
            done = torch.cuda.Event()
            done.record(stream)
            down.wait_event(done)
            with torch.cuda.stream(down):
                for j in grp:
                    h_params[j].copy_(params[j], non_blocking=True)
        # the step ends when its last parameters are on the host
        fin = torch.cuda.Event()
        fin.record(down)
        stream.wait_event(fin)

    e2e_step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, args.e2e_steps))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(ev0.elapsed_time(ev1), world, device) / steps
    return {"value": (1 if args.sharded else world) * wl.count / (ms / 1e3), "unit": "matrices/s",
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": ms, "steps": steps,
            "note": "grads H2D from pinned host memory and updated fp32 params D2H every step, pipelined "
                    "with the compute in groups of %d matrices (one muon_step call per group); momentum "
                    "stays resident in HBM" % (wl.count if args.sharded else per)}


def run_library_baseline(args, wl, grads, stream, world, device, prof):
    """Context only, not this library's path: the same Newton-Schulz iterations written with
    torch.matmul (cuBLAS bf16 GEMMs, one matrix after another, as the pages' listing does), timed
    on the same matrices. Compared with this library's summed Newton-Schulz launch time."""
    import torch
    Xs = []
    for g in grads:
        X = g.to(torch.bfloat16)
        X = X / (X.float().norm() + wl.eps).to(torch.bfloat16)
        Xs.append(X.T if X.shape[0] > X.shape[1] else X)

    def ns_all():
        for X in Xs:
            for a, b, c in wl.coeffs:
                A = X @ X.T
                B = b * A + c * (A @ A)
                X = a * X + B @ X

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            ns_all()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            ns_all()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = reduce_max(ev0.elapsed_time(ev1), world, device) / args.steps
    ours = prof["gemm"][1] / args.steps
    del Xs
    torch.cuda.empty_cache()
    return {"impl": "torch.matmul (cuBLAS), one matrix at a time", "ms_per_step": ms,
            "nominal_tflops": wl.ns_flops() / (ms * 1e-3) / 1e12, "ours_ns_ms_per_step": ours,
            "speedup_of_ours": ms / ours if ours else None}


def run_adamw(args, ns, stream, world, device, hbm_peak, peak_src):
    """AdamW step of the parameters the Muon step leaves out (by default the Llama-8B token
    embedding and head and 65 RMSNorm scales: 1.05e9 elements), timed on its own: one launch per
    step, HBM-bound."""
    import torch
    awl = synth.ADAM_WORKLOADS[args.adamw_workload]
    ps = [awl.param_torch(i, device).to(torch.float32) for i in range(awl.count)]
    gs = [awl.grad_torch(i, 1, device).to(torch.bfloat16) for i in range(awl.count)]
    ms = [torch.zeros_like(p) for p in ps]
    vs = [torch.zeros_like(p) for p in ps]
    torch.cuda.synchronize()
    kw = dict(lr=awl.lr, beta1=awl.beta1, beta2=awl.beta2, eps=awl.eps, weight_decay=awl.weight_decay,
              stream=stream)
    t = 0
    for _ in range(args.warmup):
        t += 1
        ns.adamw_step(ps, gs, ms, vs, step=t, **kw)
    ns.profile_read()
    ns.profile_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    ev0.record(stream)
    for _ in range(args.steps):
        t += 1
        ns.adamw_step(ps, gs, ms, vs, step=t, **kw)
    ev1.record(stream)
    torch.cuda.synchronize()
    prof = ns.profile_read()
    ns.profile_enable(False)
    ms_step = reduce_max(ev0.elapsed_time(ev1), world, device) / args.steps
    kernel_ms = prof["adamw"][1] / max(prof["adamw"][0], 1)
    elements = awl.elements()
    bytes_step = elements * (4 + 2 + 4 + 4 + 4 + 4 + 4)   # read p, g (bf16), m, v; write p, m, v
    achieved = bytes_step / (kernel_ms * 1e-3) / 1e9
    del ps, gs, ms, vs
    torch.cuda.empty_cache()
    return {"workload": awl.name, "elements": elements, "ms_per_step": ms_step,
            "kernel_ms": kernel_ms, "launches_per_step": prof["adamw"][0] / args.steps,
            "value": world * awl.count / (ms_step / 1e3), "unit": "tensors/s",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": None,
                         "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                         "bytes_definition": "26 B per element: p, bf16 g, m, v read; p, m, v written"}}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    sample = cpu_sample_for(wl, budget=1.0e11)
    f_sample = sum(mat_flops(wl.shapes[j], wl.coeffs) for j in sample)
    f_all = sum(mat_flops(s, wl.coeffs) for s in wl.shapes)
    for _ in range(args.warmup_ref):
        oracle_sample_seconds(wl, sample, cores)
    times = [oracle_sample_seconds(wl, sample, cores) for _ in range(args.steps_ref)]
    secs = sum(times) / len(times)
    step_secs = secs * f_all / f_sample
    value = wl.count / step_secs
    desc = (f"each step: fp64 oracle Muon step on matrices {sample} of layer 0, whole-step time "
            f"extrapolated by Newton-Schulz FLOPs to all {wl.count} matrices")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "matrices/s", "n_gpus": world,
           "steps": args.steps_ref, "warmup": args.warmup_ref, "ms_per_step": step_secs * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": wl.name, "matrices_per_gpu": wl.count},
           "cpu_baseline": {"value": value, "unit": "matrices/s", "cores": cores, "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": value, "unit": "matrices/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default="llama8b")
    ap.add_argument("--prec", choices=["bf16", "fp32"], default="bf16",
                    help="Newton-Schulz working precision: bf16 operands (default), or fp32 through "
                         "3xTF32 tensor-core products")
    ap.add_argument("--wave-elements", type=int, default=0,
                    help="muon_step wave budget in elements (0: the library default, 2^29)")
    ap.add_argument("--step-group-layers", type=int, default=0,
                    help="device-timed step as one muon_step call per group of this many layers "
                         "(0: one call over all matrices)")
    ap.add_argument("--chained-launch", type=int, choices=(0, 1, 2), default=1,
                    help="0: one launch per Newton-Schulz phase; 1 (default): the whole iteration of a "
                         "small wave in one launch; 2: every wave chained (see muon_set_chained_launch)")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-group-layers", type=int, default=1,
                    help="layers per muon_step call in the pipelined end-to-end measurement")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--library-baseline", action="store_true",
                    help="also time the same Newton-Schulz iterations written with torch.matmul (cuBLAS), "
                         "for context")
    ap.add_argument("--sharded", action="store_true",
                    help="split one weight set across the GPUs and all-gather the updated parameters "
                         "(strong scaling) instead of one independent weight set per GPU (weak scaling)")
    ap.add_argument("--adamw-workload", choices=sorted(synth.ADAM_WORKLOADS), default="llama8b_adamw")
    ap.add_argument("--no-adamw", dest="adamw", action="store_false",
                    help="skip the AdamW measurement on the parameters Muon leaves out")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    args.steps_ref = args.steps
    args.warmup_ref = args.warmup
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()

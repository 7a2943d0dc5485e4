"""Host logic of bench.py without a GPU: the max-over-ranks reduction and barrier on two gloo
ranks, the CPU-sample selection, FLOP accounting, clock parsing and the traffic record."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        mx = bench.reduce_max(10.0 + rank * 5.0, world)
        w, r, _ = bench.dist_setup()
        q.put((rank, mx, w, r))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 15.0, 2, 0), (1, 15.0, 2, 1)]


def _agree_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 fails a local step (e.g. a pinned host allocation): every rank must see it
        both = bench.all_ranks_ok(rank != 1, world)
        fine = bench.all_ranks_ok(True, world)
        q.put((rank, both, fine))
    finally:
        dist.destroy_process_group()


def test_all_ranks_ok_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_agree_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, False, True), (1, False, True)]


def test_single_rank_helpers_are_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.all_ranks_ok(True, 1) and not bench.all_ranks_ok(False, 1)
    bench.barrier(1)


def test_cpu_sample_and_flops():
    wl = synth.WORKLOADS["llama8b"]
    sample = bench.cpu_sample_for(wl)
    assert sample == [1, 2]   # Wk and Wv of layer 0, the smallest Newton-Schulz problems
    assert bench.cpu_sample_for(wl, budget=1e11) == [1]
    assert bench.mat_flops((1024, 4096), wl.coeffs) == 5 * (4 * 1024 ** 2 * 4096 + 2 * 1024 ** 3)
    assert sum(bench.mat_flops(s, wl.coeffs) for s in wl.shapes) == pytest.approx(wl.ns_flops())


def test_clock_summary_parsing():
    c = bench.ClockSampler("0")
    c.lines = ["0, 1200 MHz, 1965 MHz, 990.1 W, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1180 MHz, 1965 MHz, 995.0 W, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1900 MHz, 1965 MHz, 400.0 W, 0x0, Not Active, Not Active, Not Active, Not Active"]
    s = c.summary()
    assert s["sm_mhz"] == 1200 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]


def test_traffic_record_requires_current_kernel_source(tmp_path, monkeypatch):
    f = tmp_path / "t.txt"
    f.write_text(f"kernel_source_sha: {bench.kernel_source_hash()}\ndram_bytes_per_launch_full_workload: 1.5e9\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(f))
    assert bench.recorded_traffic() == 1.5e9
    f.write_text("kernel_source_sha: 0000\ndram_bytes_per_launch_full_workload: 1.5e9\n")
    assert bench.recorded_traffic() is None


def test_reference_arm_other_ranks_do_no_work(capsys):
    class A:
        workload = "single_256x512"
        steps_ref = 1
        warmup_ref = 0
    bench.run_reference(A(), world=2, rank=1)
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line(capsys):
    import json

    class A:
        workload = "single_256x512"
        steps_ref = 2
        warmup_ref = 1
    bench.run_reference(A(), world=1, rank=0)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "matrices/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"

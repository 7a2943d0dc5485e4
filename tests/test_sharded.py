"""Matrix-sharded Muon step: the ownership split, and the exchange that makes every replica
agree, run on two gloo ranks on CPU with a host-side stand-in for the local CUDA step. The GPU
test checks that one rank reproduces muon_step exactly."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from newton_schulz_13_b200 import sharded


def test_partition_covers_every_matrix_once_and_balances():
    shapes = synth.WORKLOADS["llama8b"].shapes
    for world in (1, 2, 4, 8):
        owner = sharded.partition(shapes, world)
        assert len(owner) == len(shapes) and set(owner) <= set(range(world))
        assert owner == sharded.partition(shapes, world)            # deterministic
        assert sharded.imbalance(shapes, owner, world) < 1.02, world
    assert sharded.partition([(4, 4)], 3) == [0]
    with pytest.raises(ValueError):
        sharded.partition(shapes, 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _fake_local_step(ps, gs, ms, lr=0.1, **kw):
    for p, g, m in zip(ps, gs, ms):
        m.add_(g)
        p.sub_(lr * m)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shapes = [(3, 5), (8, 8), (2, 9), (6, 4), (7, 7)]
        gen = torch.Generator().manual_seed(0)
        params = [torch.randn(s, generator=gen) for s in shapes]
        grads = [torch.randn(s, generator=gen) for s in shapes]
        want = [p - 0.1 * g for p, g in zip(params, grads)]
        mom = [torch.zeros(s) for s in shapes]
        owner = sharded.sharded_muon_step(params, grads, mom, local_step=_fake_local_step, lr=0.1)
        ok_params = all(torch.allclose(p, w, rtol=0, atol=1e-6) for p, w in zip(params, want))
        ok_mom = all(torch.equal(m, grads[j]) if owner[j] == rank else torch.equal(m, torch.zeros_like(m))
                     for j, m in enumerate(mom))
        flat = torch.cat([p.reshape(-1) for p in params])
        gathered = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(gathered, flat)
        same = all(torch.equal(gathered[0], g) for g in gathered)
        q.put((rank, ok_params, ok_mom, same, sorted(set(owner))))
    finally:
        dist.destroy_process_group()


def test_exchange_on_two_gloo_ranks():
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
    for rank, ok_params, ok_mom, same, owners in res:
        assert ok_params and ok_mom and same and owners == [0, 1], (rank, ok_params, ok_mom, same, owners)


@pytest.mark.gpu
def test_single_rank_matches_muon_step():
    import newton_schulz_13_b200 as ns
    wl = synth.WORKLOADS["mamba_24"]
    shapes = wl.shapes[:8]
    gen = torch.Generator(device="cuda").manual_seed(5)
    p_a = [torch.randn(s, device="cuda", generator=gen) * 0.02 for s in shapes]
    g = [torch.randn(s, device="cuda", generator=gen).bfloat16() for s in shapes]
    p_b = [p.clone() for p in p_a]
    m_a = [torch.zeros(s, device="cuda") for s in shapes]
    m_b = [torch.zeros(s, device="cuda") for s in shapes]
    ns.muon_step(p_a, g, m_a, lr=0.02, weight_decay=0.01)
    sharded.sharded_muon_step(p_b, g, m_b, lr=0.02, weight_decay=0.01)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(p_a, p_b))
    assert all(torch.equal(a, b) for a, b in zip(m_a, m_b))

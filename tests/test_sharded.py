"""Matrix-sharded Muon step: the ownership split, the grouped flat layout, and the per-group
exchange that makes every replica agree (each group's gather issued after that group's compute
and before the next group's), run on two gloo ranks on CPU with a host-side stand-in for the
local CUDA step. The GPU test checks that one rank, in several groups, reproduces muon_step
exactly."""
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


def test_layout_places_every_matrix_in_its_group_and_owner_slot():
    shapes = synth.WORKLOADS["llama8b"].shapes
    for world in (1, 2, 8):
        L = sharded.ShardedLayout(shapes, world)
        spans = []
        for j, (r, c) in enumerate(shapes):
            g, o = L.group_of[j], L.offset[j]
            slot0 = L.block_off[g] + L.owner[j] * L.cap[g]
            assert slot0 <= o and o + r * c <= slot0 + L.cap[g], (world, j)
            assert j in L.groups[L.owner[j]][g]
            spans.append((o, o + r * c))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))   # no two views overlap
        assert L.padding() < 0.08, (world, L.padding())
        # every rank's groups are balanced to within one matrix of the group's share
        assert L.n_groups == max(1, -(-max(sum(r * c for j, (r, c) in enumerate(shapes) if L.owner[j] == k)
                                          for k in range(world)) // (1 << 28)))
    with pytest.raises(ValueError):
        sharded.ShardedLayout(shapes, 2, group_elements=0)


def test_layout_invariants_on_random_shape_lists():
    """Any list of shapes, rank count and group size: every matrix sits inside its owner's slot
    of its group, no two views overlap, each matrix is in exactly one group of its owner, and the
    views have the matrices' shapes."""
    import random
    rng = random.Random(1234)
    for trial in range(60):
        n = rng.randint(1, 40)
        shapes = [(rng.randint(1, 3000), rng.randint(1, 3000)) for _ in range(n)]
        world = rng.randint(1, 8)
        total = sum(r * c for r, c in shapes)
        group = rng.choice([1 << 28, max(1, total // rng.randint(1, 12)), rng.randint(1, 5000)])
        L = sharded.ShardedLayout(shapes, world, group_elements=group)
        seen = {}
        for rk in range(world):
            assert len(L.groups[rk]) == L.n_groups
            for g, mats in enumerate(L.groups[rk]):
                for j in mats:
                    assert j not in seen, (trial, j)
                    seen[j] = (rk, g)
        assert sorted(seen) == list(range(n))
        spans = []
        for j, (r, c) in enumerate(shapes):
            rk, g = seen[j]
            assert rk == L.owner[j] and g == L.group_of[j]
            slot0 = L.block_off[g] + rk * L.cap[g]
            assert slot0 <= L.offset[j] and L.offset[j] + r * c <= slot0 + L.cap[g], (trial, j)
            spans.append((L.offset[j], L.offset[j] + r * c))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:])), trial
        assert L.total == sum(world * cap for cap in L.cap)
        views = L.views(torch.zeros(L.total))
        assert [tuple(v.shape) for v in views] == shapes


def test_expected_exchange_time():
    shapes = synth.WORKLOADS["llama8b"].shapes
    # 28 GB of fp32 parameters; at 8 ranks each receives 7/8 of them
    ms = sharded.expected_exchange_ms(shapes, 8, link_gbs=725.0)
    assert 30.0 < ms < 40.0, ms
    assert sharded.expected_exchange_ms(shapes, 1) == 0.0


def _fake_local_step(ps, gs, ms, lr=0.1, **kw):
    for p, g, m in zip(ps, gs, ms):
        m.add_(g)
        p.sub_(lr * m)


SHAPES = [(3, 5), (8, 8), (2, 9), (6, 4), (7, 7), (16, 3), (5, 5), (9, 2)]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        gen = torch.Generator().manual_seed(0)
        init = [torch.randn(s, generator=gen) for s in SHAPES]
        grads = [torch.randn(s, generator=gen) for s in SHAPES]
        events = []
        # small groups: three or more per rank, so the per-group ordering is exercised
        sm = sharded.ShardedMuon(SHAPES, group_elements=40, local_step=_fake_local_step, on_event=events.append)
        for p, v in zip(sm.params, init):
            p.copy_(v)
        mom = [torch.zeros(s) if sm.owner[j] == rank else None for j, s in enumerate(SHAPES)]
        results = {}
        for step in range(2):
            sm.step(grads, mom, lr=0.1)
            want = [v - 0.1 * (step + 1) * (step + 2) / 2 * g for v, g in zip(init, grads)]
            results[step] = all(torch.allclose(p, w, rtol=0, atol=1e-5) for p, w in zip(sm.params, want))
        ok_mom = all(torch.allclose(m, 2 * grads[j]) for j, m in enumerate(mom) if m is not None)
        flat = torch.cat([p.reshape(-1) for p in sm.params])
        gathered = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(gathered, flat)
        same = all(torch.equal(gathered[0], g) for g in gathered)
        G = sm.layout.n_groups
        # per step: compute g, then its gather, then compute g + 1 ...
        order = [("compute", g) if i % 2 == 0 else ("gather", g) for g in range(G) for i in range(2)]
        ok_order = events == order * 2
        q.put((rank, results[0] and results[1], ok_mom, same, ok_order, G, sorted(set(sm.owner))))
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
    for rank, ok_params, ok_mom, same, ok_order, G, owners in res:
        assert G >= 3, G
        assert ok_params and ok_mom and same and ok_order and owners == [0, 1], (rank, ok_params, ok_mom, same,
                                                                                 ok_order, owners)


@pytest.mark.gpu
def test_single_rank_matches_muon_step():
    import newton_schulz_13_b200 as ns
    wl = synth.WORKLOADS["mamba_24"]
    shapes = wl.shapes[:8]
    gen = torch.Generator(device="cuda").manual_seed(5)
    p_a = [torch.randn(s, device="cuda", generator=gen) * 0.02 for s in shapes]
    g = [torch.randn(s, device="cuda", generator=gen).bfloat16() for s in shapes]
    sm = sharded.ShardedMuon(shapes, "cuda", group_elements=1 << 20)
    for p, v in zip(sm.params, p_a):
        p.copy_(v)
    m_a = [torch.zeros(s, device="cuda") for s in shapes]
    m_b = [torch.zeros(s, device="cuda") for s in shapes]
    ns.muon_step(p_a, g, m_a, lr=0.02, weight_decay=0.01)
    sm.step(g, m_b, lr=0.02, weight_decay=0.01)
    torch.cuda.synchronize()
    assert sm.layout.n_groups >= 2
    assert all(torch.equal(a, b) for a, b in zip(p_a, sm.params))
    assert all(torch.equal(a, b) for a, b in zip(m_a, m_b))

"""Matrix-sharded Muon step across data-parallel ranks (one process per GPU).

The Muon step of one matrix needs only that matrix, so the matrices of a model are split across
the ranks: each rank runs muon_step on the matrices it owns and keeps momentum only for those,
then the updated parameters are all-gathered so that every replica holds the same weights.
Gradients are expected to be identical on all ranks already (the data-parallel all-reduce
happens before the optimizer step).

Ownership is a greedy largest-first balance of the Newton-Schulz FLOPs (4 m^2 n + 2 m^3 per
quintic iteration, m = min dim); it depends only on the shapes, so every rank computes the same
assignment without communicating. The exchange is one all_gather_into_tensor of fp32 buffers
padded to the largest rank share (NCCL over NVLink on GPUs, gloo on CPU in tests). No kernel here
reads another GPU's memory.
"""
from __future__ import annotations

import heapq
from typing import Callable, List, Optional, Sequence, Tuple


def ns_flops(shape: Tuple[int, int], steps: int = 5, quintic: bool = True) -> float:
    r, c = shape
    m, n = min(r, c), max(r, c)
    return steps * (4.0 * m * m * n + (2.0 * m ** 3 if quintic else 0.0))


def partition(shapes: Sequence[Tuple[int, int]], world: int) -> List[int]:
    """Owner rank of each matrix: largest first, each to the least-loaded rank (ties to the
    lowest rank). Deterministic for a given list of shapes."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda j: (-ns_flops(shapes[j]), j))
    heap = [(0.0, r) for r in range(world)]
    owner = [0] * len(shapes)
    for j in order:
        load, r = heapq.heappop(heap)
        owner[j] = r
        heapq.heappush(heap, (load + ns_flops(shapes[j]), r))
    return owner


def imbalance(shapes: Sequence[Tuple[int, int]], owner: Sequence[int], world: int) -> float:
    """Largest rank load divided by the mean load."""
    loads = [0.0] * world
    for s, o in zip(shapes, owner):
        loads[o] += ns_flops(s)
    mean = sum(loads) / world
    return max(loads) / mean if mean > 0 else 1.0


def sharded_muon_step(params: List, grads: List, momentum: List, group=None,
                      local_step: Optional[Callable] = None, **kw) -> List[int]:
    """One Muon step with the matrices split across the ranks of `group`.

    params: the full list of 2-D fp32 parameter tensors (replicated on every rank);
    grads: the full list of gradients (replicated); momentum: per matrix, the momentum buffer on
    the owning rank (tensors for other ranks' matrices are never touched and may be None).
    kw: the muon_step hyper-parameters. local_step replaces muon_step (tests on CPU).
    Returns the owner list."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    shapes = [tuple(p.shape) for p in params]
    owner = partition(shapes, world)
    mine = [j for j in range(len(params)) if owner[j] == rank]
    if local_step is None:
        from . import muon_step as local_step   # noqa: N813
    if mine:
        local_step([params[j] for j in mine], [grads[j] for j in mine], [momentum[j] for j in mine], **kw)
    if world == 1:
        return owner
    # pack this rank's updated matrices, gather every rank's buffer, unpack the others'
    sizes = [0] * world
    for j, o in enumerate(owner):
        sizes[o] += params[j].numel()
    cap = max(sizes)
    dev = params[0].device
    send = torch.zeros(cap, dtype=torch.float32, device=dev)
    off = 0
    for j in mine:
        n = params[j].numel()
        send[off:off + n].copy_(params[j].reshape(-1))
        off += n
    recv = torch.empty(world * cap, dtype=torch.float32, device=dev)
    dist.all_gather_into_tensor(recv, send, group=group)
    offs = [r * cap for r in range(world)]
    for j, o in enumerate(owner):
        n = params[j].numel()
        if o != rank:
            params[j].copy_(recv[offs[o]:offs[o] + n].view_as(params[j]))
        offs[o] += n
    return owner

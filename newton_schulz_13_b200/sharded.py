"""Matrix-sharded Muon step across data-parallel ranks (one process per GPU).

The Muon step of one matrix needs only that matrix, so the matrices of a model are split across
the ranks: each rank runs muon_step on the matrices it owns and keeps momentum only for those,
then the updated parameters are all-gathered so that every replica holds the same weights.
Gradients are expected to be identical on all ranks already (the data-parallel all-reduce
happens before the optimizer step).

Ownership is a greedy largest-first balance of the Newton-Schulz FLOPs (4 m^2 n + 2 m^3 per
quintic iteration, m = min dim); it depends only on the shapes, so every rank computes the same
assignment without communicating.

The exchange overlaps the compute. Each rank's matrices are cut into G groups (G is the same on
every rank; group g holds about 1/G of each rank's elements, in ownership order). Parameters live
in one flat fp32 buffer laid out group by group; the block of group g holds, for every rank r at
offset r * cap_g, rank r's matrices of that group back to back (cap_g is the largest rank share of
the group). Every parameter tensor is a view into that buffer, so the gather of group g is one
in-place all_gather_into_tensor of its block: no packing or unpacking copies. Group g's gather is
issued on a communication stream as soon as its muon_step call has been enqueued (ordered after it
by an event), so it runs while group g + 1 computes; the compute stream waits for the last gather
before the step ends. On CPU (gloo, in tests) the same sequence runs synchronously. No kernel here
reads another GPU's memory; the collectives are NCCL's.
"""
from __future__ import annotations

import heapq
from typing import Callable, Dict, List, Optional, Sequence, Tuple


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


class ShardedLayout:
    """Ownership, groups and the flat parameter layout of one list of shapes on `world` ranks.

    group_elements: the target number of elements of one group of one rank (the default, 2^28,
    is about one Llama-8B layer: at 8 ranks each rank's share then runs as four groups, and only
    the last group's gather is not hidden behind compute); the group count G is the largest over
    ranks of ceil(rank elements / group_elements), at least 1."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], world: int, group_elements: int = 1 << 28):
        if group_elements < 1:
            raise ValueError("group_elements must be >= 1")
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        self.world = world
        self.owner = partition(self.shapes, world)
        numel = [r * c for r, c in self.shapes]
        mine: List[List[int]] = [[j for j in range(len(self.shapes)) if self.owner[j] == r] for r in range(world)]
        total = [sum(numel[j] for j in mine[r]) for r in range(world)]
        G = max(1, max((-(-t // group_elements) for t in total), default=1))
        self.n_groups = G
        # cut each rank's ordered list into G runs of about total / G elements
        self.groups: List[List[List[int]]] = []     # [rank][group] -> matrix indices
        for r in range(world):
            runs: List[List[int]] = [[] for _ in range(G)]
            acc = 0
            for j in mine[r]:
                g = min(G - 1, (acc * G) // total[r]) if total[r] else 0
                runs[g].append(j)
                acc += numel[j]
            self.groups.append(runs)
        # block layout: group g starts at block_off[g] and holds world slots of cap[g] elements
        self.cap = [max(sum(numel[j] for j in self.groups[r][g]) for r in range(world)) for g in range(G)]
        self.block_off = []
        off = 0
        for g in range(G):
            self.block_off.append(off)
            off += world * self.cap[g]
        self.total = off
        self.offset: Dict[int, int] = {}              # matrix -> element offset in the flat buffer
        self.group_of: Dict[int, int] = {}
        for r in range(world):
            for g in range(G):
                o = self.block_off[g] + r * self.cap[g]
                for j in self.groups[r][g]:
                    self.offset[j] = o
                    self.group_of[j] = g
                    o += numel[j]

    def padding(self) -> float:
        """Fraction of the flat buffer that is padding (slots shorter than their group's cap)."""
        used = sum(r * c for r, c in self.shapes)
        return 1.0 - used / self.total if self.total else 0.0

    def views(self, flat) -> List:
        """The parameter tensors as views of a flat buffer of `total` elements."""
        if flat.numel() != self.total:
            raise ValueError(f"flat buffer has {flat.numel()} elements, the layout needs {self.total}")
        return [flat[self.offset[j]:self.offset[j] + r * c].view(r, c) for j, (r, c) in enumerate(self.shapes)]

    def block(self, flat, g: int):
        return flat[self.block_off[g]:self.block_off[g] + self.world * self.cap[g]]

    def slot(self, flat, g: int, rank: int):
        o = self.block_off[g] + rank * self.cap[g]
        return flat[o:o + self.cap[g]]


class ShardedMuon:
    """One Muon step with the matrices split across the ranks of `group`, the exchange of each
    group of matrices overlapping the compute of the next.

        sm = ShardedMuon(shapes, device)            # the same shapes on every rank
        params = sm.params                          # views of sm.flat; fill them once
        sm.step(grads, momentum, lr=0.02, ...)      # grads: full list; momentum: owned entries

    momentum[j] is read and written only on the rank that owns matrix j (others may be None).
    local_step replaces muon_step (host-side stand-in in CPU tests); on_event, if given, is called
    with ("compute", g) and ("gather", g) as each is issued (tests check the order)."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], device=None, group=None,
                 group_elements: int = 1 << 28, local_step: Optional[Callable] = None,
                 on_event: Optional[Callable] = None):
        import torch
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.layout = ShardedLayout(shapes, self.world, group_elements)
        self.device = torch.device(device) if device is not None else torch.device("cpu")
        self.flat = torch.zeros(self.layout.total, dtype=torch.float32, device=self.device)
        self.params = self.layout.views(self.flat)
        self._local_step = local_step
        self._on_event = on_event
        self._comm_stream = None
        if self.device.type == "cuda":
            self._comm_stream = torch.cuda.Stream(device=self.device)

    @property
    def owner(self) -> List[int]:
        return self.layout.owner

    def _note(self, what: str, g: int) -> None:
        if self._on_event is not None:
            self._on_event((what, g))

    def step(self, grads: List, momentum: List, stream=None, **kw) -> None:
        import torch
        import torch.distributed as dist
        L, rank = self.layout, self.rank
        cuda = self._comm_stream is not None
        compute = (stream if stream is not None else torch.cuda.current_stream(self.device)) if cuda else None
        if self._local_step is None:
            from . import muon_step

            def run(ps, gs, ms):
                muon_step(ps, gs, ms, stream=compute, **kw)
        else:
            def run(ps, gs, ms):
                self._local_step(ps, gs, ms, **kw)
        for g in range(L.n_groups):
            mine = L.groups[rank][g]
            self._note("compute", g)
            if mine:
                run([self.params[j] for j in mine], [grads[j] for j in mine], [momentum[j] for j in mine])
            if self.world == 1:
                continue
            self._note("gather", g)
            block = L.block(self.flat, g)
            src = L.slot(self.flat, g, rank)
            if cuda:
                ev = torch.cuda.Event()
                ev.record(compute)
                self._comm_stream.wait_event(ev)
                with torch.cuda.stream(self._comm_stream):
                    dist.all_gather_into_tensor(block, src, group=self.group)
            else:
                dist.all_gather_into_tensor(block, src, group=self.group)
        if cuda and self.world > 1:
            compute.wait_stream(self._comm_stream)


def expected_exchange_ms(shapes: Sequence[Tuple[int, int]], world: int, link_gbs: float = 725.0) -> float:
    """Time of the all-gathers of one step (fp32 parameters): each rank receives the (world - 1)
    shares of the others, at `link_gbs` GB/s of all-gather bus bandwidth per GPU."""
    total = sum(r * c for r, c in shapes) * 4.0
    return total * (world - 1) / world / (link_gbs * 1e9) * 1e3

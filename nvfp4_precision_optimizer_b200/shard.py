"""Data-parallel sharding of one model's Newton-Schulz steps across ranks.

The root step of "Full-Stack FP4" (Section 3.4, "NVFP4 Root Optimizer") acts on each
eligible matrix update on its own: no matrix's step reads another's.  So the matrices
of one model are split across the data-parallel ranks.
  * Each rank runs the direct NVFP4 step (fs4_root_ns_batched) on its share only.
  * One all-gather then gives every rank every update, as distributed Muon-style
    optimizers do.
A single matrix is never split: splitting X by columns would need an all-reduce of the
m x m Gram matrix three times per iteration.

The partition is longest-processing-time first over the step's algorithmic FLOPs
(K iterations of m(m+1)n + m(m+1)m + 2m^2 n for the short side m and long side n):
  * matrices in decreasing cost, ties by index;
  * each to the rank with the least load so far, ties to the lowest rank.
The plan depends only on the shapes, K and the world size, so every rank computes the
same plan without exchanging anything.

Buffers: each rank writes its updates straight into one flat FP32 send buffer, each
at a 256-byte aligned offset.  The send buffer is as long as the largest rank's share
and identical in size on every rank.  The all-gather lands each rank's buffer at
owner * chunk in the receive buffer.  Every update is therefore a view of the receive
buffer, with no pack or unpack copy on either side.  With one rank there is no
collective, and the updates are views of the send buffer.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Sequence

import torch

ALIGN_ELEMS = 64          # 256 B: every update starts on a 256-byte boundary


def ns_flops(shape, K: int) -> int:
    """Algorithmic FLOPs of K iterations on an m0 x n0 matrix (symmetric Gram halves)."""
    m, n = min(shape), max(shape)
    return K * (m * (m + 1) * n + m * (m + 1) * m + 2 * m * m * n)


def lpt_owners(costs: Sequence[float], world: int) -> list[int]:
    """Owner rank of each item: longest processing time first, least-loaded rank.
    Ties go to the item with the smaller index and to the lower rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0] * world
    owners = [0] * len(costs)
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owners[i] = r
        load[r] += costs[i]
    return owners


@dataclass(frozen=True)
class ShardPlan:
    shapes: tuple            # (rows, cols) of every matrix, caller's orientation
    owners: tuple            # owner rank of every matrix
    offsets: tuple           # element offset of every update in its owner's send buffer
    chunk: int               # elements per rank in the send buffer (the same on all ranks)
    loads: tuple             # algorithmic FLOPs per rank

    def local(self, rank: int) -> list[int]:
        """Indices of the matrices rank owns, in increasing order."""
        return [i for i, r in enumerate(self.owners) if r == rank]

    @property
    def imbalance(self) -> float:
        """Largest rank load over the mean load (1.0 = perfectly balanced)."""
        mean = sum(self.loads) / len(self.loads)
        return max(self.loads) / mean if mean > 0 else 1.0


def plan(shapes: Sequence[Sequence[int]], K: int, world: int) -> ShardPlan:
    """The LPT plan of one model's matrices over world ranks."""
    shapes = tuple((int(r), int(c)) for r, c in shapes)
    costs = [ns_flops(s, K) for s in shapes]
    owners = lpt_owners(costs, world)
    fill = [0] * world
    offsets = [0] * len(shapes)
    for i, (r, c) in enumerate(shapes):
        o = owners[i]
        offsets[i] = fill[o]
        fill[o] += -(-(r * c) // ALIGN_ELEMS) * ALIGN_ELEMS
    loads = [0] * world
    for i, o in enumerate(owners):
        loads[o] += costs[i]
    return ShardPlan(shapes, tuple(owners), tuple(offsets), max(max(fill), ALIGN_ELEMS), tuple(loads))


class ShardedRootNS:
    """One model's Newton-Schulz updates computed across the ranks of a process group.

    Call it with the momenta of every matrix, in the plan's order.  Entries this rank
    does not own are not read and may be None.  It returns the updates of every
    matrix: views of one receive buffer, which the next call overwrites.

    compute(Gs_local, outs_local, **call_options) runs the step on this rank's share.  The
    default is the CUDA path, fs4.root_ns_batched, with a workspace allocated once and the
    options given here (K, coeffs, clip_k, rht_masks, adaptive46, clip_quantile).  Options
    given to a call override these for that call: H16^r takes fresh sign masks every step,
    e.g. S(Gs, rht_masks=masks).  Every rank should pass the same ones.
    The collective is torch.distributed's all_gather_into_tensor on the group (NCCL
    across GPUs).  It is skipped when the group has one rank.
    """

    def __init__(self, shapes: Sequence[Sequence[int]], K: int = 5, coeffs=None, rank: int = 0,
                 world: int = 1, group=None, device="cuda",
                 compute: Callable | None = None, **ns_options):
        self.plan = plan(shapes, K, world)
        self.rank, self.world, self.group = rank, world, group
        self.local = self.plan.local(rank)
        p = self.plan
        self.send = torch.empty(p.chunk, dtype=torch.float32, device=device)
        self.recv = (torch.empty(world * p.chunk, dtype=torch.float32, device=device)
                     if world > 1 else self.send)

        def view(buf, base, i):
            r, c = p.shapes[i]
            return buf[base + p.offsets[i]:base + p.offsets[i] + r * c].view(r, c)

        self.local_outs = [view(self.send, 0, i) for i in self.local]
        self.outs = [view(self.recv, (p.owners[i] * p.chunk) if world > 1 else 0, i)
                     for i in range(len(p.shapes))]
        self.workspace = None             # the CUDA path's workspace (device status word)
        if compute is None:
            compute = self._cuda_compute(K, coeffs, device, ns_options)
        self.compute = compute

    def _cuda_compute(self, K, coeffs, device, opts):
        from . import MUON_COEFFS, ns_batched_workspace_size, root_ns_batched
        n = len(self.plan.shapes)
        coeffs = list(coeffs) if coeffs is not None else [MUON_COEFFS] * n
        if len(coeffs) != n:
            raise ValueError("one (a, b, c) per matrix")
        local_coeffs = [coeffs[i] for i in self.local]
        if self.local:
            need = ns_batched_workspace_size([self.plan.shapes[i] for i in self.local])
            self.workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)

        def compute(Gs, outs, **call_opts):
            root_ns_batched(Gs, K=K, coeffs=local_coeffs, outs=outs, workspace=self.workspace,
                            **{**opts, **call_opts})
        return compute

    def compute_local(self, Gs: Sequence[torch.Tensor | None], **call_options) -> None:
        """The step on this rank's share, into its send buffer (no collective)."""
        if len(Gs) != len(self.plan.shapes):
            raise ValueError("one momentum per matrix of the plan")
        if not self.local:
            return
        local = [Gs[i] for i in self.local]
        for i, G in zip(self.local, local):
            if G is None or tuple(G.shape) != self.plan.shapes[i]:
                raise ValueError(f"matrix {i} is owned by rank {self.rank} and must have shape "
                                 f"{self.plan.shapes[i]}")
        self.compute(local, self.local_outs, **call_options)

    def gather(self) -> list[torch.Tensor]:
        """The all-gather of every rank's send buffer; returns the updates of every matrix."""
        if self.world > 1:
            import torch.distributed as dist
            dist.all_gather_into_tensor(self.recv, self.send, group=self.group)
        return self.outs

    def __call__(self, Gs: Sequence[torch.Tensor | None], **call_options) -> list[torch.Tensor]:
        self.compute_local(Gs, **call_options)
        return self.gather()

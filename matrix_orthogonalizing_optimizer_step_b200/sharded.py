"""Muon step sharded over the ranks of a data-parallel group.

Every 2D parameter is an independent unit of work (momentum, Newton-Schulz
and update of one matrix touch no other matrix), so the step shards by whole
matrices.  With every rank holding all parameters and gradients (plain data
parallelism after the gradient all-reduce), each rank runs the library's
fused step on the matrices it owns and then the owners broadcast the updated
parameters (and, optionally, momentum buffers) so all ranks stay identical.

Ownership is a longest-processing-time partition on the algorithmic FLOPs of
the cheaper Newton-Schulz form of each matrix (the NanoGPT/Muon page's
scalability discussion names the cross-device cost of orthogonalising
sharded parameters as the open problem; whole-matrix ownership avoids
splitting any product across devices).

Collectives go through torch.distributed (NCCL over NVLink on GPUs); no
kernel of this library touches another GPU's memory.
"""
from __future__ import annotations

import heapq


def ns_cost(rows, cols, steps=5, restart_at=(2,)):
    """Algorithmic FLOPs of orthogonalising one rows x cols matrix with the
    cheaper of the standard and Gram forms (symmetric products at half cost)."""
    n, m = min(rows, cols), max(rows, cols)
    std = steps * (3 * n * n * m + n ** 3)
    starts = [0] + sorted(k for k in restart_at if 0 < k < steps)
    ends = starts[1:] + [steps]
    gram = 0
    for s, e in zip(starts, ends):
        gram += 3 * n * n * m
        for k in range(s, e):
            gram += n ** 3 + (n ** 3 if k > s else 0) + (2 * n ** 3 if k < e - 1 else 0)
    return min(std, gram)


def partition(shapes, world_size, steps=5):
    """Owner rank of each matrix: greedy longest-processing-time assignment
    (largest cost first, to the currently least-loaded rank; ties go to the
    lower rank).  Deterministic, so every rank computes the same answer."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    order = sorted(range(len(shapes)), key=lambda i: (-ns_cost(*shapes[i], steps=steps), i))
    heap = [(0, r) for r in range(world_size)]
    owner = [0] * len(shapes)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + ns_cost(*shapes[i], steps=steps), r))
    return owner


def loads(shapes, owner, world_size, steps=5):
    out = [0] * world_size
    for s, r in zip(shapes, owner):
        out[r] += ns_cost(*s, steps=steps)
    return out


def sharded_step(params, grads, momentum, *, mu=0.95, nesterov=True, lr=6e-4, group=None,
                 step_fn=None, sync_momentum=False, owner=None):
    """One Muon step over all parameters, work split across the ranks of
    `group` (torch.distributed).  `step_fn(params, grads, momentum, mu,
    nesterov, lr)` runs the local shard; it defaults to the library's C-ABI
    muon_step.  Returns the owner list used."""
    import torch.distributed as dist
    if step_fn is None:
        from . import muon_step as step_fn  # noqa: N813
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    shapes = [tuple(p.shape) for p in params]
    if owner is None:
        owner = partition(shapes, world)
    mine = [i for i, r in enumerate(owner) if r == rank]
    if mine:
        step_fn([params[i] for i in mine], [grads[i] for i in mine], [momentum[i] for i in mine],
                mu, nesterov, lr)
    if world > 1:
        ranks = dist.get_process_group_ranks(group) if group is not None else list(range(world))
        for i, r in enumerate(owner):
            dist.broadcast(params[i], src=ranks[r], group=group)
            if sync_momentum:
                dist.broadcast(momentum[i], src=ranks[r], group=group)
    return owner

"""Muon step sharded over the ranks of a data-parallel group.

Every 2D parameter is an independent unit of work (momentum, Newton-Schulz
and update of one matrix touch no other matrix), so the step shards by whole
matrices.  With every rank holding all parameters and gradients (plain data
parallelism after the gradient all-reduce), each rank runs the library's
fused step on the matrices it owns; then ONE all-gather per dtype spreads the
updated parameters (and, optionally, momentum buffers): every rank packs the
tensors it owns into its slot of a flat buffer, the collective runs in place,
and every rank copies the other ranks' slots back into its tensors.  The
collective count is independent of the number of matrices.

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


_GATHER_BUFS = {}


def release_gather_buffers():
    """Drop the flat buffers that gather_owned keeps between steps (one per
    dtype and device, as large as the padded all-gather of that dtype)."""
    _GATHER_BUFS.clear()


def _gather_buffer(numel, dtype, device):
    """A cached flat buffer of at least numel elements (reused across steps;
    release_gather_buffers frees them)."""
    key = (dtype, str(device))
    buf = _GATHER_BUFS.get(key)
    if buf is None or buf.numel() < numel:
        import torch
        buf = torch.empty(numel, dtype=dtype, device=device)
        _GATHER_BUFS[key] = buf
    return buf[:numel]


def gather_owned(tensors, owner, group=None):
    """Make every rank's `tensors` equal to their owners' copies: one in-place
    all-gather per dtype over slots padded to the largest rank's share.
    Tensors must be contiguous; packing and unpacking follow the tensors'
    index order, the same on every rank."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    by_dtype = {}
    for i, t in enumerate(tensors):
        if not t.is_contiguous():
            raise ValueError("sharded_step needs contiguous tensors")
        by_dtype.setdefault(t.dtype, []).append(i)
    for dt, idx in by_dtype.items():
        share = [0] * world
        for i in idx:
            share[owner[i]] += tensors[i].numel()
        slot = max(share)
        if slot == 0:
            continue
        flat = _gather_buffer(world * slot, dt, tensors[idx[0]].device)
        off = rank * slot
        for i in idx:
            if owner[i] == rank:
                n = tensors[i].numel()
                flat[off:off + n].copy_(tensors[i].view(-1))
                off += n
        dist.all_gather_into_tensor(flat, flat[rank * slot:(rank + 1) * slot], group=group)
        offs = [r * slot for r in range(world)]
        for i in idx:
            r, n = owner[i], tensors[i].numel()
            if r != rank:
                tensors[i].view(-1).copy_(flat[offs[r]:offs[r] + n])
            offs[r] += n


def sharded_step(params, grads, momentum, *, mu=0.95, nesterov=True, lr=6e-4, group=None,
                 step_fn=None, sync_momentum=False, owner=None):
    """One Muon step over all parameters, work split across the ranks of
    `group` (torch.distributed).  `step_fn(params, grads, momentum, mu,
    nesterov, lr)` runs the local shard; it defaults to the library's C-ABI
    muon_step.  `owner` (a rank per matrix) overrides the LPT partition.
    With a process group, the owned results are spread by gather_owned (also
    at world size 1, where the collective is a copy).  Returns the owner list
    used."""
    import torch.distributed as dist
    if step_fn is None:
        from . import muon_step as step_fn  # noqa: N813
    dist_on = dist.is_initialized()
    world = dist.get_world_size(group) if dist_on else 1
    rank = dist.get_rank(group) if dist_on else 0
    shapes = [tuple(p.shape) for p in params]
    if owner is None:
        owner = partition(shapes, world)
    if len(owner) != len(params) or any(not 0 <= r < world for r in owner):
        raise ValueError("owner must give a rank in [0, world) per parameter")
    mine = [i for i, r in enumerate(owner) if r == rank]
    if mine:
        step_fn([params[i] for i in mine], [grads[i] for i in mine], [momentum[i] for i in mine],
                mu, nesterov, lr)
    if dist_on:
        gather_owned(params, owner, group)
        if sync_momentum:
            gather_owned(momentum, owner, group)
    return owner

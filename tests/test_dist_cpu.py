"""Multi-rank host logic on CPU with the gloo backend (world size 2): the
whole-matrix partition of the sharded Muon step, its broadcast protocol, and
bench.py's max-over-ranks timing.  The GPU step itself is replaced by a
deterministic CPU stand-in here; the broadcast and ownership logic under
test is the same code that runs with NCCL."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

from matrix_orthogonalizing_optimizer_step_b200 import sharded  # noqa: E402
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_partition_balanced_and_deterministic():
    for wid in (2, 4, 5):
        shapes = list(wl.WORKLOADS[wid].shapes)
        for world in (1, 2, 4, 8):
            owner = sharded.partition(shapes, world)
            assert owner == sharded.partition(shapes, world)
            assert len(owner) == len(shapes) and set(owner) <= set(range(world))
            ld = sharded.loads(shapes, owner, world)
            biggest = max(sharded.ns_cost(*s) for s in shapes)
            # LPT bound: no rank exceeds the mean by more than the largest job
            assert max(ld) <= sum(ld) / world + biggest
    assert sharded.partition([(8, 8)], 3) == [0]
    with pytest.raises(ValueError):
        sharded.partition([(8, 8)], 0)


def test_ns_cost_matches_cheaper_form():
    from oracle import muon_oracle as orc
    for r, c in [(768, 2304), (3072, 768), (512, 512), (100, 37)]:
        n, m = min(r, c), max(r, c)
        want = min(orc.ns_flops(n, m, 5, "standard"), orc.ns_flops(n, m, 5, "gram"))
        assert sharded.ns_cost(r, c) == want


def _shapes():
    return [(8, 24), (24, 8), (16, 16), (4, 40), (12, 20), (20, 12), (6, 6)]


def _make(seed):
    # fp32 parameters and bf16 momentum: the gather runs once per dtype
    g = torch.Generator().manual_seed(seed)
    P = [torch.randn(s, generator=g) for s in _shapes()]
    G = [torch.randn(s, generator=g) for s in _shapes()]
    M = [torch.randn(s, generator=g).to(torch.bfloat16) for s in _shapes()]
    return P, G, M


def _standin_step(params, grads, momentum, mu, nesterov, lr):
    # deterministic CPU stand-in for the GPU step (host-logic test only)
    for p, g, m in zip(params, grads, momentum):
        m.copy_(m.float() * mu + g)
        u = g + mu * m.float() if nesterov else m.float()
        p.sub_(lr * u / (u.norm() + 1e-7))


def _worker(rank, world, port, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        P, G, M = _make(123)
        calls = []
        real = dist.all_gather_into_tensor

        def counting(*a, **k):
            calls.append(a[0].dtype)
            return real(*a, **k)
        dist.all_gather_into_tensor = counting
        owner = sharded.sharded_step(P, G, M, mu=0.9, nesterov=True, lr=0.1, step_fn=_standin_step,
                                     sync_momentum=True)
        dist.all_gather_into_tensor = real
        # one collective per dtype (fp32 parameters, bf16 momentum), not one per matrix
        assert calls == [torch.float32, torch.bfloat16], calls
        import bench
        mx = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        bench.barrier(world)
        assert sharded._GATHER_BUFS  # kept for the next step ...
        sharded.release_gather_buffers()
        assert not sharded._GATHER_BUFS  # ... until released
        out_q.put((rank, owner, [p.numpy().copy() for p in P], [m.float().numpy().copy() for m in M], mx))
    finally:
        dist.destroy_process_group()


def test_sharded_step_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort(key=lambda x: x[0])
    (_, own0, P0, M0, mx0), (_, own1, P1, M1, mx1) = results
    assert own0 == own1 and set(own0) == {0, 1}
    # every rank ends with the single-process result
    P, G, M = _make(123)
    _standin_step(P, G, M, 0.9, True, 0.1)
    for a, b, ref in zip(P0, P1, P):
        assert (a == b).all() and torch.allclose(torch.from_numpy(a), ref)
    for a, b, ref in zip(M0, M1, M):
        assert (a == b).all() and torch.equal(torch.from_numpy(a), ref.float())
    assert mx0 == mx1 == 3.0


def test_reference_arm_nonzero_rank_does_nothing(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload, steps, warmup, cpu_seconds, form = 2, 1, 0, 1.0, "auto"
    bench.run_reference(A())
    assert capsys.readouterr().out == ""

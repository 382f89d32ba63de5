"""Failure paths and scheduling robustness of the GPU path.

* Host-side fault injection (MUON_FAULT=alloc | launch): the call returns
  MUON_ERR_NO_MEMORY / MUON_ERR_CUDA, launches no kernel and leaves every
  caller tensor untouched; the next normal call succeeds with parity.
* A bounded device wait that runs out (MUON_FAULT=timeout gives the first
  tile of a chained launch a dependency count that no tile will reach, with
  a short MUON_WAIT_LIMIT_MS): the kernel gives up, the status word reads
  MUON_ERR_TIMEOUT, the context stays usable and the next normal call
  returns MUON_OK with parity.  Nothing faults, traps or hangs the GPU.
* The chained launch while other work holds SMs: tiles are claimed in list
  order, so the step completes and equals an unloaded run bit for bit.
* Calls alternating between two streams on independent buffers: the
  library's shared workspace is ordered across the streams.
"""
import time

import numpy as np
import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests._util import TOL_BF16_RELF, relF, to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
SHAPES = [(256, 768), (768, 256), (200, 200), (136, 520)]


@pytest.fixture(autouse=True)
def _fresh(monkeypatch):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    for k in ("MUON_FAULT", "MUON_WAIT_LIMIT_MS", "MUON_CHAIN_LAUNCH", "MUON_SLOT_LAUNCHES", "MUON_DEBUG_CANARY"):
        monkeypatch.delenv(k, raising=False)
    mo.muon_reset_config()
    mo.muon_release_workspace()
    yield
    for k in ("MUON_FAULT", "MUON_WAIT_LIMIT_MS", "MUON_CHAIN_LAUNCH", "MUON_SLOT_LAUNCHES", "MUON_DEBUG_CANARY"):
        monkeypatch.delenv(k, raising=False)
    mo.muon_release_workspace()
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_OK, (mo.STATUS_NAMES.get(st), bad)
    mo.muon_reset_config()


def _make_set(shapes, seed):
    G = [wl.make_single(r, c, seed + 3 * i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, seed + 3 * i + 1, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, seed + 3 * i + 2, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
    return W, G, M


def _step_and_check(shapes, seed, lr=0.1):
    """A normal step that must succeed and match the oracle."""
    W, G, M = _make_set(shapes, seed)
    W64, G64, M64 = [to64(t) for t in W], [to64(t) for t in G], [to64(t) for t in M]
    mo.muon_step(W, G, M, mu=0.95, nesterov=True, lr=lr)
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_OK, (mo.STATUS_NAMES.get(st), bad)
    for i in range(len(shapes)):
        _, _, O = orc.muon_step(W64[i], G64[i], M64[i], 0.95, True, lr, form="standard")
        assert relF((W64[i] - to64(W[i])) / lr, O) <= TOL_BF16_RELF, (shapes[i],)


@pytest.mark.parametrize("fault,code", [("alloc", mo.MUON_ERR_NO_MEMORY), ("launch", mo.MUON_ERR_CUDA)])
def test_injected_host_fault_enqueues_nothing(fault, code, monkeypatch):
    W, G, M = _make_set(SHAPES, 10)
    W0, M0 = [t.clone() for t in W], [t.clone() for t in M]
    torch.cuda.synchronize()
    monkeypatch.setenv("MUON_FAULT", fault)
    n0 = mo.muon_launch_count()
    with pytest.raises(mo.MuonError) as e:
        mo.muon_step(W, G, M, mu=0.95, nesterov=True, lr=0.1)
    assert e.value.code == code
    assert fault in str(e.value)
    torch.cuda.synchronize()
    assert mo.muon_launch_count() == n0
    for x, y in zip(W + M, W0 + M0):
        assert torch.equal(x, y)
    monkeypatch.delenv("MUON_FAULT")
    _step_and_check(SHAPES, 20)


def test_injected_alloc_failure_adamw(monkeypatch):
    P = [wl.make_single(1, n, 40 + i, "params", DEV, "f32").view(-1) for i, n in enumerate([4096, 1000])]
    G = [torch.ones_like(p, dtype=torch.bfloat16) for p in P]
    M1 = [torch.zeros_like(p) for p in P]
    M2 = [torch.zeros_like(p) for p in P]
    P0 = [p.clone() for p in P]
    monkeypatch.setenv("MUON_FAULT", "alloc")
    n0 = mo.muon_launch_count()
    with pytest.raises(mo.MuonError) as e:
        mo.muon_adamw_step(P, G, M1, M2, 1)
    assert e.value.code == mo.MUON_ERR_NO_MEMORY
    torch.cuda.synchronize()
    assert mo.muon_launch_count() == n0
    assert all(torch.equal(p, q) for p, q in zip(P, P0))
    monkeypatch.delenv("MUON_FAULT")
    mo.muon_adamw_step(P, G, M1, M2, 1)
    torch.cuda.synchronize()
    assert not torch.equal(P[0], P0[0])


def test_bounded_wait_runs_out_and_context_stays_usable(monkeypatch):
    monkeypatch.setenv("MUON_FAULT", "timeout")
    monkeypatch.setenv("MUON_WAIT_LIMIT_MS", "50")
    W, G, M = _make_set(SHAPES, 30)
    t0 = time.perf_counter()
    mo.muon_step(W, G, M, mu=0.95, nesterov=True, lr=0.1)  # enqueued: returns OK
    st, bad = mo.muon_device_status()                       # synchronises
    elapsed = time.perf_counter() - t0
    assert st == mo.MUON_ERR_TIMEOUT, mo.STATUS_NAMES.get(st)
    assert elapsed < 20.0  # every wait gave up after its 50 ms bound
    # the status word was cleared by the read; a normal call works again
    monkeypatch.delenv("MUON_FAULT")
    monkeypatch.delenv("MUON_WAIT_LIMIT_MS")
    mo.muon_release_workspace()
    _step_and_check(SHAPES, 40)


def test_chained_launch_under_sm_contention(monkeypatch):
    """Other kernels hold SMs while the chained step starts (a side stream of
    large matmuls, a few hundred ms of work): not every CTA pair of the launch
    is resident at once.  The step must complete without a timeout and equal
    the unloaded run bit for bit (a tile's arithmetic does not depend on which
    pair computes it)."""
    monkeypatch.setenv("MUON_CHAIN_LAUNCH", "1")
    shapes = [(768, 2304), (768, 768), (768, 3072), (3072, 768)] * 3
    W, G, M = _make_set(shapes, 50)
    Wr, Mr = [t.clone() for t in W], [t.clone() for t in M]
    mo.muon_step(Wr, G, Mr, mu=0.95, nesterov=True, lr=0.02)
    st, _ = mo.muon_device_status()
    assert st == mo.MUON_OK
    A = torch.randn(8192, 8192, device=DEV, dtype=torch.bfloat16)
    side = torch.cuda.Stream(DEV)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        for _ in range(300):
            B = A @ A
    mo.muon_step(W, G, M, mu=0.95, nesterov=True, lr=0.02)
    torch.cuda.synchronize()
    del B
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_OK, (mo.STATUS_NAMES.get(st), bad)
    for x, y in zip(W + M, Wr + Mr):
        assert torch.equal(x, y)


def test_calls_alternating_streams():
    """Independent batches orthogonalised alternately on two streams with no
    ordering between the caller's streams: every call reuses the library's
    workspace (a different buffer means a new plan), and the library orders
    each use after the previous one, so the results equal a serial run."""
    xs = [torch.stack([wl.make_single(1024, 4096, 60 + 8 * k + j, "gaussian", DEV, "bf16") for j in range(4)])
          for k in range(4)]
    ref = [x.clone() for x in xs]
    for x in ref:
        mo.muon_orthogonalize(x, steps=5, mode="gram")
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(DEV), torch.cuda.Stream(DEV)]
    got = [x.clone() for x in xs]
    torch.cuda.synchronize()
    for rnd in range(2):
        # buffer k always runs on stream k % 2, so each buffer's own calls are
        # ordered by its stream; only the workspace is shared across streams
        for k, x in enumerate(got):
            with torch.cuda.stream(streams[k % 2]):
                mo.muon_orthogonalize(x, steps=5, mode="gram")
        if rnd == 0:
            # pass 0 equals the serial reference
            torch.cuda.synchronize()
            for a, b in zip(got, ref):
                assert torch.equal(a, b)
    torch.cuda.synchronize()
    # pass 1 orthogonalised the outputs again: compare with the same on one stream
    for x in ref:
        mo.muon_orthogonalize(x, steps=5, mode="gram")
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    st, _ = mo.muon_device_status()
    assert st == mo.MUON_OK
    assert np.all(np.isfinite(to64(got[0])))


@pytest.mark.parametrize("env", [{}, {"MUON_SLOT_LAUNCHES": "1"}])
def test_step_captured_in_a_cuda_graph(env, monkeypatch):
    """A muon_step captured into a CUDA graph (after one eager call built its
    plan) and replayed three times equals four eager steps bit for bit, in
    the chained launch and with one launch per chain slot."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    mo.muon_release_workspace()  # the launch mode is chosen when a plan is built
    shapes = [(768, 2304), (768, 768), (3072, 768), (200, 712)]
    G = [wl.make_single(r, c, 700 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, 710 + i, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, 720 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    Wr, Mr = [t.clone() for t in W], [t.clone() for t in M]
    for _ in range(4):
        mo.muon_step(Wr, G, Mr, lr=0.02)
    torch.cuda.synchronize()
    mo.muon_step(W, G, M, lr=0.02)  # builds the plan of (W, G, M)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        mo.muon_step(W, G, M, lr=0.02)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(W + M, Wr + Mr):
        assert torch.equal(a, b)
    del graph
    mo.muon_release_workspace()


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")  # the refused capture enqueued nothing
def test_capture_that_needs_a_plan_is_refused():
    """Capturing a call whose plan does not exist yet fails with
    MUON_ERR_UNSUPPORTED before anything is enqueued (building a plan
    allocates and synchronises, which a capture does not allow)."""
    mo.muon_release_workspace()
    W = [wl.make_single(256, 512, 730, "params", DEV, "f32")]
    G = [wl.make_single(256, 512, 731, "student_t3", DEV, "bf16", 0.01)]
    M = [wl.make_single(256, 512, 732, "student_t3", DEV, "bf16", 0.01)]
    W0 = W[0].clone()
    graph = torch.cuda.CUDAGraph()
    with pytest.raises(mo.MuonError) as e:
        with torch.cuda.graph(graph):
            mo.muon_step(W, G, M, lr=0.02)
    assert e.value.code == mo.MUON_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(W[0], W0)
    del graph
    # outside a capture the same call builds its plan and runs
    mo.muon_step(W, G, M, lr=0.02)
    torch.cuda.synchronize()
    assert not torch.equal(W[0], W0)


def _canary_workload():
    """Steps over mixed, ragged and transposed shapes, a ragged orthogonalise
    with an unaligned row pitch, and the fp32 check path; returns every output."""
    shapes = [(768, 2304), (768, 768), (3072, 768), (200, 712), (37, 91), (136, 520), (520, 136)]
    G = [wl.make_single(r, c, 800 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, 820 + i, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, 840 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    for _ in range(2):
        mo.muon_step(W, G, M, lr=0.02)
    X = torch.stack([wl.make_single(200, 333, 860 + j, "gaussian", DEV, "bf16") for j in range(3)])
    mo.muon_orthogonalize(X, steps=5, mode="gram")
    F = torch.stack([wl.make_single(100, 260, 870 + j, "gaussian", DEV, "f32") for j in range(2)])
    mo.muon_orthogonalize(F, steps=5, mode="standard", fp32=True)
    torch.cuda.synchronize()
    return [t.clone() for t in W + M + [X, F]]


@pytest.mark.parametrize("env", [{}, {"MUON_SLOT_LAUNCHES": "1"}])
def test_canary_guards_stay_intact(env, monkeypatch):
    """Debug canary mode: every workspace region followed by a guard, checked
    after each call.  Over mixed, ragged, transposed and unaligned shapes and
    the fp32 check path no guard is touched, and the results are bitwise
    those of the normal layout."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    mo.muon_release_workspace()
    ref = _canary_workload()
    monkeypatch.setenv("MUON_DEBUG_CANARY", "1")
    mo.muon_release_workspace()
    got = _canary_workload()
    st, _ = mo.muon_device_status()
    assert st == mo.MUON_OK, mo.STATUS_NAMES.get(st)
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    mo.muon_release_workspace()


def test_canary_check_reports_an_overwritten_guard(monkeypatch):
    """A guard overwritten between calls (a plain memset into the library's
    own allocation, no fault) is reported by the next call's check as
    MUON_ERR_GUARD and re-armed: the call after that is clean again."""
    monkeypatch.setenv("MUON_DEBUG_CANARY", "1")
    mo.muon_release_workspace()
    shapes = [(256, 768), (200, 200)]
    G = [wl.make_single(r, c, 900 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, 910 + i, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, 920 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    mo.muon_step(W, G, M, lr=0.02)
    assert mo.muon_device_status()[0] == mo.MUON_OK
    with pytest.raises(mo.MuonError):
        mo.muon_debug_corrupt_guard(10 ** 6)  # no such guard
    mo.muon_debug_corrupt_guard(3)
    mo.muon_step(W, G, M, lr=0.02)
    assert mo.muon_device_status()[0] == mo.MUON_ERR_GUARD
    mo.muon_step(W, G, M, lr=0.02)
    assert mo.muon_device_status()[0] == mo.MUON_OK
    monkeypatch.delenv("MUON_DEBUG_CANARY")
    mo.muon_release_workspace()
    with pytest.raises(mo.MuonError):
        mo.muon_debug_corrupt_guard(0)  # the mode is off: no guards


def test_orthogonalize_captured_in_a_cuda_graph():
    """muon_orthogonalize captured after one eager call (its plan exists) and
    replayed twice equals three eager calls bit for bit."""
    X = torch.stack([wl.make_single(512, 1536, 940 + j, "gaussian", DEV, "bf16") for j in range(3)])
    Xr = X.clone()
    for _ in range(3):
        mo.muon_orthogonalize(Xr, steps=5, mode="gram")
    mo.muon_orthogonalize(X, steps=5, mode="gram")
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        mo.muon_orthogonalize(X, steps=5, mode="gram")
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(X, Xr)
    del graph
    mo.muon_release_workspace()


def test_hybrid_step_under_canary_guards(monkeypatch):
    """Debug canary mode over the hybrid step (the AdamW lane in the momentum
    launch's grid): guards intact, results equal to the normal layout."""
    shapes = [(256, 768), (200, 200), (37, 91)]
    numels = [50257 * 8, 768, 7]

    def run():
        W = [wl.make_single(r, c, 960 + i, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
        G = [wl.make_single(r, c, 970 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
        M = [wl.make_single(r, c, 980 + i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
        P = [wl.make_single(1, n, 990 + i, "params", DEV, "f32").view(-1) for i, n in enumerate(numels)]
        AG = [wl.make_single(1, n, 995 + i, "student_t3", DEV, "bf16", 0.01).view(-1) for i, n in enumerate(numels)]
        M1 = [torch.zeros(n, device=DEV) for n in numels]
        M2 = [torch.zeros(n, device=DEV) for n in numels]
        for t in (1, 2):
            mo.muon_hybrid_step(W, G, M, P, AG, M1, M2, t)
        torch.cuda.synchronize()
        return [x.clone() for x in W + M + P + M1 + M2]

    ref = run()
    monkeypatch.setenv("MUON_DEBUG_CANARY", "1")
    mo.muon_release_workspace()
    got = run()
    assert mo.muon_device_status()[0] == mo.MUON_OK
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    monkeypatch.delenv("MUON_DEBUG_CANARY")
    mo.muon_release_workspace()

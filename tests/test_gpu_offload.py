"""GPU tests of the offload step (muon_step_offload): gradients copied in from
pinned host memory and the updated parameters copied back to pinned host
memory, pipelined with the step over groups of matrices.  Every group is one
muon_step, so parameters, momentum and the host copies must equal a plain
muon_step's bit for bit; one case is also held against the fp64 oracle."""
import ctypes

import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests._util import TOL_BF16_RELF, relF, to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

# mixed shapes, ragged and transposed ones among them
SHAPES = [(256, 768), (768, 256), (200, 200), (136, 520), (520, 136), (64, 64), (384, 1024), (37, 91),
          (512, 512), (96, 300)]


@pytest.fixture(autouse=True)
def _fresh_config():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    mo.muon_reset_config()
    yield
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_OK, (mo.STATUS_NAMES.get(st), bad)
    mo.muon_reset_config()


def _make_set(shapes, seed, grad_dt="bf16", par_dt="f32", mom_dt="bf16"):
    G = [wl.make_single(r, c, seed + 3 * i, "student_t3", DEV, grad_dt, 0.01) for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, seed + 3 * i + 1, "student_t3", DEV, mom_dt, 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, seed + 3 * i + 2, "params", DEV, par_dt) for i, (r, c) in enumerate(shapes)]
    return W, G, M


def _clone(ts):
    return [t.clone() for t in ts]


def _pinned_like(ts):
    return [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ts]


def _check_equal(W, M, Wr, Mr, host_p=None):
    for i in range(len(W)):
        assert torch.equal(W[i], Wr[i]), i
        assert torch.equal(M[i], Mr[i]), i
        if host_p is not None:
            assert torch.equal(host_p[i], Wr[i].cpu()), i


@pytest.mark.parametrize("chunks", [1, 3, 8, 64])
def test_offload_equals_muon_step(chunks):
    """Two consecutive steps (the second reuses the per-group plans)."""
    W, G, M = _make_set(SHAPES, 4000)
    Wr, Mr = _clone(W), _clone(M)
    host_g = [g.cpu().pin_memory() for g in G]
    host_p = _pinned_like(W)
    Gd = [torch.zeros_like(g) for g in G]  # the device buffers the gradients land in
    for _ in range(2):
        mo.muon_step(Wr, G, Mr, mu=0.95, nesterov=True, lr=0.1)
        mo.muon_step_offload(W, Gd, M, grads_host=host_g, params_host=host_p, mu=0.95, nesterov=True, lr=0.1,
                             chunks=chunks)
        torch.cuda.synchronize()
        for i in range(len(SHAPES)):
            assert torch.equal(Gd[i], G[i]), i
        _check_equal(W, M, Wr, Mr, host_p)


def test_offload_dtypes():
    """fp32 gradients and bf16 parameters: the copies use the configured
    element sizes in both directions."""
    mo.muon_set_config(grad_dtype=mo.MUON_DTYPE_F32, param_dtype=mo.MUON_DTYPE_BF16,
                       momentum_dtype=mo.MUON_DTYPE_F32)
    W, G, M = _make_set(SHAPES[:6], 4100, grad_dt="f32", par_dt="bf16", mom_dt="f32")
    Wr, Mr = _clone(W), _clone(M)
    mo.muon_step(Wr, G, Mr, mu=0.9, nesterov=False, lr=0.2)
    host_g = [g.cpu().pin_memory() for g in G]
    host_p = _pinned_like(W)
    Gd = [torch.zeros_like(g) for g in G]
    mo.muon_step_offload(W, Gd, M, grads_host=host_g, params_host=host_p, mu=0.9, nesterov=False, lr=0.2, chunks=4)
    torch.cuda.synchronize()
    _check_equal(W, M, Wr, Mr, host_p)


def test_offload_one_direction():
    """grads_host only (the parameters stay on the device) and params_host
    only (the gradients are already on the device)."""
    W, G, M = _make_set(SHAPES, 4200)
    Wr, Mr = _clone(W), _clone(M)
    mo.muon_step(Wr, G, Mr, lr=0.05)
    Gd = [torch.zeros_like(g) for g in G]
    mo.muon_step_offload(W, Gd, M, grads_host=[g.cpu().pin_memory() for g in G], lr=0.05, chunks=5)
    torch.cuda.synchronize()
    _check_equal(W, M, Wr, Mr)
    mo.muon_step(Wr, G, Mr, lr=0.05)
    host_p = _pinned_like(W)
    mo.muon_step_offload(W, G, M, params_host=host_p, lr=0.05, chunks=5)
    torch.cuda.synchronize()
    _check_equal(W, M, Wr, Mr, host_p)


def test_offload_on_a_side_stream():
    """The call joins its copy streams into the bound stream: synchronising
    that stream alone is enough to read the host parameters."""
    W, G, M = _make_set(SHAPES, 4300)
    Wr, Mr = _clone(W), _clone(M)
    mo.muon_step(Wr, G, Mr, lr=0.1)
    torch.cuda.synchronize()
    host_g = [g.cpu().pin_memory() for g in G]
    host_p = _pinned_like(W)
    Gd = [torch.zeros_like(g) for g in G]
    s = torch.cuda.Stream(DEV)
    s.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(s):
        mo.muon_step_offload(W, Gd, M, grads_host=host_g, params_host=host_p, lr=0.1, chunks=4)
    s.synchronize()
    for i in range(len(SHAPES)):
        assert torch.equal(host_p[i], Wr[i].cpu()), i
    torch.cuda.synchronize()


def test_offload_against_oracle():
    """The host copy of the updated parameters against the fp64 oracle (the
    same bound as the muon_step parity tests)."""
    shapes = [(256, 768), (200, 200), (136, 520), (37, 91)]
    lr, mu = 0.1, 0.95
    W, G, M = _make_set(shapes, 4400)
    W64, G64, M64 = [to64(t) for t in W], [to64(t) for t in G], [to64(t) for t in M]
    host_g = [g.cpu().pin_memory() for g in G]
    host_p = _pinned_like(W)
    Gd = [torch.zeros_like(g) for g in G]
    mo.muon_step_offload(W, Gd, M, grads_host=host_g, params_host=host_p, mu=mu, nesterov=True, lr=lr, chunks=3)
    torch.cuda.synchronize()
    for i, (r, c) in enumerate(shapes):
        n, m = min(r, c), max(r, c)
        fm = "gram" if orc.ns_flops(n, m, 5, "gram") < orc.ns_flops(n, m, 5, "standard") else "standard"
        _, _, O = orc.muon_step(W64[i], G64[i], M64[i], mu, True, lr, form=fm)
        O_gpu = (W64[i] - host_p[i].double().numpy()) / lr
        assert relF(O_gpu, O) <= TOL_BF16_RELF, (shapes[i], relF(O_gpu, O))


def test_offload_rejects_pageable_host_memory():
    """Pageable host buffers: the binding raises, and the C ABI returns
    MUON_ERR_INVALID_ARG with nothing enqueued."""
    W, G, M = _make_set(SHAPES[:3], 4500)
    W0 = _clone(W)
    pageable = [g.cpu() for g in G]
    with pytest.raises(ValueError):
        mo.muon_step_offload(W, G, M, grads_host=pageable)
    vp = ctypes.c_void_p
    P = (vp * 3)(*[t.data_ptr() for t in W])
    Gp = (vp * 3)(*[t.data_ptr() for t in G])
    Mp = (vp * 3)(*[t.data_ptr() for t in M])
    H = (vp * 3)(*[t.data_ptr() for t in pageable])
    S = (ctypes.c_int * 6)(*[x for t in W for x in t.shape])
    mo._bind_stream(DEV)
    rc = mo.lib().muon_step_offload(P, H, Gp, Mp, None, 0.95, 1, 0.1, S, 3, 2)
    assert rc == mo.MUON_ERR_INVALID_ARG
    assert b"page-locked" in mo.lib().muon_last_error()
    torch.cuda.synchronize()
    for a, b in zip(W, W0):
        assert torch.equal(a, b)
    assert mo.lib().muon_step_offload(P, None, Gp, Mp, None, 0.95, 1, 0.1, S, 3, 0) == mo.MUON_ERR_INVALID_ARG


def test_offload_reports_bad_matrix_in_caller_numbering():
    """A non-finite gradient in matrix 7 (not in the first of four groups) is
    reported as matrix 7, and the other matrices are stepped as by muon_step."""
    W, G, M = _make_set(SHAPES, 4600)
    G[7][3, 5] = float("nan")
    Wr, Mr = _clone(W), _clone(M)
    mo.muon_step(Wr, G, Mr, lr=0.1)
    st, bad = mo.muon_device_status()
    assert (st, bad) == (mo.MUON_ERR_NONFINITE, 7)
    host_g = [g.cpu().pin_memory() for g in G]
    host_p = _pinned_like(W)
    Gd = [torch.zeros_like(g) for g in G]
    mo.muon_step_offload(W, Gd, M, grads_host=host_g, params_host=host_p, lr=0.1, chunks=4)
    st, bad = mo.muon_device_status()
    assert (st, bad) == (mo.MUON_ERR_NONFINITE, 7)
    bounds = mo.muon_offload_chunks([W[i].numel() * 6 for i in range(len(W))], 4)
    k = max(j for j in range(len(bounds) - 1) if bounds[j] <= 7)
    assert bounds[k] > 0  # matrix 7's group does not start at 0: its index is rebased
    for i in range(len(SHAPES)):
        assert torch.equal(host_p[i], Wr[i].cpu()), i
    assert torch.equal(M[7].float().isnan(), Mr[7].float().isnan())


def test_offload_with_shape_schedules_and_soft_threshold():
    """The offload step under a non-default config: a registered per-shape
    schedule (4 steps), the soft-threshold split and fp32 momentum.  Every
    group runs the same plan logic as one muon_step, so the results equal a
    plain muon_step's bit for bit."""
    mo.muon_set_config(soft_threshold=0.05, momentum_dtype=mo.MUON_DTYPE_F32)
    sched = [(3.0, -3.2, 1.2), (2.8, -3.0, 1.1), (2.5, -2.6, 1.0), (2.0, -1.5, 0.5)]
    mo.muon_set_shape_coeffs(256, 768, sched)
    W, G, M = _make_set(SHAPES, 4700, mom_dt="f32")
    Wr, Mr = _clone(W), _clone(M)
    mo.muon_step(Wr, G, Mr, lr=0.1)
    host_g = [g.cpu().pin_memory() for g in G]
    host_p = _pinned_like(W)
    Gd = [torch.zeros_like(g) for g in G]
    mo.muon_step_offload(W, Gd, M, grads_host=host_g, params_host=host_p, lr=0.1, chunks=4)
    torch.cuda.synchronize()
    _check_equal(W, M, Wr, Mr, host_p)


def test_offload_under_canary_guards(monkeypatch):
    """Debug canary mode over the offload step: every group's plan keeps its
    guards intact, and the results are those of the normal layout."""
    W, G, M = _make_set(SHAPES, 4800)
    Wr, Mr = _clone(W), _clone(M)
    host_g = [g.cpu().pin_memory() for g in G]
    Gd = [torch.zeros_like(g) for g in G]
    mo.muon_step_offload(Wr, Gd, Mr, grads_host=host_g, lr=0.1, chunks=3)
    monkeypatch.setenv("MUON_DEBUG_CANARY", "1")
    mo.muon_release_workspace()
    mo.muon_step_offload(W, Gd, M, grads_host=host_g, lr=0.1, chunks=3)
    assert mo.muon_device_status()[0] == mo.MUON_OK
    monkeypatch.delenv("MUON_DEBUG_CANARY")
    mo.muon_release_workspace()
    _check_equal(W, M, Wr, Mr)

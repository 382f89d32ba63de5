"""The allocation-free normalisation entry point, muon_normalize_noalloc.

It serves callers that cannot allocate device memory (their memory belongs
to a framework's allocator or a fixed budget, or an allocation on their path
is not acceptable).  Its output must equal what the existing entry point
gives for the same operation, muon_orthogonalize with steps = 0
(X / (||X||_F + eps)), on two calls in a row, and the fp64 oracle's
Frobenius normalisation of the same input.  The file name makes pytest
collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests._util import TOL_FP32_RELF, relF, to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
EPS = 1e-7  # the installed config's eps, which muon_orthogonalize uses


def _noalloc(X, Y, dtype, eps=EPS):
    lib = mo.lib()
    mo._bind_stream(X.device)
    batch, m, n = X.shape
    return lib.muon_normalize_noalloc(batch, m, n, ctypes.c_void_p(X.data_ptr()),
                                      ctypes.c_void_p(Y.data_ptr()), dtype, ctypes.c_float(eps))


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(3, 200, 712), (2, 37, 91), (1, 1024, 4096)])
def test_noalloc_matches_existing_entry_point(dt, shape):
    assert torch.cuda.is_available()
    mo.muon_reset_config()
    b, m, n = shape
    X = torch.stack([wl.make_single(m, n, 900 + i, "student_t3", DEV, dt, 0.01) for i in range(b)])
    ref = X.clone()
    mo.muon_orthogonalize(ref, steps=0, mode="standard", fp32=(dt == "f32"))
    code = mo.MUON_DTYPE_F32 if dt == "f32" else mo.MUON_DTYPE_BF16
    # bf16: both paths round s * x once; s may differ in its last fp32 bit
    tol = TOL_FP32_RELF / 10 if dt == "f32" else 1e-4
    # the fp64 oracle's normalisation of the same input, then the output's
    # storage rounding: one rounding is at most half an ulp per element, 2^-8
    # of its magnitude for bf16 and 2^-24 for fp32 (plus the fp32 scale: 1 %)
    want = [orc.frobenius_normalize(to64(X[i]), EPS) for i in range(b)]
    tol_orc = 1.01 * 2.0 ** -8 if dt == "bf16" else 1e-6
    for call in range(2):
        Y = torch.full_like(X, 7.0)
        assert _noalloc(X, Y, code) == mo.MUON_OK, mo.lib().muon_last_error()
        torch.cuda.synchronize()
        for i in range(b):
            assert relF(to64(Y[i]), to64(ref[i])) <= tol, (call, i)
            assert relF(to64(Y[i]), want[i]) <= tol_orc, (call, i)
    # in place (Y == X), twice in a row: the second call relies on the first
    # having left its ticket counters at zero
    for call in range(2):
        Z = X.clone()
        assert _noalloc(Z, Z, code) == mo.MUON_OK
        torch.cuda.synchronize()
        assert not torch.equal(Z, X)  # written, not left as the input
        for i in range(b):
            assert relF(to64(Z[i]), to64(ref[i])) <= tol, (call, i)
            assert relF(to64(Z[i]), want[i]) <= tol_orc, (call, i)


@pytest.mark.parametrize("eps", [0.0, EPS])
def test_noalloc_zero_matrix_gives_zeros(eps):
    """A zero matrix has no direction: its output is 0, also with eps = 0
    (no 0/0), and the other matrices of the batch are unaffected."""
    X = torch.stack([wl.make_single(64, 96, 990 + i, "gaussian", DEV, "bf16") for i in range(3)])
    X[1].zero_()
    for _ in range(2):
        Y = torch.full_like(X, 7.0)
        assert _noalloc(X, Y, mo.MUON_DTYPE_BF16, eps) == mo.MUON_OK
        torch.cuda.synchronize()
        assert torch.count_nonzero(Y[1]) == 0
        assert np.all(np.isfinite(to64(Y)))
        for i in (0, 2):
            assert relF(to64(Y[i]), orc.frobenius_normalize(to64(X[i]), eps)) <= 1.01 * 2.0 ** -8


def test_noalloc_allocates_nothing_and_rejects_oversize():
    X = torch.stack([wl.make_single(256, 512, 950 + i, "gaussian", DEV, "bf16") for i in range(4)])
    Y = torch.empty_like(X)
    assert _noalloc(X, Y, mo.MUON_DTYPE_BF16) == mo.MUON_OK  # first call: one-time set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _noalloc(X, Y, mo.MUON_DTYPE_BF16) == mo.MUON_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    lib = mo.lib()
    p = ctypes.c_void_p(X.data_ptr())
    # beyond the static scratch: rejected before any work
    assert lib.muon_normalize_noalloc(1025, 8, 8, p, p, mo.MUON_DTYPE_BF16,
                                      ctypes.c_float(EPS)) == mo.MUON_ERR_INVALID_ARG
    assert b"MUON_NOALLOC_MAX_MATRICES" in lib.muon_last_error()
    assert lib.muon_normalize_noalloc(2, 16385, 16384, p, p, mo.MUON_DTYPE_BF16,
                                      ctypes.c_float(EPS)) == mo.MUON_ERR_INVALID_ARG
    assert lib.muon_normalize_noalloc(1, 8, 8, p, p, 7, ctypes.c_float(EPS)) == mo.MUON_ERR_UNSUPPORTED

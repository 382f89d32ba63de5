"""The allocation-free normalisation entry point, muon_normalize_noalloc.

It serves callers that cannot allocate device memory (their memory belongs
to a framework's allocator or a fixed budget, or an allocation on their path
is not acceptable).  Its output must equal what the existing entry point
gives for the same operation, muon_orthogonalize with steps = 0
(X / (||X||_F + eps)), on two calls in a row.  The file name makes pytest
collect it last.
"""
import ctypes

import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from tests._util import TOL_FP32_RELF, relF, to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
EPS = 1e-7  # the installed config's eps, which muon_orthogonalize uses


def _noalloc(X, Y, dtype):
    lib = mo.lib()
    mo._bind_stream(X.device)
    batch, m, n = X.shape
    return lib.muon_normalize_noalloc(batch, m, n, ctypes.c_void_p(X.data_ptr()),
                                      ctypes.c_void_p(Y.data_ptr()), dtype, ctypes.c_float(EPS))


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
    for call in range(2):
        Y = torch.full_like(X, 7.0)
        assert _noalloc(X, Y, code) == mo.MUON_OK, mo.lib().muon_last_error()
        torch.cuda.synchronize()
        for i in range(b):
            assert relF(to64(Y[i]), to64(ref[i])) <= tol, (call, i)
    # in place (Y == X), twice more
    Z = X.clone()
    assert _noalloc(Z, Z, code) == mo.MUON_OK
    torch.cuda.synchronize()
    for i in range(b):
        assert relF(to64(Z[i]), to64(ref[i])) <= tol


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

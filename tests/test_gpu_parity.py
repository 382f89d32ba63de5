"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle,
element by element, on the same seeded inputs.

Tolerances (written here, from the Newton-Schulz accuracy bar): relative
Frobenius error <= 2e-2 for the bf16 tensor-core path and <= 1e-5 for the
fp32 check path; every singular value within 0.02 of the oracle's.
"""
import numpy as np
import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests._util import TOL_BF16_RELF, TOL_FP32_RELF, TOL_SIGMA, relF, sigma_maxdiff, to64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
FORMS = {"standard": "standard", "gram": "gram"}


@pytest.fixture(autouse=True)
def _fresh_config():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    mo.muon_reset_config()
    yield
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_OK, (mo.STATUS_NAMES.get(st), bad)
    mo.muon_reset_config()


def _ortho_gpu(X, form, steps=5, coeffs=mo.TUNED_COEFFS, fp32=False):
    Y = X.clone()
    mo.muon_orthogonalize(Y, coeffs=coeffs, steps=steps, mode=form, fp32=fp32)
    torch.cuda.synchronize()
    return Y


def _check(gpu, ref, tol):
    r = relF(gpu, ref)
    s = sigma_maxdiff(gpu, ref)
    assert r <= tol, f"relF {r:.3e} > {tol}"
    assert s <= TOL_SIGMA, f"max |dsigma| {s:.3e} > {TOL_SIGMA}"
    return r, s


# ---- workload 1: single 256 x 1024 fp32 N(0,1), seed 0 -------------------------

@pytest.mark.parametrize("form", ["standard", "gram"])
def test_fp32_check_path_256x1024(form):
    w = wl.WORKLOADS[1]
    X = wl.make_matrix(w, 0, wl.ROLE_GRAD, device=DEV, dtype="f32")
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, 5, form)
    Y = _ortho_gpu(X, form, fp32=True)
    _check(to64(Y), ref, TOL_FP32_RELF)


@pytest.mark.parametrize("form", ["standard", "gram"])
def test_bf16_256x1024(form):
    w = wl.WORKLOADS[1]
    X = wl.make_matrix(w, 0, wl.ROLE_GRAD, device=DEV, dtype="bf16")
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, 5, form)
    Y = _ortho_gpu(X, form)
    _check(to64(Y), ref, TOL_BF16_RELF)


# ---- ragged / edge shapes (several tiles and a ragged tail) ------------------

RAGGED = [(200, 712), (712, 200), (72, 1000), (130, 130), (37, 91), (91, 37), (8, 8), (1, 40), (1, 1), (2, 3), (3, 2), (1, 4097),
          (40, 1), (384, 1536), (1000, 136), (264, 520), (520, 264), (300, 300)]


@pytest.mark.parametrize("shape", RAGGED)
@pytest.mark.parametrize("form", ["standard", "gram"])
def test_ragged_bf16(shape, form):
    r, c = shape
    X = wl.make_single(r, c, 7 + r * 31 + c, "gaussian", DEV, "bf16")
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, 5, form)
    Y = _ortho_gpu(X, form)
    _check(to64(Y), ref, TOL_BF16_RELF)


@pytest.mark.parametrize("shape", [(256, 768), (768, 256)])
@pytest.mark.parametrize("form", ["standard", "gram"])
def test_misaligned_base_bf16(shape, form):
    """X starting one element past a 16-byte boundary (width a multiple of 8):
    element-wise loads and plain stores, same result; nothing outside X is
    written."""
    r, c = shape
    X0 = wl.make_single(r, c, 4242 + r, "gaussian", DEV, "bf16")
    buf = torch.full((r * c + 16,), 7.0, dtype=torch.bfloat16, device=DEV)
    X = buf[1:1 + r * c].view(r, c)
    assert X.data_ptr() % 16 != 0
    X.copy_(X0)
    ref = orc.orthogonalize(to64(X0), orc.TUNED_COEFFS, 5, form)
    mo.muon_orthogonalize(X, steps=5, mode=form)
    torch.cuda.synchronize()
    _check(to64(X), ref, TOL_BF16_RELF)
    assert float(buf[0]) == 7.0 and bool((buf[1 + r * c:] == 7.0).all())


@pytest.mark.parametrize("shape", [(200, 712), (712, 200), (37, 91), (300, 300)])
@pytest.mark.parametrize("form", ["standard", "gram"])
def test_ragged_fp32(shape, form):
    r, c = shape
    X = wl.make_single(r, c, 11 + r + c, "gaussian", DEV, "f32")
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, 5, form)
    Y = _ortho_gpu(X, form, fp32=True)
    _check(to64(Y), ref, TOL_FP32_RELF)


@pytest.mark.parametrize("steps", [1, 2, 3])
@pytest.mark.parametrize("form", ["standard", "gram"])
def test_few_steps(steps, form):
    X = wl.make_single(256, 640, 5, "gaussian", DEV, "bf16")
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, steps, form)
    Y = _ortho_gpu(X, form, steps=steps)
    _check(to64(Y), ref, TOL_BF16_RELF)


def test_per_step_coefficients():
    co = [(3.4445, -4.7750, 2.0315), (2.9, -4.0, 1.9), (2.5, -3.0, 1.4), (2.0, -1.5, 0.5),
          (1.875, -1.25, 0.375)]
    X = wl.make_single(192, 448, 6, "gaussian", DEV, "bf16")
    for form in ("standard", "gram"):
        ref = orc.orthogonalize(to64(X), co, 5, form)
        Y = _ortho_gpu(X, form, coeffs=co)
        _check(to64(Y), ref, TOL_BF16_RELF)


@pytest.mark.parametrize("mask", [0, 1 << 1, 1 << 2, 1 << 3, (1 << 2) | (1 << 3), 0b11110])
def test_gram_restart_schedules(mask):
    mo.muon_set_config(restart_mask=mask)
    X = wl.make_single(256, 768, 8, "student_t3", DEV, "bf16")
    restarts = tuple(k for k in range(1, 5) if (mask >> k) & 1)
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, 5, "gram", restarts=restarts)
    Y = _ortho_gpu(X, "gram")
    _check(to64(Y), ref, TOL_BF16_RELF)


def test_batch_of_matrices():
    X = torch.stack([wl.make_single(128, 384, 40 + i, "gaussian", DEV, "bf16") for i in range(5)])
    for form in ("standard", "gram"):
        Y = _ortho_gpu(X, form)
        for i in range(5):
            ref = orc.orthogonalize(to64(X[i]), orc.TUNED_COEFFS, 5, form)
            _check(to64(Y[i]), ref, TOL_BF16_RELF)


def test_batch_larger_than_sm_count():
    X = torch.stack([wl.make_single(64, 96, 500 + i, "gaussian", DEV, "bf16") for i in range(200)])
    Y = _ortho_gpu(X, "gram")
    for i in (0, 77, 199):
        ref = orc.orthogonalize(to64(X[i]), orc.TUNED_COEFFS, 5, "gram")
        _check(to64(Y[i]), ref, TOL_BF16_RELF)


def test_steps_zero_normalises():
    X = wl.make_single(100, 300, 9, "gaussian", DEV, "bf16")
    Y = _ortho_gpu(X, "standard", steps=0)
    ref = orc.orthogonalize(to64(X), orc.TUNED_COEFFS, 0, "standard")
    assert relF(to64(Y), ref) < 4e-3  # one bf16 rounding of the output


def test_zero_matrix_gives_zero():
    X = torch.zeros(64, 128, dtype=torch.bfloat16, device=DEV)
    for form in ("standard", "gram"):
        Y = _ortho_gpu(X, form)
        assert torch.count_nonzero(Y).item() == 0


def test_nonfinite_matrix_is_flagged_and_left_untouched():
    X = torch.stack([wl.make_single(64, 128, 60 + i, "gaussian", DEV, "bf16") for i in range(3)])
    X[1, 3, 5] = float("inf")
    before = X.clone()
    mo.muon_orthogonalize(X, steps=5, mode="gram")
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_ERR_NONFINITE and bad == 1
    assert torch.equal(X[1], before[1])
    ref = orc.orthogonalize(to64(before[0]), orc.TUNED_COEFFS, 5, "gram")
    _check(to64(X[0]), ref, TOL_BF16_RELF)


def test_scale_invariance_bf16():
    X = wl.make_single(128, 512, 12, "gaussian", DEV, "bf16")
    Y1 = _ortho_gpu(X, "gram")
    Y2 = _ortho_gpu((X.float() * 64).to(torch.bfloat16), "gram")  # exact power-of-two scale
    # s differs from s/64 only through eps and fp32 rounding of s
    assert relF(to64(Y1), to64(Y2)) < 1e-2


# ---- aspect-ratio sweep (workload 3), sampled matrices -------------------------

def _sv_gram(x):
    """Singular values from the eigenvalues of the short-side Gram matrix
    (the same values as an SVD, far cheaper at these sizes)."""
    x = np.asarray(x, dtype=np.float64)
    g = x @ x.T if x.shape[0] <= x.shape[1] else x.T @ x
    return np.sqrt(np.clip(np.linalg.eigvalsh(g), 0, None))


@pytest.mark.slow
@pytest.mark.parametrize("shape", [(2048, 2048), (2048, 8192), (1024, 16384)])
def test_aspect_sweep_batch16_all(shape):
    """Workload 3 (aspect-ratio sweep, batch 16): every matrix of the batch,
    standard and Gram forms, against the oracle.  The oracle's two forms agree
    to 1e-12 in fp64 (pinned on the CPU), so one oracle result per matrix
    serves both GPU forms."""
    w = wl.WORKLOADS[3]
    idx = [i for i, s in enumerate(w.shapes) if s == shape]
    X = torch.stack([wl.make_matrix(w, i, wl.ROLE_GRAD, device=DEV) for i in idx])
    Ys = {form: to64(_ortho_gpu(X, form)) for form in ("standard", "gram")}
    n, m = min(shape), max(shape)
    cheap = "gram" if orc.ns_flops(n, m, 5, "gram") < orc.ns_flops(n, m, 5, "standard") else "standard"
    worst = {}
    for j in range(len(idx)):
        ref = orc.orthogonalize(to64(X[j]), orc.TUNED_COEFFS, 5, cheap)
        sv_ref = _sv_gram(ref)
        for form, Y in Ys.items():
            r = relF(Y[j], ref)
            sd = float(np.max(np.abs(_sv_gram(Y[j]) - sv_ref)))
            worst[form] = max(worst.get(form, 0.0), r)
            assert r <= TOL_BF16_RELF, (form, j, r)
            assert sd <= TOL_SIGMA, (form, j, sd)
    print(shape, "worst relF", worst)


def test_fitted_per_shape_schedule():
    """Per-shape coefficients fitted on the host (ROOT-style adaptive NS) run
    through the same kernels and match the oracle with those coefficients;
    the bf16 output is closer to orthogonal than with the fixed set."""
    from matrix_orthogonalizing_optimizer_step_b200 import coeffs as C
    sched = C.fit_schedule(384, 1536)
    X = wl.make_single(384, 1536, 33, "gaussian", DEV, "bf16")
    errs = {}
    for name, co in (("fit", sched), ("tuned", mo.TUNED_COEFFS)):
        for form in ("standard", "gram"):
            ref = orc.orthogonalize(to64(X), co, 5, form)
            Y = _ortho_gpu(X, form, coeffs=co)
            _check(to64(Y), ref, TOL_BF16_RELF)
            errs[name, form] = np.mean((np.linalg.svd(to64(Y), compute_uv=False) - 1) ** 2)
    for form in ("standard", "gram"):
        assert errs["fit", form] < 0.5 * errs["tuned", form], errs

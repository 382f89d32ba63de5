"""Per-shape coefficient schedules (ROOT page, adaptive Newton-Schulz):
the spectrum model against real SVDs, and the fitted schedules against the
oracle's own iteration."""
import numpy as np
import pytest

from matrix_orthogonalizing_optimizer_step_b200 import coeffs as C
from oracle import muon_oracle as orc


@pytest.mark.parametrize("shape", [(256, 1024), (512, 512), (384, 1536)])
def test_mp_spectrum_matches_gaussian_svd(shape):
    m, n = shape
    X = np.random.default_rng(1).standard_normal(shape)
    s_true = np.sort(np.linalg.svd(X / np.linalg.norm(X), compute_uv=False))[::-1]
    s_mp = C.mp_singular_values(m, n)
    assert s_mp.size == s_true.size
    # quantiles agree up to the finite-size fluctuation of one sample
    assert np.max(np.abs(s_mp - s_true)) < 0.03 * s_true.max()
    assert abs(np.mean(s_mp ** 2) - np.mean(s_true ** 2)) < 1e-3 * np.mean(s_true ** 2)


@pytest.mark.parametrize("shape", [(256, 1024), (384, 1536), (512, 512)])
def test_fitted_schedule_reduces_orthogonality_error(shape):
    m, n = shape
    sched = C.fit_schedule(m, n)
    assert len(sched) == 5
    # guard (a penalty): the fitted map stays within about [0, 1.25] on [0, 1]
    g = C.apply_schedule(np.linspace(0, 1, 2001), sched)
    assert g.min() >= -1e-3 and g.max() <= 1.27
    X = np.random.default_rng(2).standard_normal(shape)
    for form in ("standard", "gram"):
        out_tuned = orc.orthogonalize(X, orc.TUNED_COEFFS, 5, form)
        out_fit = orc.orthogonalize(X, sched, 5, form)
        e_tuned = np.mean((np.linalg.svd(out_tuned, compute_uv=False) - 1) ** 2)
        e_fit = np.mean((np.linalg.svd(out_fit, compute_uv=False) - 1) ** 2)
        assert e_fit < 0.5 * e_tuned, (form, e_fit, e_tuned)

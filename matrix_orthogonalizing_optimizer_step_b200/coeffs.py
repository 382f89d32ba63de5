"""Per-shape Newton-Schulz coefficient schedules (host-side configuration).

The ROOT summary page ("ROOT优化器的技术创新") proposes adapting the quintic
Newton-Schulz coefficients to each matrix shape (m, n) instead of one fixed
set, because a fixed set leaves a shape-dependent orthogonalisation error
("现有优化器的核心局限": MSE 0.0499 on 2048 x 2048).  The page gives no
fitting procedure; the reading taken here:

  * the target is the singular-value map f = p_T o ... o p_1 with
    p_k(s) = a_k s + b_k s^3 + c_k s^5 (one triple per step);
  * the singular values to fit are those of a Gaussian matrix of the shape
    after Frobenius normalisation: the Marchenko-Pastur law with ratio
    lambda = n/m gives the eigenvalues of X X^T / m, and sigma_i^2 =
    e_i / sum_j e_j;
  * the objective is the mean of (f(sigma_i) - 1)^2 over those quantiles,
    plus a guard that keeps f within [0, 1.25] on the whole of [0, 1]
    (inputs outside the fitted spectrum must not blow up);
  * start from the tuned set (3.4445, -4.7750, 2.0315) and minimise with a
    derivative-free local search.

The result is a plain list of (a, b, c) for muon_set_config(coeffs=...) or
muon_orthogonalize(coeffs=...); no step of the optimizer runs here.
"""
from __future__ import annotations

import numpy as np

TUNED = (3.4445, -4.7750, 2.0315)


def mp_singular_values(m, n, count=None):
    """Singular values of a Frobenius-normalised Gaussian m x n matrix, as
    quantiles of the Marchenko-Pastur law (short side n' = min(m, n))."""
    lo_n, hi_m = min(m, n), max(m, n)
    lam = lo_n / hi_m
    k = count or min(lo_n, 2048)
    a, b = (1 - np.sqrt(lam)) ** 2, (1 + np.sqrt(lam)) ** 2
    # inverse CDF of the MP density by integrating it on a fine grid
    x = np.linspace(a, b, 20001)
    dens = np.sqrt(np.clip((b - x) * (x - a), 0, None)) / (2 * np.pi * lam * np.maximum(x, 1e-300))
    cdf = np.concatenate([[0.0], np.cumsum((dens[1:] + dens[:-1]) * np.diff(x) / 2)])
    cdf /= cdf[-1]
    q = (np.arange(k) + 0.5) / k
    e = np.interp(q, cdf, x)
    # Frobenius normalisation: sum of all lo_n squared singular values is 1
    return np.sqrt(e / (lo_n * e.mean()))[::-1]


def apply_schedule(sigma, coeffs):
    s = np.asarray(sigma, dtype=np.float64)
    for a, b, c in coeffs:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def schedule_error(sigma, coeffs):
    return float(np.mean((apply_schedule(sigma, coeffs) - 1.0) ** 2))


def fit_schedule(m, n, steps=5, init=TUNED, iters=4000, seed=0):
    """Per-step coefficients for an m x n matrix (see the module docstring).
    Returns a list of `steps` (a, b, c) triples."""
    from scipy.optimize import minimize

    sigma = mp_singular_values(m, n)
    grid = np.linspace(0.0, 1.0, 401)

    def unpack(z):
        return [tuple(z[3 * k:3 * k + 3]) for k in range(steps)]

    def objective(z):
        cs = unpack(z)
        err = schedule_error(sigma, cs)
        g = apply_schedule(grid, cs)
        guard = np.sum(np.clip(g - 1.25, 0, None) ** 2) + np.sum(np.clip(-g, 0, None) ** 2)
        return err + 10.0 * guard

    z0 = np.array(list(init) * steps if len(np.shape(init)) == 1 else np.ravel(init), dtype=np.float64)
    best = minimize(objective, z0, method="Nelder-Mead",
                    options={"maxiter": iters, "maxfev": iters * 2, "xatol": 1e-6, "fatol": 1e-10})
    z = best.x if best.fun <= objective(z0) else z0
    return unpack(z)

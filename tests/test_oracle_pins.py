"""Pins of the fp64 oracle against facts that do not come from the oracle.

* the spectral closed form of an odd matrix polynomial (textbook SVD):
  NS_T(X) = U diag(f(sigma)) V^T with f the scalar quintic iterated T times;
* the Gram rewrite p(t) = t q(t^2) (Gram Newton-Schulz page, section on the
  algorithm's advantage): the Gram iteration equals the standard one;
* the coefficient claims of the NanoGPT/Muon page (section on coefficient
  tuning): (2, -1.5, 0.5) converges to polar(X) = U V^T, the tuned set lands
  singular values in roughly [0.7, 1.3] after five steps;
* the ROOT page's worked number (golden file): MSE 0.0499 on 2048 x 2048;
* the closed form of SGD momentum under a constant gradient;
* invariances (transpose, positive scale) and special cases (zero input,
  zero steps).

The last block plants plausible mistakes in copies of the oracle and checks
that these pins catch every one of them.
"""
import os

import numpy as np
import pytest

from oracle import muon_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _scalar_f(sigma, coeffs, steps):
    """f = p_T o ... o p_1 applied to scalars, p_k(s) = a s + b s^3 + c s^5."""
    s = np.array(sigma, dtype=np.float64)
    for a, b, c in orc._coeff_list(coeffs, steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def _spectral_ns(X, coeffs, steps):
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    return (U * _scalar_f(S, coeffs, steps)) @ Vt


def _relF(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


SHAPES = [(24, 40), (32, 32), (40, 24), (7, 61)]
COEFFS = [orc.TUNED_COEFFS, orc.CLASSIC_COEFFS,
          # per-step coefficients (one triple per step)
          ((3.4445, -4.7750, 2.0315), (2.9, -4.0, 1.9), (2.5, -3.0, 1.4),
           (2.0, -1.5, 0.5), (1.875, -1.25, 0.375))]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("coeffs", COEFFS)
@pytest.mark.parametrize("form", ["standard", "gram"])
def test_ns_matches_spectral_closed_form(shape, coeffs, form):
    X = _rng(1).standard_normal(shape)
    X0 = X / (np.linalg.norm(X) + orc.DEFAULT_EPS)
    got = orc.orthogonalize(X, coeffs, 5, form)
    want = _spectral_ns(X0, coeffs, 5)
    assert _relF(got, want) < 1e-11


@pytest.mark.parametrize("restarts", [(), (1,), (2,), (3,), (2, 3), (1, 2, 3, 4)])
@pytest.mark.parametrize("steps", [1, 2, 5, 7])
def test_gram_equals_standard(restarts, steps):
    X = _rng(2).standard_normal((20, 52))
    X /= np.linalg.norm(X)
    std = orc.ns_standard(X, orc.TUNED_COEFFS, steps)
    gram = orc.ns_gram(X, orc.TUNED_COEFFS, steps, restarts)
    assert _relF(gram, std) < 1e-12


def test_classic_coefficients_converge_to_polar():
    X = _rng(3).standard_normal((48, 80))
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    # spread the singular values over [1e-3, 1] to exercise the slow end
    S = np.geomspace(1e-3, 1.0, S.size)[::-1]
    X = (U * S) @ Vt
    polar = U @ Vt
    for form in ("standard", "gram"):
        got = orc.orthogonalize(X, orc.CLASSIC_COEFFS, 40, form,
                                restarts=(10, 20, 30))
        assert np.max(np.abs(got - polar)) < 1e-10
        sv = np.linalg.svd(got, compute_uv=False)
        assert np.max(np.abs(sv - 1.0)) < 1e-10


def test_tuned_coefficients_range():
    """Five tuned steps send every singular value in [3e-3, 1] into about
    [0.68, 1.21]; the page rounds this to [0.7, 1.3]."""
    grid = np.linspace(3e-3, 1.0, 200001)
    f = _scalar_f(grid, orc.TUNED_COEFFS, 5)
    lo, hi = f.min(), f.max()
    assert 0.66 < lo < 0.70 and 1.15 < hi < 1.30
    for shape, dist in [((64, 256), "gauss"), ((128, 128), "gauss"),
                        ((96, 300), "t3")]:
        r = _rng(4)
        X = r.standard_normal(shape) if dist == "gauss" else r.standard_t(3, shape)
        X0 = X / np.linalg.norm(X)
        smin = np.linalg.svd(X0, compute_uv=False).min()
        out = orc.orthogonalize(X, orc.TUNED_COEFFS, 5, "standard")
        sv = np.linalg.svd(out, compute_uv=False)
        if smin >= 3e-3:
            assert sv.min() >= lo - 1e-9 and sv.max() <= hi + 1e-9


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    return vals


def test_root_page_mse_2048():
    g = _read_golden("root_orthogonality_mse.txt")
    rows, cols = int(g["rows"]), int(g["cols"])
    X = _rng(0).standard_normal((rows, cols))
    out = orc.orthogonalize(X, (g["a"], g["b"], g["c"]), int(g["steps"]),
                            "standard")
    sv = np.linalg.svd(out, compute_uv=False)
    mse = float(np.mean((sv - 1.0) ** 2))
    assert abs(mse - g["mse"]) < g["tol"], mse


def test_momentum_closed_form():
    G = _rng(5).standard_normal((6, 9))
    mu = 0.95
    M = np.zeros_like(G)
    for t in range(1, 12):
        M, U = orc.momentum_update(M, G, mu, nesterov=True)
        Mt = G * (1 - mu ** t) / (1 - mu)
        assert np.allclose(M, Mt, rtol=1e-13, atol=0)
        assert np.allclose(U, G + mu * Mt, rtol=1e-13, atol=0)
    M2, U2 = orc.momentum_update(M, G, mu, nesterov=False)
    assert np.array_equal(U2, M2)


def test_transpose_equivariance():
    X = _rng(6).standard_normal((30, 70))
    for form in ("standard", "gram"):
        a = orc.orthogonalize(X, steps=5, form=form)
        b = orc.orthogonalize(X.T.copy(), steps=5, form=form)
        assert _relF(b, a.T) < 1e-13


def test_scale_invariance():
    X = _rng(7).standard_normal((16, 40))
    # exact invariance holds with eps = 0 (eps / ||X|| differs between scales)
    a = orc.orthogonalize(X, form="standard", eps=0.0)
    b = orc.orthogonalize(37.5 * X, form="standard", eps=0.0)
    assert _relF(a, b) < 1e-12


def test_zero_and_zero_steps():
    Z = np.zeros((8, 12))
    assert np.array_equal(orc.orthogonalize(Z, form="gram"), Z)
    assert np.array_equal(orc.orthogonalize(Z, form="standard"), Z)
    X = _rng(8).standard_normal((8, 12))
    want = X / (np.linalg.norm(X) + orc.DEFAULT_EPS)
    for form in ("standard", "gram"):
        assert np.allclose(orc.orthogonalize(X, steps=0, form=form), want,
                           rtol=1e-15, atol=0)


def test_muon_step_update():
    r = _rng(9)
    W, G, M = (r.standard_normal((10, 14)) for _ in range(3))
    W1, M1, O = orc.muon_step(W, G, M, mu=0.9, nesterov=True, lr=0.01,
                              form="gram")
    assert np.allclose(M1, 0.9 * M + G)
    U = G + 0.9 * M1
    assert _relF(O, _spectral_ns(U / (np.linalg.norm(U) + 1e-7),
                                 orc.TUNED_COEFFS, 5)) < 1e-11
    assert np.allclose(W1, W - 0.01 * O)


def test_flop_formulas():
    n, m = 96, 320
    assert orc.ns_flops(n, m, 5, "standard") == 15 * n * n * m + 5 * n ** 3
    assert orc.ns_flops(n, m, 5, "gram", ()) == 3 * n * n * m + 17 * n ** 3
    assert orc.ns_flops(n, m, 5, "gram", (2,)) == 6 * n * n * m + 14 * n ** 3


# ---------------------------------------------------------------------------
# planted mistakes: each mutant is the oracle with one plausible error; the
# pins above must reject all of them.

def _mut_std_sign(X, coeffs, steps):
    X = X.copy()
    for a, b, c in orc._coeff_list(coeffs, steps):
        A = X @ X.T
        X = a * X + (-b * A + c * (A @ A)) @ X
    return X


def _mut_std_dropped_term(X, coeffs, steps):
    X = X.copy()
    for a, b, c in orc._coeff_list(coeffs, steps):
        A = X @ X.T
        X = a * X + (b * A) @ X
    return X


def _mut_std_transposed(X, coeffs, steps):
    # multiplies q(X X^T) on the wrong side: X B instead of B X (square X)
    X = X.copy()
    for a, b, c in orc._coeff_list(coeffs, steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + X @ B
    return X


def _mut_std_coeff_index(X, coeffs, steps):
    X = X.copy()
    for a, b, c in orc._coeff_list(coeffs, steps):
        A = X @ X.T
        X = a * X + (c * A + b * (A @ A)) @ X
    return X


def _mut_gram_no_right_z(X, coeffs, steps, restarts=(2,)):
    X = X.copy()
    n = X.shape[0]
    I = np.eye(n)
    R = X @ X.T
    Q = I.copy()
    for k, (a, b, c) in enumerate(orc._coeff_list(coeffs, steps)):
        if k in restarts and k > 0:
            X = Q @ X
            R = X @ X.T
            Q = I.copy()
        Z = a * I + b * R + c * (R @ R)
        Q = Z @ Q
        R = Z @ R
    return Q @ X


def _mut_gram_restart_keeps_q(X, coeffs, steps, restarts=(2,)):
    X = X.copy()
    n = X.shape[0]
    I = np.eye(n)
    R = X @ X.T
    Q = I.copy()
    for k, (a, b, c) in enumerate(orc._coeff_list(coeffs, steps)):
        if k in restarts and k > 0:
            X = Q @ X
            R = X @ X.T
        Z = a * I + b * R + c * (R @ R)
        Q = Z @ Q
        R = Z @ R @ Z
    return Q @ X


@pytest.mark.parametrize("mutant", [_mut_std_sign, _mut_std_dropped_term,
                                    _mut_std_transposed, _mut_std_coeff_index])
def test_planted_standard_mistakes_are_caught(mutant):
    X = _rng(1).standard_normal((32, 32))
    X0 = X / (np.linalg.norm(X) + orc.DEFAULT_EPS)
    want = _spectral_ns(X0, orc.TUNED_COEFFS, 5)
    assert _relF(orc.ns_standard(X0, orc.TUNED_COEFFS, 5), want) < 1e-11
    with np.errstate(over="ignore", invalid="ignore"):
        bad = mutant(X0, orc.TUNED_COEFFS, 5)
    err = _relF(bad, want) if np.all(np.isfinite(bad)) else np.inf
    assert err > 1e-4


@pytest.mark.parametrize("mutant", [_mut_gram_no_right_z,
                                    _mut_gram_restart_keeps_q])
def test_planted_gram_mistakes_are_caught(mutant):
    X = _rng(2).standard_normal((20, 52))
    X /= np.linalg.norm(X)
    std = orc.ns_standard(X, orc.TUNED_COEFFS, 5)
    assert _relF(mutant(X, orc.TUNED_COEFFS, 5), std) > 1e-4


# ---------------------------------------------------------------------------
# AdamW lane

def test_adamw_matches_torch_adamw_fp64():
    """Against the library routine torch.optim.AdamW (fp64, CPU) over several
    steps with a changing gradient."""
    import torch
    r = _rng(20)
    p0 = r.standard_normal((7, 13))
    grads = [r.standard_normal((7, 13)) for _ in range(6)]
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=6e-4, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = orc.adamw_step(p, g, m, v, t)
        assert np.allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-15)


def test_adamw_closed_forms():
    # constant gradient from zero state: bias-corrected m = g, v = g^2, so the
    # Adam part of every step is lr * g / (|g| + eps)
    g = np.array([[0.5, -2.0, 1e-3]])
    p = np.array([[1.0, 1.0, 1.0]])
    m = v = np.zeros_like(g)
    lr, wd = 1e-2, 0.0
    for t in range(1, 5):
        p_prev = p
        p, m, v = orc.adamw_step(p, g, m, v, t, lr=lr, weight_decay=wd)
        assert np.allclose(p_prev - p, lr * g / (np.abs(g) + 1e-8), rtol=1e-12)
    # zero gradient: pure decoupled decay, p_t = p_0 (1 - lr wd)^t
    p0 = np.array([[2.0, -3.0]])
    p, m, v = p0, np.zeros_like(p0), np.zeros_like(p0)
    for t in range(1, 6):
        p, m, v = orc.adamw_step(p, np.zeros_like(p0), m, v, t, lr=0.1, weight_decay=0.2)
        assert np.allclose(p, p0 * (1 - 0.1 * 0.2) ** t, rtol=1e-14)


def _adamw_mutant(kind):
    """Plausible wrong AdamW variants (planted on the CPU, never in the oracle)."""
    def step(p, g, m, v, t, lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1):
        if kind == "coupled":
            g = g + weight_decay * p  # L2 regularisation instead of decoupled decay
        elif kind != "decay_after":
            p = p - lr * weight_decay * p
        m = beta1 * m + (1 - beta1) * g
        v = beta2 * v + (1 - beta2) * g * g
        if kind == "no_bias_correction":
            upd = m / (np.sqrt(v) + eps)
        else:
            upd = (m / (1 - beta1 ** t)) / (np.sqrt(v / (1 - beta2 ** t)) + eps)
        p_new = p - lr * upd
        if kind == "decay_after":
            p_new = p_new - lr * weight_decay * p_new
        return p_new, m, v
    return step


@pytest.mark.parametrize("kind", ["no_bias_correction", "coupled", "decay_after"])
def test_adamw_pin_rejects_planted_mistakes(kind):
    """The torch.optim.AdamW comparison above tells each mutant apart."""
    import torch
    r = _rng(21)
    p0 = r.standard_normal((5, 9))
    grads = [r.standard_normal((5, 9)) for _ in range(4)]
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=1e-2, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    step = _adamw_mutant(kind)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    worst = 0.0
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = step(p, g, m, v, t, lr=1e-2)
        worst = max(worst, float(np.max(np.abs(p - tp.detach().numpy()))))
    assert worst > 1e-7, worst


# ---------------------------------------------------------------------------
# Soft-threshold split ([ROOT] "ROOT优化器的技术创新")

def test_soft_threshold_split_minimises_the_objective_by_brute_force():
    """Each element of O minimises (m - o)^2 + lam |o| (the objective with the
    robust part held at the residual): check against a dense grid search."""
    r = _rng(30)
    M = r.standard_normal((4, 6)) * 2.0
    lam = 1.3
    _, O = orc.soft_threshold_split(M, lam)
    grid = np.linspace(-8, 8, 160001)
    for mval, o in zip(M.ravel(), O.ravel()):
        f = (mval - grid) ** 2 + lam * np.abs(grid)
        best = grid[np.argmin(f)]
        assert abs(best - o) <= 2e-4, (mval, o, best)


def test_soft_threshold_split_invariants_and_limits():
    r = _rng(31)
    M = r.standard_normal((9, 5))
    lam = 0.8
    B, O = orc.soft_threshold_split(M, lam)
    assert np.allclose(B + O, M, rtol=0, atol=1e-15)        # a split of M
    assert np.all(np.abs(B) <= lam / 2 + 1e-15)             # robust part bounded
    small = np.abs(M) <= lam / 2
    assert np.all(O[small] == 0) and np.all(B[small] == M[small])
    assert np.all(np.sign(O[~small]) == np.sign(M[~small]))
    # lam -> infinity: no outliers, plain Muon; lam -> 0: everything is outlier
    B_inf, O_inf = orc.soft_threshold_split(M, 1e9)
    assert np.array_equal(B_inf, M) and not O_inf.any()
    B0, _ = orc.soft_threshold_split(M, 0.0)
    assert not B0.any()


def test_soft_threshold_muon_step_orthogonalises_the_clipped_update():
    r = _rng(32)
    G = r.standard_normal((6, 10)) * 0.01
    G[2, 3] = 3.0  # one outlier
    W = r.standard_normal((6, 10))
    M = np.zeros_like(G)
    lam = 0.06
    W1, M1, O = orc.muon_step(W, G, M, 0.9, True, 0.1, form="standard", soft_threshold=lam)
    _, U = orc.momentum_update(M, G, 0.9, True)
    assert np.allclose(M1, G)  # the momentum buffer keeps the outlier
    expect = orc.orthogonalize(np.clip(U, -lam / 2, lam / 2), form="standard")
    assert np.allclose(O, expect, rtol=0, atol=1e-14)
    # without the split the outlier dominates: the two updates differ
    _, _, O_plain = orc.muon_step(W, G, M, 0.9, True, 0.1, form="standard")
    assert np.linalg.norm(O - O_plain) > 0.1


@pytest.mark.parametrize("shape", [(16, 48), (24, 24), (7, 90)])
def test_gram_q_closed_form(shape):
    """[Gram-NS] "ข้อได้เปรียบของอัลกอริทึม": the Gram iteration's Q is a
    polynomial in R0 = X0 X0^T that approximates R0^{-1/2}.  Without restarts,
    in R0's eigenbasis (eigenvalues l = sigma^2) Q is diagonal with entries
    f(sigma) / sigma, f the composed quintic: checked against numpy's
    symmetric eigendecomposition."""
    r = _rng(40 + shape[0])
    X = r.standard_normal(shape)
    X /= np.linalg.norm(X)
    _, Q, X_last = orc.ns_gram(X, orc.TUNED_COEFFS, 5, restarts=(), return_q=True)
    assert np.array_equal(X_last, X)
    lam, V = np.linalg.eigh(X @ X.T)
    sigma = np.sqrt(np.maximum(lam, 0.0))
    f = sigma.copy()
    for _ in range(5):
        a, b, c = orc.TUNED_COEFFS
        f = a * f + b * f ** 3 + c * f ** 5
    expect = V @ np.diag(f / sigma) @ V.T
    assert np.allclose(Q, expect, rtol=1e-9, atol=1e-9 * np.abs(expect).max())
    # with the classic coefficients and many steps, Q -> R0^{-1/2}
    _, Q40, _ = orc.ns_gram(X, orc.CLASSIC_COEFFS, 40, restarts=(), return_q=True)
    inv_sqrt = V @ np.diag(1.0 / sigma) @ V.T
    assert np.allclose(Q40, inv_sqrt, rtol=1e-6, atol=1e-6 * np.abs(inv_sqrt).max())

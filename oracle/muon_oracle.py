"""Plain fp64 CPU oracle for one Muon optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA path.

Every function follows the steps of the method in the order the sources give
them, in fp64 NumPy, with ``@`` (a library matmul) as the only primitive.
There is no blocking, fusion or reordering beyond what the method states.

Sources (web pages; formulas were lost in extraction, the prose survives):

* [Gram-NS] "GPU เร่งความเร็วใหม่! อัลกอริทึม Gram Newton-Schulz ..." (itsolotime.com),
  sections "ข้อได้เปรียบของอัลกอริทึม" (Muon as steepest descent under the
  spectral norm; polar(X) = U V^T; the standard iteration costs three matrix
  products per step; an odd polynomial p(t) = t q(t^2) moves the iteration
  onto R = X X^T, which approximates R^{-1/2}) and
  "ความท้าทายด้านความเสถียรและแนวทางแก้ไข" (naive Gram form is unstable in
  float16; restart that re-forms the Gram matrix).
* [NanoGPT-Muon] "2 分钟训练 124M 参数 NanoGPT：Muon 优化器与工程复现实践"
  (blog.hotdry.top), sections "从 SGD 到 Muon" (orthogonalise the
  SGD-momentum update; exact route is an SVD), "Newton-Schulz 迭代的系数调优与
  FLOP 开销分析" (coefficients (3.4445, -4.7750, 2.0315), five steps, older
  (2, -1.5, 0.5)), "工程复现清单" (momentum 0.95, nesterov=True, lr 6e-4).

Readings where the sources are silent:

* momentum: M <- mu*M + G; Nesterov U = G + mu*M, else U = M;
* Frobenius normalisation X0 = U / (||U||_F + eps), eps = 1e-7;
* the Gram side is the shorter one: a matrix with rows > cols is transposed;
* update W <- W - lr * O with no extra shape factor and no weight decay;
* restart schedule: a set of step indices at which X is re-materialised;
* soft-threshold split ([ROOT] "ROOT优化器的技术创新"): outliers are the
  soft-thresholded momentum at lam / 2, the robust part is the rest.
"""
from __future__ import annotations

import numpy as np

TUNED_COEFFS = (3.4445, -4.7750, 2.0315)
CLASSIC_COEFFS = (2.0, -1.5, 0.5)
DEFAULT_EPS = 1e-7
DEFAULT_RESTARTS = (2,)


def _coeff_list(coeffs, steps):
    """Per-step (a, b, c): a single triple is repeated for every step."""
    c = np.asarray(coeffs, dtype=np.float64).reshape(-1, 3)
    if c.shape[0] == 1:
        c = np.repeat(c, steps, axis=0)
    if c.shape[0] < steps:
        raise ValueError("need one (a, b, c) triple per step")
    return [tuple(row) for row in c[:steps]]


def momentum_update(M, G, mu, nesterov):
    """SGD momentum with optional Nesterov look-ahead ([NanoGPT-Muon] "工程复现清单";
    [Gram-NS] "ข้อได้เปรียบของอัลกอริทึม": mu is the momentum coefficient).

    Returns (M_new, U): the new momentum buffer and the matrix Muon
    orthogonalises.
    """
    M = np.asarray(M, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M_new = mu * M + G
    U = G + mu * M_new if nesterov else M_new
    return M_new, U


def frobenius_normalize(U, eps=DEFAULT_EPS):
    """X0 = U / (||U||_F + eps).  Frobenius norm >= spectral norm, so every
    singular value of X0 is at most 1, the interval the coefficients target."""
    U = np.asarray(U, dtype=np.float64)
    return U / (np.sqrt(np.sum(U * U)) + eps)


def ns_standard(X, coeffs=TUNED_COEFFS, steps=5):
    """Standard quintic Newton-Schulz on X (n x m, n <= m), T = steps.

    Per step ([Gram-NS] "ข้อได้เปรียบของอัลกอริทึม": three matrix products per
    step; [NanoGPT-Muon] "Newton-Schulz 迭代的系数调优"):
        A = X X^T
        B = b A + c A^2
        X = a X + B X
    which applies p(s) = a s + b s^3 + c s^5 to every singular value.
    """
    X = np.asarray(X, dtype=np.float64).copy()
    for a, b, c in _coeff_list(coeffs, steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X


def ns_gram(X, coeffs=TUNED_COEFFS, steps=5, restarts=DEFAULT_RESTARTS, return_q=False):
    """Gram Newton-Schulz with restarts on X (n x m, n <= m).

    [Gram-NS] "ข้อได้เปรียบของอัลกอริทึม": the odd polynomial is p(t) = t q(t^2),
    so the iteration runs on R = X X^T (n x n) and the result is Q X with Q a
    polynomial in R.  With X_k = Q_k X_0 and R_k = X_k X_k^T one step is
        Z = a I + b R + c R^2      (q evaluated at R)
        Q <- Z Q
        R <- Z R Z                 (= X_{k+1} X_{k+1}^T, Z and R commute)
    [Gram-NS] "ความท้าทายด้านความเสถียรและแนวทางแก้ไข": a restart re-forms the
    Gram matrix from the current iterate: X <- Q X, R <- X X^T, Q <- I.
    ``restarts`` lists the step indices k (0 < k < steps) at which that
    happens before step k is taken.  The output is Q X (with return_q, also
    the last segment's Q and the X it multiplies).
    """
    X = np.asarray(X, dtype=np.float64).copy()
    n = X.shape[0]
    I = np.eye(n)
    R = X @ X.T
    Q = I.copy()
    for k, (a, b, c) in enumerate(_coeff_list(coeffs, steps)):
        if k in restarts and k > 0:
            X = Q @ X
            R = X @ X.T
            Q = I.copy()
        Z = a * I + b * R + c * (R @ R)
        Q = Z @ Q
        R = Z @ R @ Z
    if return_q:
        return Q @ X, Q, X
    return Q @ X


def orthogonalize(U, coeffs=TUNED_COEFFS, steps=5, form="standard",
                  eps=DEFAULT_EPS, restarts=DEFAULT_RESTARTS):
    """NS(U / (||U||_F + eps)) for one r x c matrix, in U's layout.

    The iteration runs on the short side ([Gram-NS]: the Gram matrix lives on
    the smaller dimension): a matrix with rows > cols is transposed first and
    transposed back at the end.
    """
    U = np.asarray(U, dtype=np.float64)
    trans = U.shape[0] > U.shape[1]
    X = frobenius_normalize(U.T if trans else U, eps)
    if form == "standard":
        O = ns_standard(X, coeffs, steps)
    elif form == "gram":
        O = ns_gram(X, coeffs, steps, restarts)
    else:
        raise ValueError(form)
    return O.T if trans else O


def soft_threshold_split(M, lam):
    """Split of a momentum matrix into a robust part and an outlier part
    ([ROOT] "ROOT优化器的技术创新": soft-threshold denoising, objective
    min ||M - B - O||_F^2 + lam ||O||_1, only the robust part B is
    orthogonalised).

    Reading: O is the minimiser of ||M - O||_F^2 + lam ||O||_1, which is
    elementwise soft-thresholding at lam / 2,
        O = sign(M) * max(|M| - lam/2, 0),
    and B = M - O is what remains (M clipped to [-lam/2, lam/2]).
    Returns (B, O).
    """
    M = np.asarray(M, dtype=np.float64)
    O = np.sign(M) * np.maximum(np.abs(M) - lam / 2.0, 0.0)
    return M - O, O


def muon_step(W, G, M, mu=0.95, nesterov=True, lr=6e-4, coeffs=TUNED_COEFFS,
              steps=5, form="standard", eps=DEFAULT_EPS,
              restarts=DEFAULT_RESTARTS, soft_threshold=0.0):
    """One Muon step for one 2D parameter ([Gram-NS] "ข้อได้เปรียบของอัลกอริทึม";
    [NanoGPT-Muon] "从 SGD 到 Muon"): momentum, orthogonalise, W <- W - lr * O.
    With soft_threshold = lam > 0 the matrix orthogonalised is the robust
    part of U ([ROOT] "ROOT优化器的技术创新", see soft_threshold_split);
    the momentum buffer keeps the full M.

    Returns (W_new, M_new, O).
    """
    M_new, U = momentum_update(M, G, mu, nesterov)
    if soft_threshold > 0:
        U, _ = soft_threshold_split(U, soft_threshold)
    O = orthogonalize(U, coeffs, steps, form, eps, restarts)
    W_new = np.asarray(W, dtype=np.float64) - lr * O
    return W_new, M_new, O


def ns_flops(n, m, steps=5, form="standard", restarts=DEFAULT_RESTARTS):
    """Algorithmic FLOPs of one orthogonalisation of an n x m matrix (n <= m)
    with symmetric-output products counted at half cost.

    standard, per step: X X^T (n^2 m), A A (n^3), B X (2 n^2 m).
    Gram: each segment starts with X X^T (n^2 m); per step R R (n^3), plus
    Z Q (n^3) unless it is the segment's first step, plus Z R and Z (Z R)
    (2 n^3) unless it is the segment's last step; each segment ends with one
    Q X (2 n^2 m).
    """
    if form == "standard":
        return steps * (3 * n * n * m + n ** 3)
    starts = [0] + sorted(k for k in set(restarts) if 0 < k < steps)
    ends = starts[1:] + [steps]
    total = 0
    for s, e in zip(starts, ends):
        total += 3 * n * n * m
        for k in range(s, e):
            total += n ** 3
            if k > s:
                total += n ** 3
            if k < e - 1:
                total += 2 * n ** 3
    return total


def adamw_step(p, g, m, v, step, lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8,
               weight_decay=0.1):
    """One AdamW step for a parameter that Muon does not handle (embeddings,
    output head, 1-D parameters: [NanoGPT-Muon] "从 SGD 到 Muon" and
    "工程复现清单", lr 6e-4, betas (0.9, 0.95), weight decay 0.1).

    Decoupled weight decay, then the bias-corrected Adam update, in the
    plainest reading of AdamW:
        p <- p - lr * wd * p
        m <- beta1 m + (1 - beta1) g
        v <- beta2 v + (1 - beta2) g^2
        p <- p - lr * (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
    `step` is t >= 1 (the step being taken).  Returns (p, m, v).
    """
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    p = p - lr * weight_decay * p
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v

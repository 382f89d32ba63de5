"""Shared helpers of the test suites (comparison metrics and tolerances)."""
import numpy as np

# Tolerances of the Newton-Schulz output against the fp64 oracle on the same
# (already rounded) inputs: relative Frobenius error and the largest change
# of any singular value.
TOL_BF16_RELF = 2e-2
TOL_FP32_RELF = 1e-5
TOL_SIGMA = 2e-2


def relF(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def sigma_maxdiff(a, b):
    sa = np.linalg.svd(np.asarray(a, dtype=np.float64), compute_uv=False)
    sb = np.linalg.svd(np.asarray(b, dtype=np.float64), compute_uv=False)
    return float(np.max(np.abs(sa - sb))) if sa.size else 0.0


def to64(t):
    return t.detach().to("cpu").double().numpy()

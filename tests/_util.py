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


def fmaf32(a, b, c):
    """Elementwise fp32 fused multiply-add a*b + c with ONE rounding to fp32
    (round to nearest even), as the GPU's fmaf computes it, for fp32-exact
    operands given as float64 arrays.

    a*b is exact in fp64 when a and b carry at most 24 significant bits each
    (48 bits < 53).  s = p + c is then rounded once to fp64 and the TwoSum
    error e = (p + c) - s is exact.  Rounding s to fp32 gives the correctly
    rounded result unless s lies exactly on a midpoint between two fp32
    neighbours (no other fp32 midpoint can separate s from p + c, since every
    fp32 midpoint is an fp64 number); there the sign of e decides."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    p = a * b
    s = p + c
    bb = s - p
    e = (p - (s - bb)) + (c - bb)
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    d = s - r64                      # exact: |d| <= half an fp32 ulp of s
    with np.errstate(over="ignore", invalid="ignore"):
        up = np.nextafter(r, np.float32(np.inf)).astype(np.float64)
        dn = np.nextafter(r, np.float32(-np.inf)).astype(np.float64)
    tie_up = (d > 0) & (d == (up - r64) / 2)   # s is the midpoint of (r, up)
    tie_dn = (d < 0) & (d == (dn - r64) / 2)   # s is the midpoint of (dn, r)
    out = r64.copy()
    out = np.where(tie_up & (e > 0), up, out)
    out = np.where(tie_dn & (e < 0), dn, out)
    return out


def bf16_round(x64):
    """Round float64 values (already fp32-exact) to bf16, nearest even, as
    float64."""
    import torch
    return torch.from_numpy(np.asarray(x64, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()

"""The tests' emulation of the GPU's fp32 fused multiply-add, checked
against exact rational arithmetic (it decides bitwise momentum parity)."""
from fractions import Fraction

import numpy as np

from tests._util import bf16_round, fmaf32


def _exact_fmaf32(a, b, c):
    """a*b + c computed exactly, then rounded to fp32 (nearest, ties to even)."""
    x = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    f = np.float32(float(x))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    return float(min(cands, key=lambda y: (abs(Fraction(float(y)) - x), int(np.float32(y).view(np.uint32)) & 1)))


def test_fmaf32_random_operands():
    rng = np.random.default_rng(5)
    a = np.float32(0.95)
    M = rng.standard_normal(4000).astype(np.float32)
    G = (rng.standard_normal(4000) * np.exp(rng.uniform(-30, 30, 4000))).astype(np.float32)
    got = fmaf32(np.float64(a), M.astype(np.float64), G.astype(np.float64))
    for i in range(len(M)):
        assert got[i] == _exact_fmaf32(a, M[i], G[i])


def test_fmaf32_midpoint_cases():
    """(1 + 2^-12)^2 = 1 + 2^-11 + 2^-24 lies exactly between two fp32
    neighbours: a tiny addend decides the rounding.  fp64 evaluation followed
    by a second rounding to fp32 gets these wrong; the emulation must not."""
    a = np.float32(1 + 2 ** -12)
    cases = [(s * a, a, np.float32(c)) for s in (1, -1) for c in (2.0 ** -80, -2.0 ** -80, 0.0, 2.0 ** -60)]
    A = np.array([x[0] for x in cases], dtype=np.float64)
    B = np.array([x[1] for x in cases], dtype=np.float64)
    C = np.array([x[2] for x in cases], dtype=np.float64)
    got = fmaf32(A, B, C)
    naive = (A * B + C).astype(np.float32).astype(np.float64)
    want = np.array([_exact_fmaf32(*x) for x in cases])
    assert np.array_equal(got, want)
    assert not np.array_equal(naive, want)  # the cases do exercise the ties


def test_bf16_round_nearest_even():
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties to even -> 1
    assert bf16_round(np.array([1 + 2 ** -8]))[0] == 1.0
    assert bf16_round(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6

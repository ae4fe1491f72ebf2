"""The load-time pack's two shortcuts, checked on the CPU against the oracle.

[Production] "1. Absmean Weight Quantization": gamma = mean |W| (read as
max(RN32(RN64(S) / (N K)), 1e-5) with S the exact sum of |W|) and
t = Clip(Round(W / gamma), -1, 1) (read as RNE of the IEEE fp32 quotient).

  * Ternarisation: the kernels compare w with the fp32 threshold
    T = RD32(gamma (0.5 + 2^-25)) instead of dividing: t = +1 iff w > T,
    -1 iff w < -T.  Checked against IEEE fp32 division for many gamma and
    every fp32 within 64 ulps of the thresholds, and against the oracle's
    ternarise on whole matrices.
  * gamma: the kernels sum |W| in fp64 and take gamma from that sum when
    the bound |S^ - S| <= 1.003 h 2^-53 S^ + count 2^-126 (h = the
    summation tree's height) makes both ends of the interval round to the
    same gamma; else the exact integer buckets.  Checked: the bound holds
    against exact rational sums, a decided gamma is the oracle's, and
    matrices whose mean |W| sits on an fp32 rounding midpoint are never
    decided.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import reference as ref

M_HALF = Fraction(1, 2) + Fraction(1, 2 ** 25)


def rd32(q):
    """The largest fp32 <= the rational q (q > 0, in the normal range)."""
    f = np.float32(float(q))  # nearest (fp64 then fp32: at most one ulp off)
    while Fraction(float(f)) > q:
        f = np.nextafter(f, np.float32(-np.inf))
    while Fraction(float(np.nextafter(f, np.float32(np.inf)))) <= q:
        f = np.nextafter(f, np.float32(np.inf))
    return f


def threshold(gamma):
    return rd32(Fraction(float(gamma)) * M_HALF)


def around(v, n=64):
    out = [v]
    a = b = v
    for _ in range(n):
        a = np.nextafter(a, np.float32(-np.inf))
        b = np.nextafter(b, np.float32(np.inf))
        out += [a, b]
    return np.array(out, np.float32)


def gammas():
    rng = np.random.default_rng(3)
    g = [np.float32(1e-5), np.float32(1.0), np.float32(0.02), np.float32(3.0),
         np.float32(np.nextafter(np.float32(2.0), np.float32(0))), np.float32(1e30)]
    g += list(np.exp(rng.uniform(np.log(1e-5), np.log(1e3), 200)).astype(np.float32))
    return g


def test_threshold_matches_ieee_division_near_every_boundary():
    for g in gammas():
        T = threshold(g)
        half = np.float32(g) * np.float32(0.5)  # gamma / 2, exact
        ws = np.concatenate([around(T), around(half), around(np.float32(1.5) * g)])
        ws = np.concatenate([ws, -ws])
        q = ws / np.float32(g)  # IEEE fp32 division, round to nearest even
        want = np.clip(np.rint(q), -1, 1)
        got = np.where(ws > T, 1, np.where(ws < -T, -1, 0))
        np.testing.assert_array_equal(got, want, err_msg=f"gamma={g!r}")


def test_threshold_matches_the_oracle_ternarise():
    rng = np.random.default_rng(4)
    for dist in ("normal", "laplace"):
        W = (rng.normal(0, 0.02, (64, 257)) if dist == "normal"
             else rng.laplace(0, 0.02, (64, 257))).astype(np.float32)
        gamma, _ = ref.absmean_gamma(W)
        T = threshold(gamma)
        W[0, :129] = around(T)  # every weight within 64 ulps of the threshold
        W[1, :129] = -around(T)
        gamma2, _ = ref.absmean_gamma(W)
        T2 = threshold(gamma2)
        t = ref.ternarise(W, gamma2)
        np.testing.assert_array_equal(np.where(W > T2, 1, np.where(W < -T2, -1, 0)), t)


def decide(absw, h):
    """gamma from an fp64 sum with tree height h, as k_gamma_decide forms
    it; outward rounding replaced by one extra ulp at each end (stricter)."""
    S = 0.0
    for v in absw.ravel():
        S = S + float(v)
    count = absw.size
    B = 1.003 * h * 2.0 ** -53 * S + count * 2.0 ** -126
    lo = max(math.nextafter(S - B, -math.inf), 0.0)
    hi = math.nextafter(S + B, math.inf)
    a = max(np.float32(lo / count), np.float32(1e-5))
    b = max(np.float32(hi / count), np.float32(1e-5))
    return a == b, a, S


@pytest.mark.parametrize("shape", [(1, 8), (8, 64), (40, 250)])
def test_fp64_gamma_within_bound_and_decided_correctly(shape):
    rng = np.random.default_rng(shape[1])
    for W in ((rng.normal(0, 0.02, shape)).astype(np.float32),
              (rng.standard_normal(shape) * np.exp2(rng.integers(-60, 60, shape))).astype(np.float32)):
        a = np.abs(W)
        ok, g, S = decide(a, a.size)  # a sequential sum: height = count
        exact = sum(Fraction(float(v)) for v in a.ravel())
        B = Fraction(1.003) * a.size * Fraction(2) ** -53 * Fraction(S) + a.size * Fraction(2) ** -126
        assert abs(Fraction(S) - exact) <= B
        want, _ = ref.absmean_gamma(W)
        if ok:
            assert g == want


@pytest.mark.parametrize("n", [1, 8, 500])
def test_midpoint_matrices_are_never_decided_by_the_fp64_sum(n):
    """n weights 2^k and n weights 2^(k-24) (and 8n - 2n zeros): mean |W| =
    2^k (1 + 2^-24) / 8, the midpoint between two fp32 values; with n more
    weights 2^(k-50) it lies 2^-50 (relative) above it."""
    for k in (-3, 0, 5):
        for extra in (False, True):
            W = np.zeros(8 * n, np.float32)
            W[:n] = 2.0 ** k
            W[n:2 * n] = -(2.0 ** (k - 24))
            if extra:
                W[2 * n:3 * n] = 2.0 ** (k - 50)
            ok, _, _ = decide(np.abs(W), W.size + 20)
            assert not ok
            want = np.float32(2.0 ** (k - 3))
            if extra:
                want = np.nextafter(want, np.float32(np.inf))
            g, _ = ref.absmean_gamma(W.reshape(1, -1))
            assert g == want

"""Pins of the oracle's RMSNorm (no affine, eps = 1e-6, before the
quantiser) against exact arithmetic, closed forms and planted mistakes."""
from fractions import Fraction
import math

import numpy as np
import pytest

from oracle import reference as ref


def exact_norm(row):
    """x / sqrt(mean(x^2) + 1e-6) in exact rationals except for one square
    root taken in 60-digit decimal arithmetic."""
    import decimal
    decimal.getcontext().prec = 60
    K = len(row)
    ms = sum(Fraction(float(v)) ** 2 for v in row) / K + Fraction(float(np.float32(1e-6)))
    d = decimal.Decimal(ms.numerator) / decimal.Decimal(ms.denominator)
    root = d.sqrt()
    return [float(decimal.Decimal(float(v)) / root) for v in row]


def ulps(a, b):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float64).astype(np.float32)
    return np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))


@pytest.mark.parametrize("seed,K,scale", [(0, 64, 1.0), (1, 3200, 1.0), (2, 257, 1e-3), (3, 1000, 30.0)])
def test_rmsnorm_within_a_few_ulps_of_the_exact_value(seed, K, scale):
    rng = np.random.default_rng(seed)
    x = (rng.normal(0, scale, (2, K))).astype(np.float32)
    got = ref.rmsnorm(x)
    for m in range(2):
        # five fp32 roundings (mean, +eps, sqrt, 1/s, x*r): a few ulps at most
        assert ulps(got[m], exact_norm(x[m])).max() <= 4


def test_constant_row_closed_form():
    x = np.full((1, 64), 0.5, np.float32)
    got = ref.rmsnorm(x)
    want = 0.5 / math.sqrt(0.25 + float(np.float32(1e-6)))
    assert ulps(got[0], [want] * 64).max() <= 2
    assert np.all(got[0] == got[0, 0])


def test_zero_row_quantises_to_zero_with_the_eta_floor():
    x = np.zeros((1, 128), np.float32)
    xq, eta, xsum = ref.rmsnorm_quant_act(x)
    assert not xq.any() and eta[0] == np.float32(1e-5) and xsum[0] == 0


def test_largest_value_maps_to_127_and_sign_is_kept():
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (3, 512)).astype(np.float32)
    xq, eta, _ = ref.rmsnorm_quant_act(x)
    for m in range(3):
        k = np.argmax(np.abs(x[m]))
        assert abs(int(xq[m, k])) == 127 and np.sign(xq[m, k]) == np.sign(x[m, k])
        assert np.all(np.sign(xq[m])[xq[m] != 0] == np.sign(x[m])[xq[m] != 0])


def test_planted_mistakes_fail():
    rng = np.random.default_rng(4)
    x = (rng.normal(0, 1e-3, (1, 257))).astype(np.float32)  # mean(x^2) ~ eps: eps placement matters
    exact = exact_norm(x[0])
    good = ref.rmsnorm(x)[0]
    assert ulps(good, exact).max() <= 4
    # eps outside the square root
    bad1 = x[0] / (np.sqrt(np.float32(np.mean(x[0].astype(np.float64) ** 2))) + np.float32(1e-6))
    assert ulps(bad1, exact).max() > 4
    # sum instead of mean
    bad2 = x[0] / np.sqrt(np.float32(np.sum(x[0].astype(np.float64) ** 2)) + np.float32(1e-6))
    assert ulps(bad2, exact).max() > 4
    # eps 1e-5 (the quantisers' floor) in place of 1e-6
    bad3 = x[0] / np.sqrt(np.float32(np.mean(x[0].astype(np.float64) ** 2)) + np.float32(1e-5))
    assert ulps(bad3, exact).max() > 4
    # mean over K - 1 values
    bad4 = x[0] / np.sqrt(np.float32(np.sum(x[0].astype(np.float64) ** 2) / 256) + np.float32(1e-6))
    assert ulps(bad4, exact).max() > 4

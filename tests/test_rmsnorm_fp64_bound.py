"""The fp64 shortcut of the streamed RMSNorm kernel, checked on the CPU.

[Production] "2. Absmax Dynamic Activation Quantization" normalises with
RMSNorm, mean(x^2) read as RN32(RN64(exact sum of x^2) / K).  The streamed
kernel (k_rmsnorm_rows) sums the squares in fp64 instead and takes that
mean only when an error bound proves it; otherwise it sums exactly.  This
test replays the kernel's summation tree in fp64 (256 threads, each adding
the squares of its 16-byte vectors in order; a 32-lane xor butterfly; thread
0 adding the 8 warp sums in order -- bf16 squares are exact in fp64, so each
DFMA is one rounded fp64 add) and checks, against exact rational sums:
  * |S^ - S| <= B = 1.003 h 2^-53 S^ + K 2^-252 (h = the tree height);
  * whenever both ends of [S^ - B, S^ + B] give the same mean, it is the
    oracle's mean;
  * rows whose mean lies on a rounding midpoint are never decided by it.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import reference as ref
from ternary_weight_linear_04_b200 import inputs

NT, NWARP = 256, 8


def kernel_fp64_sum(x):
    """S^ for one row as the kernel forms it (x: bf16 values as float32)."""
    K = x.size
    nv = K // 8
    sq = np.square(x.astype(np.float64))  # exact for bf16 values
    lane_sums = np.zeros(NT)
    for t in range(NT):
        s = 0.0
        for v in range(t, nv, NT):
            for e in sq[8 * v:8 * v + 8]:
                s = s + float(e)
        lane_sums[t] = s
    warp_sums = []
    for w in range(NWARP):
        vals = [float(v) for v in lane_sums[32 * w:32 * w + 32]]
        for o in (16, 8, 4, 2, 1):
            vals = [vals[l] + vals[l ^ o] for l in range(32)]
        warp_sums.append(vals[0])
    S = warp_sums[0]
    for w in range(1, NWARP):
        S = S + warp_sums[w]
    h = 8 * ((nv + NT - 1) // NT) + 5 + (NWARP - 1)
    return S, h


def mean_f32(S, K):
    return np.float32(S / K)


def decide(x):
    """(decided, mean) as the kernel's thread 0 forms them.  Directed
    rounding is replaced by widening the interval by one ulp at each end,
    which only makes the check stricter than the kernel's."""
    K = x.size
    S, h = kernel_fp64_sum(x)
    B = 1.003 * h * 2.0 ** -53 * S + K * 2.0 ** -252
    lo = max(math.nextafter(S - B, -math.inf), 0.0)
    hi = math.nextafter(S + B, math.inf)
    a, b = mean_f32(lo, K), mean_f32(hi, K)
    return a == b, a, S, h


def exact_sum(x):
    return sum(Fraction(float(v)) ** 2 for v in x)


def oracle_mean(x):
    S = math.fsum(float(v) * float(v) for v in x)
    return np.float32(S / x.size)


@pytest.mark.parametrize("K", [8, 64, 520, 3200, 8640])
@pytest.mark.parametrize("dist", ["normal", "student_t_outliers", "laplace_wide"])
def test_fp64_sum_within_bound_and_decides_correctly(K, dist):
    rng = np.random.default_rng(K)
    if dist == "laplace_wide":
        x = rng.laplace(0.0, 1.0, (6, K)) * np.exp2(rng.integers(-60, 60, size=(6, K)))
        x = inputs.to_bf16_values(x.astype(np.float32))
    else:
        x = inputs.draw_activations(rng, 6, K, dist, "bf16")
    for row in x:
        ok, m, S, h = decide(row)
        err = abs(Fraction(S) - exact_sum(row))
        B = Fraction(1.003) * h * Fraction(2) ** -53 * Fraction(S) + K * Fraction(2) ** -252
        assert err <= B
        if ok:
            assert m == oracle_mean(row)


@pytest.mark.parametrize("K", [8, 64, 3200])
def test_midpoint_rows_go_to_the_exact_sum(K):
    """K/8 values 2^k and K/8 values 2^(k-12): mean(x^2) = 4^k (1 + 2^-24) / 8,
    the midpoint of two fp32 values; with K/8 more values 2^(k-25) the mean
    lies 2^-50 (relative) above it, a distance RN64 keeps but the fp64 sum's
    bound does not resolve.  Neither may be decided in fp64."""
    for k in (-3, 0, 1, 7):
        for extra in (False, True):
            n = K // 8
            row = np.zeros(K, np.float32)
            row[:n] = 2.0 ** k
            row[n:2 * n] = 2.0 ** (k - 12)
            if extra:
                row[2 * n:3 * n] = 2.0 ** (k - 25)
            ok, _, _, _ = decide(row)
            assert not ok
            # the exact mean is the tie to even, or rounded up
            want = np.float32(2.0 ** (2 * k - 3))
            if extra:
                want = np.nextafter(want, np.float32(np.inf))
            assert oracle_mean(row) == want
            assert ref.rmsnorm(row[None, :]).shape == (1, K)


def test_zeros_and_subnormals_only_widen_the_bound():
    """Zeros and subnormal bf16 values widen to wrong fp64 values below
    2^-126 in the kernel; rows of them still decide the mean (0) or fall
    back, never decide it wrongly."""
    rng = np.random.default_rng(1)
    for K in (8, 64, 3200):
        bits = rng.integers(1, 0x80, size=K).astype(np.uint32)  # subnormal bf16 patterns
        sub = (bits << 16).view(np.float32)
        for row in (np.zeros(K, np.float32), sub, np.concatenate([sub[:-1], [1.0]]).astype(np.float32)):
            # the kernel's widening: exponent field 0 reads as 2^-127 (1 + m/128)
            h = (row.view(np.uint32) >> 16) & 0x7FFF
            e0 = (h >> 7) == 0
            widened = np.where(e0, 2.0 ** -127 * (1 + (h & 0x7F) / 128.0), np.abs(row.astype(np.float64)))
            ok, m, _, _ = decide(widened.astype(np.float32))
            if ok:
                assert m == oracle_mean(row)

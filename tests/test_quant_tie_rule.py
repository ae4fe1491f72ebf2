"""Exhaustive host check of the division-free rule the CUDA quantiser uses
for bf16 activations (the kernel's own results are checked against the
oracle by the GPU tests; this pins the arithmetic argument itself).

For x and eta both bf16 values, the kernel takes the candidate
n0 = RNE(RN32(x * RN32(127 * RN32(1/eta)))), forms e = 127x - n0*eta with
one fma, and moves n0 by one when |e| > eta/2 (to the even neighbour when
|e| = eta/2).  The claims checked here, for every bf16 x with |x| <= eta and
every bf16 mantissa of eta at several exponents:
  * e is exactly representable in fp32 (so the fma gives it exactly);
  * the corrected code equals RNE(RN32(RN32(127x)/eta)), the definition of
    [Production] "2. Absmax Dynamic Activation Quantization" (product and
    quotient each rounded once in fp32, round half to even).
"""
import numpy as np
import pytest

MAGIC = np.float32(12582912.0)  # 1.5 * 2^23


def _all_bf16_upto(eta):
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[v <= eta]
    return np.concatenate([v, -v[1:]])


def _rule(x, eta):
    f32 = np.float32
    s = f32(f32(127.0) * f32(f32(1.0) / eta))
    c = (x * s).astype(np.float32)
    t = (c + MAGIC).astype(np.float32)
    n0 = (t - MAGIC).astype(np.float32)
    e64 = x.astype(np.float64) * 127.0 - n0.astype(np.float64) * np.float64(eta)
    assert np.all(e64.astype(np.float32).astype(np.float64) == e64), "e not exact in fp32"
    h = np.float64(eta) / 2
    n = n0.astype(np.int64)
    n = n + (e64 > h) - (e64 < -h)
    tie = np.abs(e64) == h
    odd = (n0.astype(np.int64) & 1) == 1
    n = np.where(tie & odd, n0.astype(np.int64) + np.sign(e64).astype(np.int64), n)
    return n


def _reference(x, eta):
    a = (x * np.float32(127.0)).astype(np.float32)
    q = (a / eta).astype(np.float32)  # IEEE fp32 division
    return np.clip(np.rint(q), -127, 127).astype(np.int64)


@pytest.mark.parametrize("exp", [-12, -3, 0, 5, 20])
def test_tie_rule_matches_the_definition_for_every_bf16_pair(exp):
    ties = 0
    for m in range(128, 256):
        eta = np.float32(np.ldexp(m / 128.0, exp))
        x = _all_bf16_upto(eta)
        got = _rule(x, eta)
        ref = _reference(x, eta)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, (m, exp, x[bad[:5]], got[bad[:5]], ref[bad[:5]])
        q = ((x * np.float32(127)).astype(np.float32) / eta).astype(np.float32)
        ties += int(np.count_nonzero(q - np.floor(q) == 0.5))
    assert ties > 100  # exact .5 ties do occur among bf16 ratios, so the tie branch is exercised


def test_naive_candidate_alone_is_wrong_on_ties():
    """Without the correction the fast candidate is wrong for some values
    (eta = 135/128 has two among its 32765 bf16 inputs): the rule is
    needed, not decorative."""
    eta = np.float32(135 / 128.0)
    x = _all_bf16_upto(eta)
    f32 = np.float32
    s = f32(f32(127.0) * f32(f32(1.0) / eta))
    naive = np.rint((x * s).astype(np.float32)).astype(np.int64)
    assert np.count_nonzero(naive != _reference(x, eta)) > 0

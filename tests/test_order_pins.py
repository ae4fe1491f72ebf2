"""Pins of the oracle's fp32 evaluation orders, on inputs where the order
decides the result.

The expected values in ``golden/fp32_order_pins.json`` are exact rational
evaluations of the readings (``golden/make_order_pins.py`` computes them with
``fractions.Fraction`` and an explicit IEEE round-to-nearest-even; it calls
neither the oracle nor the CUDA library).  Each case also records what the
plausible other orders give, and those differ from the expected value:

* quantiser, [Production] "2. Absmax Dynamic Activation Quantization"
  (``x * 127.0 / eta``): RN32(RN32(x*127)/eta), not x*RN32(127/eta);
* rescale, [Production] pipeline step 5 and BitLinear158.forward
  (``(eta * gamma) / 127.0`` then times y): RN32(y * RN32(RN32(eta*gamma)/127));
* RMSNorm, [Production] BitLinear158.forward (``x * rsqrt(...)``):
  RN32(x * RN32(1 / RN32(sqrt v))), not a division by the root, not an fp64
  or correctly rounded reciprocal square root.

The ternarisation's divide-then-round reading needs no golden value: the last
test shows that it agrees with the compare |W| > gamma/2 on every fp32
input, so no input could tell the two apart.
"""
import json
import os

import numpy as np
import pytest

from oracle import native, reference

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "fp32_order_pins.json")))


def f32(bits):
    return np.array(bits, dtype=np.uint32).view(np.float32)


class _Native:
    @staticmethod
    def quant_act(x):
        return native.quant_act(x, nthreads=1)

    @staticmethod
    def forward(xq, eta, packed, gamma, K):
        return native.forward(xq, eta, packed, gamma, K, packed.shape[0], nthreads=1)


ORACLES = {"numpy": reference, "c": _Native}


@pytest.fixture(params=sorted(ORACLES))
def orc(request):
    return ORACLES[request.param]


def check_quantiser(orc):
    for case in GOLDEN["quantiser"]:
        x = f32(case["x_bits"])[None, :]
        xq, eta, xsum = orc.quant_act(x)
        assert np.asarray(eta, np.float32).view(np.uint32)[0] == case["eta_bits"]
        np.testing.assert_array_equal(np.asarray(xq)[0], case["xq"])
        assert int(np.asarray(xsum)[0]) == case["xsum"]


def _row_for(y_int):
    """An int8 row whose sum is y_int (entries within +-127)."""
    n = max(1, -(-abs(y_int) // 127))
    n += n % 2  # even length keeps a whole number of packed bytes simple
    q, r = divmod(abs(y_int), n)
    row = np.full(n, q, np.int64)
    row[:r] += 1
    return (np.sign(y_int) * row).astype(np.int8)


def check_rescale(orc):
    for case in GOLDEN["rescale"]:
        xq = _row_for(case["y_int"])[None, :]
        K = xq.shape[1]
        t = np.ones((1, K), np.int8)              # every weight +1: y_int = sum of the row
        packed = reference.pack2(t)
        eta = f32([case["eta_bits"]])
        gamma = f32([case["gamma_bits"]])[0]
        y_int, y = orc.forward(xq, eta, packed, gamma, K)
        assert int(np.asarray(y_int)[0, 0]) == case["y_int"]
        assert np.asarray(y, np.float32).view(np.uint32)[0, 0] == case["y_bits"], case


def check_rmsnorm(rmsnorm):
    for case in GOLDEN["rmsnorm"]:
        x = f32(case["x_bits"])[None, :]
        out = np.asarray(rmsnorm(x), np.float32)
        np.testing.assert_array_equal(out.view(np.uint32)[0], case["out_bits"])


def test_quantiser_order(orc):
    check_quantiser(orc)


def test_rescale_order(orc):
    check_rescale(orc)


def test_rmsnorm_order():
    check_rmsnorm(reference.rmsnorm)


def test_cases_separate_the_orders():
    """Each stored case is one on which the alternatives disagree with it."""
    for case in GOLDEN["quantiser"]:
        for k in case["separating_index"]:
            assert case["alternatives"]["x*RN32(127/eta)"][case["separating_index"].index(k)] != case["xq"][k]
    for case in GOLDEN["rescale"]:
        assert all(v != case["y_bits"] for v in case["alternatives_bits"].values())
    for case in GOLDEN["rmsnorm"]:
        assert all(case["alternatives_differ_at"].values())


def test_hand_worked_quantiser_case():
    """The first case, by hand: eta = 15, x = 7.5 -> 952.5 / 15 = 63.5 exactly
    -> 64 (half to even); 7.5 * RN32(127/15) = 63.4999962 -> 63."""
    case = GOLDEN["quantiser"][0]
    assert list(f32(case["x_bits"])) == [15.0, 7.5]
    assert case["xq"] == [127, 64]
    s = np.float32(np.float32(127) / np.float32(15))
    assert int(np.array(s).view(np.uint32)) == 0x41077777  # 8877943 / 2^20
    assert np.rint(np.float32(np.float32(7.5) * s)) == 63


def test_divide_then_round_equals_the_half_gamma_compare():
    """For fp32 W and gamma (normal), RNE(RN32(W/gamma)) is nonzero exactly
    when |W| > gamma/2: W/gamma never lands within half an fp32 ulp above
    0.5, because (W - gamma/2)/gamma >= ulp(gamma/2)/gamma > 2^-25.  Checked
    on every significand of gamma in [1, 2) with W at gamma/2 and its two
    fp32 neighbours, both signs (scaling by powers of two changes nothing)."""
    m = np.arange(1 << 23, dtype=np.uint32)
    gamma = ((m | 0x3F800000).view(np.float32))        # [1, 2)
    half = gamma * np.float32(0.5)                       # exact
    for W in (np.nextafter(half, np.float32(0)), half, np.nextafter(half, np.float32(2))):
        for sgn in (1, -1):
            Ws = (W * np.float32(sgn)).astype(np.float32)
            divide = np.clip(np.rint(Ws / gamma), -1, 1)
            compare = np.where(np.abs(Ws) > half, np.sign(Ws), 0)
            np.testing.assert_array_equal(divide, compare)


# --------------------------------------------------------------------------
# Planted mistakes: each other order, put into a copy of the oracle, fails
# --------------------------------------------------------------------------

class _QuantMutant:
    def __init__(self, scale_fn):
        self.scale_fn = scale_fn

    def quant_act(self, x):
        x = np.asarray(x, np.float32)
        eta = np.maximum(np.max(np.abs(x), axis=1).astype(np.float32), np.float32(1e-5))
        q = self.scale_fn(x, eta)
        xq = np.clip(np.rint(q), -127, 127).astype(np.int8)
        return xq, eta, xq.astype(np.int64).sum(axis=1)


def test_planted_quantiser_orders_fail():
    f = np.float32
    mutants = [
        lambda x, eta: (x * (f(127) / eta).astype(f)[:, None]).astype(f),          # x * RN32(127/eta)
        lambda x, eta: (x * (f(127) * (f(1) / eta).astype(f)).astype(f)[:, None]).astype(f),
        lambda x, eta: ((x / eta[:, None]).astype(f) * f(127)).astype(f),          # (x/eta)*127
    ]
    for mk in mutants:
        with pytest.raises(AssertionError):
            check_quantiser(_QuantMutant(mk))


def _forward_with(rescale):
    class M:
        @staticmethod
        def forward(xq, eta, packed, gamma, K):
            y_int = reference.accumulate(xq, reference.unpack2(packed, K))
            return y_int, rescale(y_int, np.asarray(eta, np.float32), np.float32(gamma))
    return M


def test_planted_rescale_orders_fail():
    f = np.float32
    mutants = [
        lambda y, eta, g: y.astype(f) * (eta * (g / f(127)))[:, None],              # eta * RN32(gamma/127)
        lambda y, eta, g: y.astype(f) * (g * (eta / f(127)))[:, None],              # gamma * RN32(eta/127)
        lambda y, eta, g: y.astype(f) * ((eta * g) * (f(1) / f(127)))[:, None],     # RN32(eta*gamma) * RN32(1/127)
        lambda y, eta, g: ((y.astype(f) * eta[:, None]) * g) / f(127),              # y*eta, *gamma, /127
    ]
    for mk in mutants:
        with pytest.raises(AssertionError):
            check_rescale(_forward_with(mk))


def test_planted_rmsnorm_orders_fail():
    import math

    def norm_with(r_fn):
        def rmsnorm(x):
            x = np.asarray(x, np.float32)
            out = np.empty_like(x)
            for m in range(x.shape[0]):
                S = math.fsum(float(v) * float(v) for v in x[m])
                v = np.float32(np.float32(S / x.shape[1]) + np.float32(1e-6))
                out[m] = r_fn(x[m], v)
            return out
        return rmsnorm

    f = np.float32
    mutants = [
        lambda row, v: row / np.sqrt(v, dtype=f),                                   # divide by the root
        lambda row, v: (row.astype(np.float64) * (1.0 / math.sqrt(float(v)))).astype(f),  # fp64 rsqrt
        lambda row, v: row * f(1.0 / math.sqrt(float(v))),                           # one-rounding rsqrt
    ]
    for mk in mutants:
        with pytest.raises(AssertionError):
            check_rmsnorm(norm_with(mk))
    # the reading itself, written the same way, passes
    check_rmsnorm(norm_with(lambda row, v: row * (f(1) / np.sqrt(v, dtype=f))))

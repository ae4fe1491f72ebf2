"""Writes ``fp32_order_pins.json``: inputs on which the order of the fp32
roundings decides the result, with the expected outputs worked out in exact
rational arithmetic.

Nothing here calls the oracle or the CUDA library.  Each expected value is
the definition evaluated with ``fractions.Fraction`` (exact) and one explicit
round-to-nearest-even to the IEEE format after every step the readings name;
``rn`` below is that rounding, written from the IEEE 754 definition (the
nearest representable value, ties to the even significand).

Readings pinned (page title tags as in the oracle's headers):

* quantiser, [Production] "2. Absmax Dynamic Activation Quantization",
  ActivationQuantizerSTE.forward, which writes ``x * 127.0 / eta``:
  x~ = RNE(RN32(RN32(x * 127) / eta)), eta = max(max |x|, 1e-5);
* rescale, [Production] pipeline figure step 5 and BitLinear158.forward,
  ``scale = (eta * gamma) / 127.0; output = y_raw * scale``:
  y = RN32(y_int * RN32(RN32(eta * gamma) / 127));
* RMSNorm, [Production] BitLinear158.forward (``x * rsqrt(mean(x^2) + eps)``,
  eps = 1e-6): v = RN32(RN32(RN64(sum x^2) / K) + RN32(1e-6)),
  r = RN32(1 / RN32(sqrt(v))), out = RN32(x * r).

The cases are chosen (by a search that only selects inputs) so that each
plausible other order gives a different answer; the "alternatives" field of
every case records those answers, evaluated the same exact way.

Run:  python tests/golden/make_order_pins.py   (rewrites the JSON beside it)
"""
import json
import math
import os
from fractions import Fraction

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "fp32_order_pins.json")


# ----------------------------------------------------------------------------
# IEEE round to nearest, ties to even, from the definition
# ----------------------------------------------------------------------------

def rn(v, p, emin):
    """Nearest number with a p-bit significand and exponent >= emin
    (subnormals below 2^emin), ties to the even significand."""
    v = Fraction(v)
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - p + 1)
    n = a / quantum
    whole = n.numerator // n.denominator
    rest = n - whole
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and whole % 2 == 1):
        whole += 1
    return sign * whole * quantum


def rn32(v):
    return rn(v, 24, -126)


def rn64(v):
    return rn(v, 53, -1022)


def rne_int(v):
    """Round half to even to an integer."""
    v = Fraction(v)
    whole = v.numerator // v.denominator
    rest = v - whole
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and whole % 2 == 1):
        whole += 1
    return whole


def fr(x):
    """The exact value of a float32 / float64 number."""
    return Fraction(float(x))


def bits32(v):
    """fp32 bit pattern of an exactly representable value."""
    f = np.float32(float(v))
    assert fr(f) == Fraction(v), "value is not an fp32 number"
    return int(np.array(f).view(np.uint32))


def f32_neighbours(c):
    f = np.float32(float(c))
    return (fr(np.nextafter(f, np.float32(-np.inf))), fr(np.nextafter(f, np.float32(np.inf))))


def rn32_sqrt(v):
    """RN32 of the exact square root of v >= 0: candidate from the fp64
    square root, then moved until v lies between the squares of the
    midpoints to its neighbours (an exact comparison)."""
    if v == 0:
        return Fraction(0)
    c = rn32(Fraction(math.sqrt(float(v))))
    for _ in range(8):
        lo, hi = f32_neighbours(c)
        m_hi, m_lo = (c + hi) / 2, (c + lo) / 2
        if v > m_hi * m_hi or (v == m_hi * m_hi and bits32(c) & 1):
            c = hi
        elif v < m_lo * m_lo or (v == m_lo * m_lo and bits32(c) & 1):
            c = lo
        else:
            return c
    raise AssertionError("square root rounding did not settle")


EPS_Q = rn32(Fraction(1, 100000))       # 1e-5 as an fp32 number
EPS_N = rn32(Fraction(1, 1000000))      # 1e-6 as an fp32 number


# ----------------------------------------------------------------------------
# The readings, exactly
# ----------------------------------------------------------------------------

def quant_row(x):
    """(x~ list, eta) for one row of fp32 values (as Fractions)."""
    eta = max(max(abs(v) for v in x), EPS_Q)
    return [max(-127, min(127, rne_int(rn32(rn32(v * 127) / eta)))) for v in x], eta


def quant_row_alternatives(x, eta):
    s = rn32(Fraction(127) / eta)
    inv = rn32(Fraction(1) / eta)
    return {
        "x*RN32(127/eta)": [rne_int(rn32(v * s)) for v in x],
        "RN32(x*RN32(127*RN32(1/eta)))": [rne_int(rn32(v * rn32(127 * inv))) for v in x],
        "RN32(RN32(x/eta)*127)": [rne_int(rn32(rn32(v / eta) * 127)) for v in x],
        "exact x*127/eta": [rne_int(v * 127 / eta) for v in x],
    }


def rescale(y_int, eta, gamma):
    return rn32(y_int * rn32(rn32(eta * gamma) / 127))


def rescale_alternatives(y_int, eta, gamma):
    return {
        "eta*RN32(gamma/127)": rn32(y_int * rn32(eta * rn32(gamma / 127))),
        "gamma*RN32(eta/127)": rn32(y_int * rn32(gamma * rn32(eta / 127))),
        "RN32(eta*gamma)*RN32(1/127)": rn32(y_int * rn32(rn32(eta * gamma) * rn32(Fraction(1, 127)))),
        "RN32(RN32(y*eta)*gamma)/127": rn32(rn32(rn32(y_int * eta) * gamma) / 127),
        "exact y*eta*gamma/127": rn32(Fraction(y_int) * eta * gamma / 127),
    }


def rmsnorm_row(x):
    K = len(x)
    S = sum(v * v for v in x)
    ms = rn32(rn64(rn64(S) / K))
    v = rn32(ms + EPS_N)
    s = rn32_sqrt(v)
    r = rn32(Fraction(1) / s)
    return [rn32(xv * r) for xv in x], v, s, r


def rmsnorm_alternatives(x, v, s):
    sq64 = rn64(Fraction(math.sqrt(float(v))))          # fp64 square root of v (correctly rounded by the host)
    r_cr = rn32(1 / Fraction(math.sqrt(float(v))))       # near-correct rsqrt, one rounding
    return {
        "RN32(x/RN32(sqrt v))": [rn32(xv / s) for xv in x],
        "RN32(x*RN64(1/sqrt64(v)))": [rn32(xv * rn64(1 / sq64)) for xv in x],
        "RN32(x*RN32(1/sqrt(v)))": [rn32(xv * r_cr) for xv in x],
    }


# ----------------------------------------------------------------------------
# Case search (selects inputs only; the expected values come from the above)
# ----------------------------------------------------------------------------

def search_quant_rows(n_rows, K, seed):
    """N(0,1) fp32 rows (the single-layer fp32 workload's distribution) that
    hold at least one element on which x*RN32(127/eta) gives another code."""
    rng = np.random.default_rng(seed)
    f32 = np.float32
    rows = []
    while len(rows) < n_rows:
        x = rng.standard_normal((4096, K)).astype(f32)
        eta = np.max(np.abs(x), axis=1)
        q1 = np.rint(((x * f32(127)).astype(f32) / eta[:, None]).astype(f32))
        s = (f32(127) / eta).astype(f32)
        q2 = np.rint((x * s[:, None]).astype(f32))
        hit = np.nonzero(np.any(q1 != q2, axis=1))[0]
        rows.extend(x[h] for h in hit[: n_rows - len(rows)])
    return rows


def search_rescale(seed, n):
    """(y_int, eta, gamma) in the decode ranges where the pages' order differs
    from every alternative at once."""
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        eta = fr(np.float32(abs(rng.standard_normal()) + 2.5))
        gamma = fr(np.float32(0.0159 * (1 + 0.1 * rng.standard_normal())))
        y_int = int(rng.integers(-20000, 20000))
        want = rescale(y_int, eta, gamma)
        alts = rescale_alternatives(y_int, eta, gamma)
        if all(a != want for a in alts.values()):
            out.append((y_int, eta, gamma))
    return out


def search_rmsnorm_rows(seed, K, n):
    rng = np.random.default_rng(seed)
    rows = []
    while len(rows) < n:
        x = [fr(v) for v in rng.standard_normal(K).astype(np.float32)]
        out, v, s, r = rmsnorm_row(x)
        alts = rmsnorm_alternatives(x, v, s)
        if all(a != out for a in alts.values()):
            rows.append(x)
    return rows


def main():
    cases = {"_about": __doc__.split("\n\n")[0] + " Generated by make_order_pins.py.",
             "quantiser": [], "rescale": [], "rmsnorm": []}

    # quantiser: the hand-worked row, then N(0,1) rows of the 256-wide layer
    hand = [Fraction(15), Fraction(15, 2)]
    rows = [hand] + [[fr(v) for v in r] for r in search_quant_rows(3, 256, 7)]
    for i, x in enumerate(rows):
        xq, eta = quant_row(x)
        alts = quant_row_alternatives(x, eta)
        diff = [k for k in range(len(x)) if alts["x*RN32(127/eta)"][k] != xq[k]]
        assert diff, "the row must separate the two orders"
        case = {"x_bits": [bits32(v) for v in x], "eta_bits": bits32(eta), "xq": xq,
                "xsum": sum(xq), "separating_index": diff,
                "alternatives": {k: [a[j] for j in diff] for k, a in alts.items()}}
        if i == 0:
            case["why"] = (
                "eta = max|x| = 15. x = 7.5: 7.5*127 = 952.5 exactly, 952.5/15 = 63.5 exactly, so "
                "RN32 leaves it and round-half-even gives 64. The other order: 127/15 = 8.4666..., "
                "RN32 = 8877943/2^20 = 8.46666622 (fp32 step 2^-20 in [8,16)); 7.5 times that is "
                "66584572.5/2^20 = 63.4999966, which RN32 (step 2^-18 in [32,64)) takes to "
                "63.5 - 2^-18 = 63.4999962, and rounding gives 63.")
        cases["quantiser"].append(case)

    # rescale: a hand-worked triple, then decode-range triples
    triples = [(3, Fraction(3), Fraction(3, 4))] + search_rescale(11, 6)
    for i, (y_int, eta, gamma) in enumerate(triples):
        want = rescale(y_int, eta, gamma)
        alts = rescale_alternatives(y_int, eta, gamma)
        assert all(a != want for a in alts.values())
        case = {"y_int": y_int, "eta_bits": bits32(eta), "gamma_bits": bits32(gamma),
                "y_bits": bits32(want),
                "alternatives_bits": {k: bits32(a) for k, a in alts.items()}}
        if i == 0:
            s = rn32(rn32(eta * gamma) / 127)
            case["why"] = (
                "eta*gamma = 3*0.75 = 2.25 exactly; 2.25/127 rounds to s = %d/2^%d; y = RN32(3*s) = "
                "%r. Every other grouping (listed) rounds at a different place and lands on another "
                "fp32 value." % (s.numerator, s.denominator.bit_length() - 1, float(want)))
        cases["rescale"].append(case)

    # RMSNorm: rows of the decode width where all three alternatives differ somewhere
    for x in search_rmsnorm_rows(13, 64, 3):
        out, v, s, r = rmsnorm_row(x)
        alts = rmsnorm_alternatives(x, v, s)
        cases["rmsnorm"].append({
            "x_bits": [bits32(t) for t in x], "v_bits": bits32(v), "sqrt_bits": bits32(s),
            "r_bits": bits32(r), "out_bits": [bits32(t) for t in out],
            "alternatives_differ_at": {k: [j for j in range(len(x)) if a[j] != out[j]]
                                       for k, a in alts.items()}})

    with open(OUT, "w") as fh:
        json.dump(cases, fh, indent=1)
        fh.write("\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()

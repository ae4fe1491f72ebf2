"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

Nothing here compares the oracle with itself: each test checks it against a
hand-worked example, a closed form, a textbook routine, brute force or an
invariant of the method.  Both oracle implementations (NumPy twin and scalar
C) are held to every pin.  The last block plants mistakes in a copy of the
oracle and checks that the pins notice.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import native, reference

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


class NativeOracle:
    """The C oracle behind the same call shapes as ``oracle.reference``."""

    @staticmethod
    def absmean_gamma(W):
        return native.absmean_gamma(W)

    @staticmethod
    def pack_weights(W):
        packed, gamma, t = native.pack_weights(W, want_ternary=True)
        return packed, gamma, t

    @staticmethod
    def quant_act(x):
        return native.quant_act(x, nthreads=1)

    @staticmethod
    def forward(xq, eta, packed, gamma, K):
        N = packed.shape[0]
        return native.forward(xq, eta, packed, gamma, K, N, nthreads=1)


ORACLES = {"numpy": reference, "c": NativeOracle}


@pytest.fixture(params=sorted(ORACLES))
def orc(request):
    return ORACLES[request.param]


def layer(orc, W, x):
    packed, gamma, t = orc.pack_weights(W)
    xq, eta, xsum = orc.quant_act(x)
    y_int, y = orc.forward(xq, eta, packed, gamma, np.asarray(W).shape[1])
    return dict(packed=packed, gamma=gamma, t=t, xq=xq, eta=eta, xsum=xsum,
                y_int=np.asarray(y_int, np.int64), y=np.asarray(y, np.float32))


# --------------------------------------------------------------------------
# Hand-worked examples (tests/golden)
# --------------------------------------------------------------------------

def test_worked_example_2x4(orc):
    g = json.load(open(os.path.join(GOLDEN, "worked_example_2x4.json")))
    W = np.array(g["W"], np.float32)
    x = np.array(g["x"], np.float32)
    r = layer(orc, W, x)
    assert float(r["gamma"]) == g["gamma"]
    np.testing.assert_array_equal(r["t"], g["ternary"])
    np.testing.assert_array_equal(r["packed"], g["packed"])
    np.testing.assert_array_equal(r["eta"], g["eta"])
    np.testing.assert_array_equal(r["xq"], g["xq"])
    np.testing.assert_array_equal(r["xsum"], g["xsum"])
    np.testing.assert_array_equal(r["y_int"], g["y_int"])
    np.testing.assert_array_equal(r["y"], np.array(g["y"], np.float32))
    np.testing.assert_array_equal(reference.f32_to_bf16_bits(r["y"]), g["y_bf16_bits"])
    np.testing.assert_array_equal(native.f32_to_bf16_bits(r["y"]), g["y_bf16_bits"])


def test_pack_codes_golden():
    g = json.load(open(os.path.join(GOLDEN, "pack_codes.json")))
    for case in g["cases"]:
        t = np.array(case["ternary"], np.int8)
        np.testing.assert_array_equal(reference.pack2(t), case["packed"], err_msg=case["why"])
        np.testing.assert_array_equal(reference.unpack2(np.array(case["packed"], np.uint8),
                                                        t.shape[1]), t)
        # the C oracle packs from latent weights: W = t gives back t (idempotence)
        if np.any(t != 0):
            packed, _, tt = native.pack_weights(t.astype(np.float32), want_ternary=True)
            np.testing.assert_array_equal(tt, t)
            np.testing.assert_array_equal(packed, case["packed"], err_msg=case["why"])


def test_unpack_rejects_code_11():
    with pytest.raises(ValueError):
        reference.unpack2(np.array([[0xFF]], np.uint8), 4)
    xq = np.ones((1, 4), np.int8)
    with pytest.raises(RuntimeError):
        native.forward(xq, np.ones(1, np.float32), np.array([[0xC0]], np.uint8), 1.0, 4, 1)


# --------------------------------------------------------------------------
# Rounding: half to even, in both quantisers (closed forms)
# --------------------------------------------------------------------------

def test_weight_ties_round_to_even(orc):
    # mean|W| = 8/4 = 2, W/gamma = [-0.5, 0.5, 1, 2] -> [0, 0, 1, 1]
    W = np.array([[-1.0, 1.0, 2.0, 4.0]], np.float32)
    packed, gamma, t = orc.pack_weights(W)
    assert float(gamma) == 2.0
    np.testing.assert_array_equal(t, [[0, 0, 1, 1]])
    # 1.5*gamma rounds to 2 and clips to 1; 2.5*gamma likewise
    W = np.array([[1.5, -1.5, 2.5, -2.5, 0.0, 0.0, 0.0, 0.0]], np.float32)  # mean = 1
    _, gamma, t = orc.pack_weights(W)
    assert float(gamma) == 1.0
    np.testing.assert_array_equal(t, [[1, -1, 1, -1, 0, 0, 0, 0]])


def test_activation_ties_round_to_even(orc):
    # eta = 127 makes x*127/eta == x exactly for these values
    x = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5]], np.float32)
    xq, eta, xsum = orc.quant_act(x)
    assert float(eta[0]) == 127.0
    np.testing.assert_array_equal(xq, [[127, 0, 2, 2, 0, -2, -2, 126]])
    assert int(xsum[0]) == 127 + 0 + 2 + 2 + 0 - 2 - 2 + 126


def test_argmax_maps_to_127(orc):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 97)) * rng.uniform(1e-3, 1e3, (64, 1))).astype(np.float32)
    xq, eta, _ = orc.quant_act(x)
    idx = np.argmax(np.abs(x), axis=1)
    np.testing.assert_array_equal(np.abs(xq[np.arange(64), idx]), 127)
    np.testing.assert_array_equal(eta, np.max(np.abs(x), axis=1))
    assert np.all(np.abs(xq.astype(np.int32)) <= 127)


def test_eta_and_gamma_floor(orc):
    x = np.zeros((2, 5), np.float32)
    x[1, 2] = 1e-7
    xq, eta, xsum = orc.quant_act(x)
    np.testing.assert_array_equal(eta, np.float32(1e-5))
    # 1e-7 * 127 / 1e-5 = 1.27 -> 1
    np.testing.assert_array_equal(xq, [[0] * 5, [0, 0, 1, 0, 0]])
    W = np.full((3, 4), 1e-7, np.float32)
    packed, gamma, t = orc.pack_weights(W)
    assert gamma == np.float32(1e-5)
    assert not np.any(t)


# --------------------------------------------------------------------------
# gamma: the exact mean of |W|
# --------------------------------------------------------------------------

def _exact_gamma(W):
    """gamma from exact rational arithmetic (Python's Fraction and its
    correctly rounded float conversion), independent of both oracles."""
    s = sum(Fraction(float(v)) for v in np.abs(W.astype(np.float64)).ravel())
    return np.float32(float(s) / W.size), float(s)


@pytest.mark.parametrize("case", ["lost_in_naive_sum", "tie_to_even", "subnormals", "mixed"])
def test_gamma_exact_sum(orc, case):
    if case == "lost_in_naive_sum":
        W = np.ones((1, 4097), np.float32)
        W[0, 0] = 2.0 ** 60  # a naive fp32 running sum drops every 1.0
    elif case == "tie_to_even":
        W = np.array([[2.0 ** 53, 2.0, 1.0]], np.float32)  # 2^53 + 3 ties -> 2^53 + 4
    elif case == "subnormals":
        W = np.array([[2.0 ** -149, -(2.0 ** -149), 3 * 2.0 ** -149, 2.0 ** -126]], np.float32)
    else:
        rng = np.random.default_rng(5)
        W = (rng.standard_normal((17, 33)) * np.exp2(rng.integers(-60, 60, (17, 33)))).astype(np.float32)
    g_exact, s_exact = _exact_gamma(W)
    gamma, s = orc.absmean_gamma(W)
    assert s == s_exact
    assert np.float32(gamma) == max(g_exact, np.float32(1e-5))
    if case == "tie_to_even":
        assert s == 2.0 ** 53 + 4


def test_gamma_is_mean_abs(orc):
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (300, 77)).astype(np.float32)
    gamma, _ = orc.absmean_gamma(W)
    m64 = np.mean(np.abs(W), dtype=np.float64)
    assert abs(float(gamma) - m64) <= float(np.spacing(np.float32(m64)))
    assert gamma == _exact_gamma(W)[0]


# --------------------------------------------------------------------------
# Accumulation: add/sub/skip identity, textbook routines, brute force
# --------------------------------------------------------------------------

def test_accumulate_matches_int64_matmul_and_fp32_linear(orc):
    import torch
    rng = np.random.default_rng(7)
    for (M, K, N) in [(1, 256, 256), (3, 65, 17), (5, 200, 33), (2, 1, 3)]:
        W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
        x = rng.normal(0, 1, (M, K)).astype(np.float32)
        r = layer(orc, W, x)
        t = reference.unpack2(r["packed"], K)
        np.testing.assert_array_equal(t, r["t"])
        ref_int = np.dot(r["xq"].astype(np.int64), t.astype(np.int64).T)  # textbook matmul
        np.testing.assert_array_equal(r["y_int"], ref_int)
        # p1's F.linear on integer-valued fp32 is exact while partial sums stay < 2^24
        lin = torch.nn.functional.linear(torch.from_numpy(r["xq"].astype(np.float32)),
                                         torch.from_numpy(t.astype(np.float32)))
        np.testing.assert_array_equal(lin.numpy().astype(np.int64), ref_int)
        # y_int = sum(x~ * (code)) - xsum, with code = t + 1
        np.testing.assert_array_equal(
            r["y_int"], np.dot(r["xq"].astype(np.int64), (t.astype(np.int64) + 1).T)
            - r["xsum"].astype(np.int64)[:, None])


XGRID = np.array([-127, -64, -1, 0, 1, 2, 63, 127], np.int8)


@pytest.mark.parametrize("N,K", [(1, 1), (1, 2), (1, 3), (1, 4), (2, 1), (2, 2), (2, 3),
                                 (3, 2), (3, 1), (1, 5), (1, 6), (6, 1)])
def test_brute_force_all_ternary_matrices(orc, N, K):
    """Every W~ in {-1,0,1}^(N x K) used as its own latent W: ternarise(W~) ==
    W~ (idempotence), and for a grid of x~ rows y_int is the plain dot
    product written as a Python loop."""
    xs = np.array(list(itertools.product(XGRID, repeat=K)), np.int8)
    if xs.shape[0] > 64:
        xs = xs[np.random.default_rng(K).choice(xs.shape[0], 64, replace=False)]
    eta = np.ones(xs.shape[0], np.float32) * 127
    for flat in itertools.product((-1, 0, 1), repeat=N * K):
        t = np.array(flat, np.int8).reshape(N, K)
        packed, gamma, tt = orc.pack_weights(t.astype(np.float32))
        np.testing.assert_array_equal(tt, t)
        nnz = int(np.count_nonzero(t))
        assert float(gamma) == (max(np.float32(nnz / (N * K)), np.float32(1e-5)))
        y_int, y = orc.forward(xs, eta, packed, gamma, K)
        for i in range(xs.shape[0]):
            for n in range(N):
                dot = 0
                for k in range(K):
                    dot += int(xs[i, k]) * int(t[n, k])
                assert int(y_int[i][n]) == dot


def test_all_zero_weights_give_zero(orc):
    rng = np.random.default_rng(1)
    W = np.zeros((9, 70), np.float32)
    x = rng.normal(0, 3, (4, 70)).astype(np.float32)
    r = layer(orc, W, x)
    assert r["gamma"] == np.float32(1e-5)
    assert not np.any(r["t"])
    assert not np.any(r["y_int"])
    assert np.all(r["y"] == 0) and not np.any(np.signbit(r["y"]))


@pytest.mark.parametrize("K", [1, 4, 7, 64, 130])
@pytest.mark.parametrize("sign", [1, -1])
def test_signed_identity_dequantises(orc, K, sign):
    """W = sign*K*I_K: gamma = K*K/(K*K) = 1 exactly, W~ = sign*I, y_int =
    sign*x~, and y is the dequantised x: within half a quantisation step
    (eta/127/2, plus a few fp32 ulps) of sign*x."""
    W = (sign * K * np.eye(K)).astype(np.float32)
    rng = np.random.default_rng(K)
    x = rng.normal(0, 1, (3, K)).astype(np.float32)
    r = layer(orc, W, x)
    assert r["gamma"] == 1.0
    np.testing.assert_array_equal(r["t"], sign * np.eye(K, dtype=np.int8))
    np.testing.assert_array_equal(r["y_int"], sign * r["xq"].astype(np.int64))
    step = r["eta"].astype(np.float64) / 127.0
    err = np.abs(r["y"].astype(np.float64) - sign * x.astype(np.float64))
    assert np.all(err <= step[:, None] * (0.5 + 1e-5))


# --------------------------------------------------------------------------
# Invariants: symmetry, scaling, Round-then-Clip == Clip-then-Round
# --------------------------------------------------------------------------

def test_symmetry_and_power_of_two_scaling(orc):
    rng = np.random.default_rng(2)
    W = rng.normal(0, 0.02, (40, 96)).astype(np.float32)
    x = rng.normal(0, 1, (3, 96)).astype(np.float32)
    base = layer(orc, W, x)
    neg_x = layer(orc, W, -x)
    np.testing.assert_array_equal(neg_x["xq"], -base["xq"])
    np.testing.assert_array_equal(neg_x["eta"], base["eta"])
    neg_w = layer(orc, -W, x)
    np.testing.assert_array_equal(neg_w["t"], -base["t"])
    assert neg_w["gamma"] == base["gamma"]
    np.testing.assert_array_equal(neg_w["y_int"], -base["y_int"])
    twice_x = layer(orc, W, 2 * x)
    np.testing.assert_array_equal(twice_x["xq"], base["xq"])
    np.testing.assert_array_equal(twice_x["eta"], 2 * base["eta"])
    np.testing.assert_array_equal(twice_x["y"], 2 * base["y"])
    twice_w = layer(orc, 2 * W, x)
    np.testing.assert_array_equal(twice_w["t"], base["t"])
    assert twice_w["gamma"] == 2 * base["gamma"]
    np.testing.assert_array_equal(twice_w["y"], 2 * base["y"])


def test_round_then_clip_equals_clip_then_round(orc):
    """[Production] '1. Absmean Weight Quantization' writes Clip(Round(.));
    [No-Multiply] 'Straight-Through Estimator Training' writes round(clip(.)).
    They agree on every input, ties included."""
    rng = np.random.default_rng(4)
    W = rng.normal(0, 0.02, (50, 64)).astype(np.float32)
    W[0, :8] = [0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 1.0, -1.0]
    packed, gamma, t = orc.pack_weights(W)
    q = W / np.float32(gamma)
    np.testing.assert_array_equal(t, np.rint(np.clip(q, -1, 1)).astype(np.int8))


# --------------------------------------------------------------------------
# Statistics: zero fraction of W~ for Gaussian and Laplace latents
# --------------------------------------------------------------------------

def test_zero_fraction_statistics():
    """For N(0, s^2) latents, gamma -> s*sqrt(2/pi) and P(|W| <= gamma/2) =
    2*Phi(sqrt(2/pi)/2) - 1 = 0.3101; for Laplace(0, b), gamma -> b and
    P(|W| <= b/2) = 1 - exp(-1/2) = 0.3935.  The pages quote ~33% zeros.
    The sign() variant ([No-Multiply] 'Weight Quantization') gives none."""
    rng = np.random.default_rng(9)
    Wn = rng.normal(0, 0.02, (512, 1024)).astype(np.float32)
    Wl = rng.laplace(0, 0.02, (512, 1024)).astype(np.float32)
    _, _, tn = native.pack_weights(Wn, want_ternary=True)
    _, _, tl = native.pack_weights(Wl, want_ternary=True)
    pn = 2 * 0.5 * (1 + math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))) - 1
    assert abs(pn - 0.3101) < 1e-4
    assert abs(np.mean(tn == 0) - pn) < 0.005
    assert abs(np.mean(tl == 0) - (1 - math.exp(-0.5))) < 0.005
    assert set(np.unique(tn).tolist()) <= {-1, 0, 1}
    sign_variant = np.clip(np.rint(np.sign(Wn / (np.mean(np.abs(Wn)) + 1e-8))), -1, 1)
    assert np.mean(sign_variant == 0) < 1e-3


# --------------------------------------------------------------------------
# The two oracle implementations agree, including ragged K
# --------------------------------------------------------------------------

@pytest.mark.parametrize("K", [1, 2, 3, 5, 63, 64, 65, 255])
def test_numpy_and_c_oracles_agree(K):
    rng = np.random.default_rng(K + 100)
    W = rng.laplace(0, 0.02, (23, K)).astype(np.float32)
    x = (rng.standard_t(3, (4, K)) * 3).astype(np.float32)
    a = layer(reference, W, x)
    b = layer(NativeOracle, W, x)
    for key in a:
        np.testing.assert_array_equal(np.asarray(a[key]), np.asarray(b[key]), err_msg=key)


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(6)
    y = (rng.standard_normal(4096) * np.exp2(rng.integers(-20, 20, 4096))).astype(np.float32)
    # exact ties at the bf16 midpoint, both parities
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40A18000], np.uint32).view(np.float32)
    y = np.concatenate([y, ties])
    want = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(reference.f32_to_bf16_bits(y), want)
    np.testing.assert_array_equal(native.f32_to_bf16_bits(y), want)


# --------------------------------------------------------------------------
# Planted mistakes: a broken copy of the oracle must fail the pins above
# --------------------------------------------------------------------------

class _Mutant:
    """reference with one step replaced."""

    def __init__(self, **overrides):
        self.__dict__.update({k: getattr(reference, k) for k in
                              ("absmean_gamma", "quant_act", "forward", "pack2", "unpack2",
                               "ternarise", "accumulate", "rescale")})
        self.__dict__.update(overrides)

    def pack_weights(self, W):
        gamma, _ = self.absmean_gamma(W)
        t = self.ternarise(W, gamma)
        return self.pack2(t), gamma, t


def _round_half_away(q):
    return np.sign(q) * np.floor(np.abs(q) + 0.5)


def test_planted_round_half_away_is_caught():
    def ternarise(W, gamma):
        return np.clip(_round_half_away(np.asarray(W, np.float32) / np.float32(gamma)), -1, 1).astype(np.int8)
    with pytest.raises(AssertionError):
        test_weight_ties_round_to_even(_Mutant(ternarise=ternarise))


def test_planted_sign_variant_is_caught():
    def ternarise(W, gamma):
        W = np.asarray(W, np.float32)
        return np.clip(np.rint(np.sign(W / np.float32(gamma))), -1, 1).astype(np.int8)
    with pytest.raises(AssertionError):
        test_worked_example_2x4(_Mutant(ternarise=ternarise))


def test_planted_swapped_codes_are_caught():
    def pack2(t):
        return reference.pack2(-np.asarray(t, np.int8))  # +1 and -1 codes swapped
    with pytest.raises(AssertionError):
        test_worked_example_2x4(_Mutant(pack2=pack2))


def test_planted_wrong_row_index_is_caught():
    """Output feature n reads weight row N-1-n (an index mistake)."""
    def forward(xq, eta, packed, gamma, K):
        t = reference.unpack2(packed, K)[::-1]
        y_int = reference.accumulate(xq, t)
        return y_int, reference.rescale(y_int, eta, gamma)
    with pytest.raises(AssertionError):
        test_worked_example_2x4(_Mutant(forward=forward))


def test_planted_transposed_codes_are_caught():
    """Bits of a byte read from the top (element j at bits 6-2j)."""
    def unpack2(packed, K):
        packed = np.asarray(packed, np.uint8)
        N, P = packed.shape
        codes = np.stack([(packed >> (6 - 2 * j)) & 3 for j in range(4)], axis=2).reshape(N, 4 * P)
        return codes[:, :K].astype(np.int8) - 1

    def forward(xq, eta, packed, gamma, K):
        t = unpack2(packed, K)
        y_int = reference.accumulate(xq, t)
        return y_int, reference.rescale(y_int, eta, gamma)
    with pytest.raises(AssertionError):
        test_worked_example_2x4(_Mutant(forward=forward))


def test_planted_dropped_clamp_is_caught():
    def absmean_gamma(W):
        W = np.asarray(W, np.float32)
        s = math.fsum(np.abs(W.astype(np.float64)).ravel().tolist())
        return np.float32(s / W.size), s  # no 1e-5 floor
    with pytest.raises((AssertionError, FloatingPointError, ValueError)):
        with np.errstate(divide="raise", invalid="raise"):
            test_all_zero_weights_give_zero(_Mutant(absmean_gamma=absmean_gamma))


def test_planted_wrong_rescale_is_caught():
    def rescale(y_int, eta, gamma):
        eta = np.asarray(eta, np.float32)
        return np.asarray(y_int).astype(np.float32) * (eta * np.float32(gamma) / np.float32(128))[:, None]
    m = _Mutant(rescale=rescale)

    def forward(xq, eta, packed, gamma, K):
        t = reference.unpack2(packed, K)
        y_int = reference.accumulate(xq, t)
        return y_int, rescale(y_int, eta, gamma)
    m.forward = forward
    with pytest.raises(AssertionError):
        test_worked_example_2x4(m)

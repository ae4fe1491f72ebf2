"""Pins of the oracle's base-3 packing (compact ternary packing, five trits
per byte) against facts other than its own formula: a hand-worked example,
the bijection between the 243 five-trit tuples and the byte values 0..242,
agreement with the pinned 2-bit path, and the stride arithmetic."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import reference as ref

HERE = os.path.dirname(os.path.abspath(__file__))


def test_hand_worked_example():
    g = json.load(open(os.path.join(HERE, "golden", "base3_example.json")))
    t = np.array(g["t"], np.int8)
    p = ref.pack3(t)
    np.testing.assert_array_equal(p, np.array(g["packed3"], np.uint8))
    np.testing.assert_array_equal(ref.unpack3(p, g["K"]), t)


def test_all_243_tuples_are_a_bijection_onto_0_to_242():
    tuples = np.array(list(itertools.product([-1, 0, 1], repeat=5)), np.int8)  # 243 x 5
    p = ref.pack3(tuples)[:, 0]
    assert sorted(p.tolist()) == list(range(243))
    np.testing.assert_array_equal(ref.unpack3(ref.pack3(tuples), 5), tuples)


def test_first_trit_is_least_significant():
    t = np.zeros((5, 5), np.int8)
    for j in range(5):
        t[j, j] = 1                      # digit 2 at position j, digit 1 elsewhere
    got = ref.pack3(t)[:, 0].astype(int)
    assert got.tolist() == [121 + 3 ** j for j in range(5)]


@pytest.mark.parametrize("N,K", [(3, 1), (5, 7), (17, 64), (9, 3200), (4, 8192), (2, 28672)])
def test_same_trits_as_the_two_bit_path(N, K):
    rng = np.random.default_rng(N * 1000 + K)
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    packed2, gamma, t = ref.pack_weights(W)
    p3 = ref.pack3(t)
    assert p3.shape == (N, ref.packed3_stride(K))
    np.testing.assert_array_equal(ref.unpack3(p3, K), ref.unpack2(packed2, K))
    assert p3.max() <= 242


def test_forward3_equals_forward_on_the_same_trits():
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, (33, 640)).astype(np.float32)
    x = rng.normal(0, 1, (3, 640)).astype(np.float32)
    packed2, gamma, t = ref.pack_weights(W)
    xq, eta, _ = ref.quant_act(x)
    yi2, y2 = ref.forward(xq, eta, packed2, gamma, 640)
    yi3, y3 = ref.forward3(xq, eta, ref.pack3(t), gamma, 640)
    np.testing.assert_array_equal(yi3, yi2)
    np.testing.assert_array_equal(y3.view(np.uint32), y2.view(np.uint32))


def test_stride_and_bytes_per_weight():
    assert [ref.packed3_stride(K) for K in (1, 5, 80, 81, 3200, 8192, 28672)] == \
        [16, 16, 16, 32, 640, 1648, 5744]
    # 20 % fewer bytes than 2 bits per weight once K is large
    assert ref.packed3_stride(3200) / ((3200 + 3) // 4) == 0.8


def test_planted_mistakes_fail():
    tuples = np.array(list(itertools.product([-1, 0, 1], repeat=5)), np.int8)
    # most-significant-first digit order, or codes t instead of t+1, break the pins
    msb = (tuples.astype(np.int64) + 1) @ np.array([81, 27, 9, 3, 1])
    assert not np.array_equal(msb.astype(np.uint8), ref.pack3(tuples)[:, 0])
    no_offset = (tuples.astype(np.int64) % 3) @ ref.POW3
    assert not np.array_equal(no_offset.astype(np.uint8), ref.pack3(tuples)[:, 0])

"""The RMSNorm kernel's exact sum of squares, rounded once to fp64, checked
on the host against Python's correctly rounded integer division.

The kernel sums x^2 = m^2 * 2^(2e-268) of bf16 values exactly: a 128-bit
window near the row's largest exponent plus 64-bit buckets below it, then
rounds the total once (nearest even).  Its rounding routines are host
callable; this test compiles them into a small host program with nvcc (no
GPU needed) and compares bit patterns on random sums, exact ties and the
whole exponent range.
"""
import os
import random
import shutil
import struct
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "ternary_weight_linear_04_b200", "csrc")


@pytest.fixture(scope="module")
def driver():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tempfile.mkdtemp(prefix="sumsq_")
    exe = os.path.join(d, "host_sumsq")
    subprocess.run([nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", CSRC, "-o", exe, os.path.join(HERE, "host_sumsq.cu")],
                   check=True, capture_output=True)
    yield exe
    shutil.rmtree(d, ignore_errors=True)


def _f64_bits(v):
    return struct.unpack("<Q", struct.pack("<d", v))[0]


def _cases(seed, n):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        wb = rng.randint(1, 254)
        kind = i % 6
        if kind == 0:
            win = rng.getrandbits(rng.randint(1, 120))
        elif kind == 1:    # a 53-bit value followed by exactly half an ulp: a tie
            sh = rng.randint(1, 60)
            win = ((rng.getrandbits(52) | (1 << 52)) << sh) | (1 << (sh - 1))
        elif kind == 2:    # just above and below a tie
            sh = rng.randint(2, 60)
            base = (rng.getrandbits(52) | (1 << 52)) << sh
            win = base + (1 << (sh - 1)) + rng.choice((-1, 1))
        elif kind == 3:
            win = 1 << rng.randint(0, 119)
        elif kind == 4:
            win = 0
        else:              # the largest window total the kernel can form
            win = (1 << 120) - 1 - rng.getrandbits(30)
        ents = []
        if wb > 1 and (i % 3 or win == 0):
            for _ in range(rng.randint(1, 5)):
                ents.append((rng.randint(1, wb - 1), rng.randint(1, (1 << 48) - 1)))
        if wb > 1 and kind == 1 and i % 3:  # a tie created across window and buckets
            ents = [(wb - 1, 1 << 47)]
        out.append((win, wb, ents))
    return out


@pytest.mark.parametrize("seed", [1, 2])
def test_sum_of_squares_rounds_like_exact_arithmetic(driver, seed):
    cases = _cases(seed, 6000)
    lines = "".join("%d %d %d %d %s\n" % (w >> 64, w & ((1 << 64) - 1), wb, len(e),
                                          " ".join("%d %d" % be for be in e))
                    for w, wb, e in cases)
    p = subprocess.run([driver], input=lines, capture_output=True, text=True, check=True)
    got = p.stdout.split("\n")
    assert len(got) >= len(cases)
    for (w, wb, e), line in zip(cases, got):
        num = (w << (2 * wb - 2)) + sum(v << (2 * b - 2) for b, v in e)
        want = _f64_bits(num / (1 << 266))  # correctly rounded, ties to even
        s, u = (int(t, 16) for t in line.split())
        assert s == want, (w, wb, e)
        if not e:
            assert u == want, (w, wb)


def test_planted_rounding_mistake_is_caught():
    """Truncation in place of round-to-nearest-even differs on these cases,
    so the comparison above can tell the two apart."""
    differs = 0
    for w, wb, e in _cases(3, 600):
        num = (w << (2 * wb - 2)) + sum(v << (2 * b - 2) for b, v in e)
        if num == 0:
            continue
        exact = num / (1 << 266)
        top = num.bit_length()
        trunc = (num >> max(0, top - 53)) << max(0, top - 53)
        differs += (trunc / (1 << 266)) != exact
    assert differs > 100

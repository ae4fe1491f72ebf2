"""Exhaustive host checks of the division-free rules and bit-level helpers the kernels use.

* The bf16 quantiser (quant.cuh, code_bits_bf16_r): x~ = RNE(RN32(RN32(x*127)
  /eta)) of [Production] "2. Absmax Dynamic Activation Quantization", formed
  from an approximate reciprocal and an exact fma residual.  Checked for
  every bf16 x with |x| <= eta, for every bf16 significand of eta at five
  exponents, with the reciprocal perturbed by up to 8 ulps either way.
* The same rule with its tie test voted over 4 or 8 values
  (code_bits_bf16_n, what the quantiser kernels run) against the rule value
  by value.
* The pack's and the RMSNorm kernel's fp64 widening of |W| and |x| from
  bit patterns (pack.cuh), and the ternary threshold that replaces the
  division W / gamma ([Production] "1. Absmean Weight Quantization").
* The rescale's division by 127 (common.cuh, div127_rn): s = RN32(RN32(eta *
  gamma) / 127) of [Production] pipeline step 5, by a correctly rounded
  reciprocal and one fma correction.  Checked against the IEEE quotient for
  every normal fp32 a >= 2^-119.

All these routines are __host__ __device__; this test compiles them for the host
with nvcc (no GPU needed; contraction off, as in the kernels).
"""
import os
import re
import shutil
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
    d = tempfile.mkdtemp(prefix="rules_")
    exe = os.path.join(d, "host_rules")
    subprocess.run([nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-Xcompiler", "-ffp-contract=off,-fopenmp", "-I", CSRC, "-o", exe,
                    os.path.join(HERE, "host_rules.cu"), "-lgomp"],
                   check=True, capture_output=True)
    yield exe
    shutil.rmtree(d, ignore_errors=True)


def _counts(out):
    return {k: int(v) for k, v in re.findall(r"(\w+)=(\d+)", out)}


def test_bf16_quantiser_rule_is_exact(driver):
    c = _counts(subprocess.run([driver, "quant"], check=True, capture_output=True, text=True).stdout)
    assert c["checked"] > 100_000_000
    assert c["mismatches"] == 0
    assert c["ties"] > 100  # exact .5 ties occur, so the tie branch is exercised


def test_voted_tie_rule_matches_the_rule_value_by_value(driver):
    """code_bits_bf16_n, the form the quantiser kernels run (the tie test
    voted over groups of 4 or 8 values), gives the same bits as
    code_bits_bf16_r for every value, in groups with and without ties."""
    c = _counts(subprocess.run([driver, "vote"], check=True, capture_output=True, text=True).stdout)
    assert c["checked"] > 10_000_000
    assert c["mismatches"] == 0
    assert c["tie_groups"] > 1000


def test_fp64_widening_of_every_fp32_and_bf16_magnitude(driver):
    """widen_f32_mag / widen_bf16_mag (the fp64 sums of the pack and the
    streamed RMSNorm kernel): exact for every normal magnitude, and in
    [2^-127, 2^-126) for exponent field 0, as the sums' error bounds
    assume."""
    c = _counts(subprocess.run([driver, "widen"], check=True, capture_output=True, text=True).stdout)
    assert c["checked"] == 2 ** 31 + 2 ** 16
    assert c["mismatches"] == 0
    assert c["zero_field"] == 2 ** 23


def test_ternary_threshold_matches_ieee_division(driver):
    """ternary_code(w, ternary_threshold(gamma)), the pack kernels' test,
    against Clip(RNE(RN32(w / gamma)), -1, 1) near every boundary."""
    c = _counts(subprocess.run([driver, "thresh"], check=True, capture_output=True, text=True).stdout)
    assert c["checked"] > 3_000_000
    assert c["mismatches"] == 0
    assert 0 < c["nonzero"] < c["checked"]


def test_division_by_127_is_correctly_rounded(driver):
    c = _counts(subprocess.run([driver, "div127"], check=True, capture_output=True, text=True).stdout)
    assert c["checked"] > 2_000_000_000
    assert c["mismatches"] == 0
    assert c["inv127_nearest"] == 1

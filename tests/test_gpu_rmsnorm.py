"""Fused RMSNorm + quantiser (CUDA) vs. the oracle, element by element.

[Production] "2. Absmax Dynamic Activation Quantization": activations are
RMS-normalised (no affine parameters, eps 1e-6) before the absmax quantiser.
"""
import numpy as np
import pytest
import torch

from oracle import native as orc
from oracle import reference as ref
from ternary_weight_linear_04_b200 import bitlinear as bl
from ternary_weight_linear_04_b200 import build as libbuild
from ternary_weight_linear_04_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert bl.device_error() == 0


def check_rows(xt):
    """xt: bf16 CUDA tensor (any strides the binding accepts)."""
    x32 = xt.float().cpu().numpy()
    want_q, want_eta, want_sum = ref.rmsnorm_quant_act(x32)
    xq, eta, xsum = bl.rmsnorm_quant_act(xt)
    np.testing.assert_array_equal(eta.cpu().numpy().view(np.uint32), want_eta.view(np.uint32))
    np.testing.assert_array_equal(xq.cpu().numpy(), want_q)
    np.testing.assert_array_equal(xsum.cpu().numpy(), want_sum)
    return xq, eta, xsum


@pytest.mark.parametrize("dist", ["normal", "student_t_outliers"])
@pytest.mark.parametrize("K", [1, 2, 7, 8, 64, 100, 1001, 2048, 3200, 8640])
def test_rmsnorm_quant_matches_oracle(K, dist):
    rng = np.random.default_rng(100 + K)
    x = inputs.draw_activations(rng, 9, K, dist, "bf16")
    check_rows(torch.from_numpy(x).cuda().to(torch.bfloat16))


def test_rmsnorm_quant_special_rows():
    """Zeros, constants, one-hot rows, rows whose squares leave the fp32 range
    (above 2^128 and below 2^-149) and subnormal bf16 values."""
    K = 520
    rows = [np.zeros(K), np.full(K, 3.0), np.full(K, -0.125)]
    one = np.zeros(K); one[17] = 5.0; rows.append(one)
    big = np.ones(K); big[3] = 2.0e19; rows.append(big)             # x^2 > fp32 max, mean finite
    huge = np.full(K, 3.0e30); rows.append(huge)                     # mean overflows fp32: r = 0
    tiny = np.full(K, 1.0e-30); tiny[::7] = -2.0e-38; rows.append(tiny)
    sub = np.full(K, 9.2e-41); sub[5] = 1.0; rows.append(sub)        # bf16 subnormals
    mix = np.random.default_rng(1).normal(size=K); mix[::13] *= 1.0e-25; rows.append(mix)
    x = inputs.to_bf16_values(np.stack(rows).astype(np.float32))
    check_rows(torch.from_numpy(x).cuda().to(torch.bfloat16))


def test_rmsnorm_quant_scalar_path_and_offsets():
    """K that breaks the 8-wide vector loads, and a base pointer one element
    off 16-byte alignment, take the scalar loop."""
    rng = np.random.default_rng(5)
    for K in (13, 129, 1000):
        x = inputs.draw_activations(rng, 4, K, "student_t_outliers", "bf16")
        check_rows(torch.from_numpy(x).cuda().to(torch.bfloat16))
    big = torch.from_numpy(inputs.draw_activations(rng, 4, 257, "normal", "bf16")).cuda().to(torch.bfloat16)
    check_rows(big.reshape(-1)[1:1 + 4 * 256].reshape(4, 256))


def test_rmsnorm_quant_many_rows_grid_stride():
    """More rows than the launch's CTAs: each CTA loops over rows."""
    rng = np.random.default_rng(6)
    x = inputs.draw_activations(rng, 1300 * 1, 64, "normal", "bf16")
    check_rows(torch.from_numpy(x).cuda().to(torch.bfloat16))


@pytest.mark.parametrize("K", [8, 64, 3200, 8640])
def test_rmsnorm_quant_mean_square_on_a_rounding_midpoint(K):
    """Rows whose mean(x^2) is exactly the midpoint of two consecutive fp32
    values, or 2^-50 (relative) above it: K/8 values 2^k, K/8 values
    2^(k-12), optionally K/8 values 2^(k-25), the rest zero, shuffled, random
    signs, so mean(x^2) = 4^k (1 + 2^-24 (+ 2^-50)) / 8.  The kernel's fp64
    sum cannot decide these: ms must come out as the tie to even, or rounded
    up."""
    rng = np.random.default_rng(K)
    rows = []
    for k in (-20, -3, 0, 1, 2, 5, 7, 12, 30):  # most of these scales turn a wrong ms into a wrong eta
        for extra in (False, True):
            n = K // 8
            row = np.zeros(K, np.float32)
            row[:n] = 2.0 ** k
            row[n:2 * n] = 2.0 ** (k - 12)
            if extra:
                row[2 * n:3 * n] = 2.0 ** (k - 25)
            rows.append(rng.permutation(row) * rng.choice([-1.0, 1.0], K).astype(np.float32))
    check_rows(torch.from_numpy(np.stack(rows).astype(np.float32)).cuda().to(torch.bfloat16))


def test_rmsnorm_quant_rows_reuse_every_buffer():
    """Far more rows than resident CTAs: every CTA streams several rows
    through each of its row buffers."""
    rng = np.random.default_rng(8)
    x = inputs.draw_activations(rng, 5000, 64, "student_t_outliers", "bf16")
    check_rows(torch.from_numpy(x).cuda().to(torch.bfloat16))


def test_rmsnorm_quant_empty_and_dtype():
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    xq, eta, xsum = bl.rmsnorm_quant_act(e)
    assert xq.shape == (0, 64) and eta.numel() == 0 and xsum.numel() == 0
    with pytest.raises(ValueError):
        bl.rmsnorm_quant_act(torch.zeros((2, 64), device="cuda"))


@pytest.mark.parametrize("idx", [0, 1])
def test_rmsnorm_then_layer_decode_3b(idx):
    """Normalised codes through the accumulate path, at the decode_3b shapes
    (all 64 rows): y_int and y bit-exact against the oracle's layer."""
    w = inputs.WORKLOADS["decode_3b"]
    W, x = inputs.make_matrix_inputs(w, idx)
    N, K = W.shape
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    packed, gamma = bl.pack_weights(torch.from_numpy(W).cuda())
    xq, eta, xsum = check_rows(torch.from_numpy(x).cuda().to(torch.bfloat16))
    want_q, want_eta, _ = ref.rmsnorm_quant_act(x)
    ref_yint, ref_y = orc.forward(want_q, want_eta, ref_packed, ref_gamma, K, N)
    for M in (1, 4, 64):
        y, y_int = bl.forward(xq[:M], eta[:M], xsum[:M], packed, gamma, N,
                              out_dtype=torch.float32, want_int=True)
        np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint[:M])
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), ref_y[:M].view(np.uint32))


def test_bitlinear_module_with_rmsnorm():
    """BitLinear(rmsnorm=True): norm, quantise, accumulate, rescale, against
    the oracle's chain on the same inputs (fp32 and bf16 outputs)."""
    N, K = 200, 512
    W, x = inputs.make_case(4600, 3, K, N, act_dtype="bf16")
    layer = bl.BitLinear.from_latent(torch.from_numpy(W).cuda(), rmsnorm=True)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    want_q, want_eta, _ = ref.rmsnorm_quant_act(x)
    _, ref_y = orc.forward(want_q, want_eta, ref_packed, ref_gamma, K, N)
    y = layer(xd, out_dtype=torch.float32)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))
    yb = layer(xd)
    np.testing.assert_array_equal(yb.cpu().view(torch.int16).numpy().view(np.uint16),
                                  orc.f32_to_bf16_bits(ref_y))

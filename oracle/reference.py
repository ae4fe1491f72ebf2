"""NumPy oracle: the BitLinear forward written out from its definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Every floating-point step is one IEEE fp32 operation (NumPy float32 scalars
and arrays do not promote), in the order the pages write it; the gamma sum is
exact (``math.fsum`` returns the correctly rounded sum of its fp64 inputs, and
|W| widened from fp32 to fp64 is exact).  Suitable for small shapes only.

Citations (page title tags as in ``bitlinear_oracle.c``):
  absmean gamma, ternarise  -- [Production] "1. Absmean Weight Quantization",
                               WeightQuantizerSTE.forward
  absmax int8 quantisation  -- [Production] "2. Absmax Dynamic Activation
                               Quantization", ActivationQuantizerSTE.forward
  add / subtract / skip     -- [Production] "The MatMul-Free Breakthrough";
                               [Additive] "3. Additive Integer Accumulation"
  2-bit codes and bit order -- [Production] "Production Deployment Standards"
                               guideline 1; [No-Multiply] "Kernel
                               Implementation: The Lookup Table Approach"
  RMSNorm before the quant  -- [Production] "2. Absmax Dynamic Activation
                               Quantization" (normalised first, no affine),
                               BitLinear158.forward (rsqrt(mean(x^2) + 1e-6))
  base-3 packing            -- [Additive] "Energy, Memory Bandwidth, and
                               Serving Economics" (compact ternary packing,
                               named only: the layout is this library's
                               reading, see pack3)
  rescale                   -- [Production] pipeline figure step 5,
                               BitLinear158.forward
"""
import math

import numpy as np

GAMMA_MIN = np.float32(1e-5)
ETA_MIN = np.float32(1e-5)
QB = np.float32(127.0)


def absmean_gamma(W):
    """gamma = max(RN32(RN64(sum |W|) / (n*m)), 1e-5).

    The exact sum is rounded once to fp64 (``math.fsum``), divided by the
    element count in fp64 and rounded once to fp32, then clamped below at
    1e-5 as WeightQuantizerSTE does.  Returns (gamma as np.float32, the fp64
    sum)."""
    W = np.asarray(W, dtype=np.float32)
    if W.size == 0:
        raise ValueError("empty weight matrix")
    s = math.fsum(np.abs(W.astype(np.float64)).ravel().tolist())
    g = np.float32(s / float(W.size))
    return max(g, GAMMA_MIN), s


def ternarise(W, gamma):
    """W~ = Clip(Round(RN32(W / gamma)), -1, 1) with Round = half to even."""
    W = np.asarray(W, dtype=np.float32)
    q = W / np.float32(gamma)          # fp32 IEEE division
    t = np.clip(np.rint(q), -1.0, 1.0)  # np.rint rounds half to even
    return t.astype(np.int8)


def pack2(t):
    """2-bit codes code = t + 1 (00=-1, 01=0, 10=+1), four per byte along K,
    element j of a byte in bits 2j..2j+1; tail codes 01.  Returns N x ceil(K/4)
    uint8."""
    t = np.asarray(t, dtype=np.int8)
    N, K = t.shape
    P = (K + 3) // 4
    codes = np.ones((N, 4 * P), dtype=np.uint8)
    codes[:, :K] = (t + 1).astype(np.uint8)
    codes = codes.reshape(N, P, 4)
    packed = (codes[:, :, 0]
              | (codes[:, :, 1] << 2)
              | (codes[:, :, 2] << 4)
              | (codes[:, :, 3] << 6))
    return packed.astype(np.uint8)


def unpack2(packed, K):
    """Inverse of pack2: codes read as bits 2j..2j+1 of byte k>>2; code 11 is
    rejected (packing never writes it)."""
    packed = np.asarray(packed, dtype=np.uint8)
    N, P = packed.shape
    if P != (K + 3) // 4:
        raise ValueError("packed width does not match K")
    codes = np.stack([(packed >> (2 * j)) & 3 for j in range(4)], axis=2).reshape(N, 4 * P)
    if np.any(codes == 3):
        raise ValueError("invalid 2-bit code 11 in packed weights")
    return (codes[:, :K].astype(np.int8) - 1)


def packed3_stride(K):
    """Row stride of the base-3 layout: ceil(K/5) bytes rounded up to a
    multiple of 16 (this library's reading; the pages give no layout)."""
    return 16 * ((((K + 4) // 5) + 15) // 16)


POW3 = np.array([1, 3, 9, 27, 81], dtype=np.int64)


def pack3(t):
    """Base-3 "compact ternary packing" ([Additive] "Energy, Memory Bandwidth,
    and Serving Economics"; 3^5 = 243 <= 256): byte g of a row holds the trits
    5g .. 5g+4 as sum_j (t + 1) * 3^j.  Trits past K are 0; the row is padded
    to packed3_stride(K) with bytes of five zero trits (value 121).
    Returns N x packed3_stride(K) uint8."""
    t = np.asarray(t, dtype=np.int8)
    N, K = t.shape
    S = packed3_stride(K)
    digits = np.ones((N, 5 * S), dtype=np.int64)   # digit = t + 1; padding digit 1 (t = 0)
    digits[:, :K] = t.astype(np.int64) + 1
    return (digits.reshape(N, S, 5) * POW3).sum(axis=2).astype(np.uint8)


def unpack3(packed3, K):
    """Inverse of pack3: the base-3 digits of each byte, least significant
    first, minus one; byte values above 242 are rejected."""
    b = np.asarray(packed3, dtype=np.uint8).astype(np.int64)
    N, S = b.shape
    if S != packed3_stride(K):
        raise ValueError("packed3 width does not match K")
    if np.any(b > 242):
        raise ValueError("byte above 242 in base-3 packed weights")
    digits = np.stack([(b // int(p)) % 3 for p in POW3], axis=2).reshape(N, 5 * S)
    return (digits[:, :K] - 1).astype(np.int8)


def forward3(xq, eta, packed3, gamma, K):
    """The layer on base-3 packed weights: the same trits, so the same
    (y_int, y) as forward() on the 2-bit packing of them."""
    t = unpack3(packed3, K)
    y_int = accumulate(xq, t)
    return y_int, rescale(y_int, eta, gamma)


RMS_EPS = np.float32(1e-6)


def rmsnorm(x):
    """RMSNorm without affine parameters, before the quantiser ([Production]
    "2. Absmax Dynamic Activation Quantization" and BitLinear158.forward:
    norm = rsqrt(mean(x^2) + 1e-6), x_norm = x * norm), per token.
    Readings: mean(x^2) = RN32(RN64(exact sum of x^2) / K) with the
    division in fp64 (the sum order is unspecified on the pages; the exact
    sum makes it order-free, as for gamma); rsqrt(v) = RN32(1 / RN32(sqrt(v)))
    (an IEEE fp32 square root, then an IEEE fp32 division); every other step
    one fp32 rounding."""
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    out = np.empty_like(x)
    for m in range(M):
        S = math.fsum(float(v) * float(v) for v in x[m])   # squares exact in fp64; fsum = RN64 of the exact sum
        ms = np.float32(S / K)                               # fp64 division, then RN32
        v = np.float32(ms + RMS_EPS)
        s = np.sqrt(v, dtype=np.float32)                     # IEEE fp32 square root
        r = np.float32(1.0) / s                              # IEEE fp32 division
        out[m] = x[m] * r
    return out


def rmsnorm_quant_act(x):
    """RMSNorm then the per-token absmax int8 quantiser: (x~, eta, xsum)."""
    return quant_act(rmsnorm(x))


def pack_weights(W):
    """Load-time half of the layer: (packed bytes, gamma, ternary matrix)."""
    gamma, _ = absmean_gamma(W)
    t = ternarise(W, gamma)
    return pack2(t), gamma, t


def quant_act(x):
    """Per-token absmax int8 quantisation.

    eta_m = max(max_k |x|, 1e-5); x~ = Clip(Round(RN32(RN32(x*127)/eta_m)),
    -127, 127); also returns xsum_m = sum_k x~ (int64)."""
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("x must be M x K")
    eta = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    eta = np.maximum(eta.astype(np.float32), ETA_MIN)
    scaled = x * QB                      # RN32
    q = scaled / eta[:, None]            # RN32
    xq = np.clip(np.rint(q), -127, 127).astype(np.int8)
    return xq, eta, xq.astype(np.int64).sum(axis=1)


def accumulate(xq, t):
    """y_int[m, n] = sum_{k: t[n,k]=+1} x~[m,k] - sum_{k: t[n,k]=-1} x~[m,k]."""
    xq = np.asarray(xq, dtype=np.int64)
    plus = (np.asarray(t) == 1).astype(np.int64)
    minus = (np.asarray(t) == -1).astype(np.int64)
    return xq @ plus.T - xq @ minus.T


def rescale(y_int, eta, gamma):
    """s_m = RN32(RN32(eta_m * gamma) / 127); y = RN32(float32(y_int) * s_m)."""
    eta = np.asarray(eta, dtype=np.float32)
    s = (eta * np.float32(gamma)) / QB
    return np.asarray(y_int).astype(np.float32) * s[:, None]


def f32_to_bf16_bits(y):
    """Round fp32 to bf16, nearest-even, on the bit pattern; returns uint16."""
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + up.astype(np.uint64)).astype(np.uint16)


def forward(xq, eta, packed, gamma, K):
    """Integer accumulation from the packed bytes, then the rescale.
    Returns (y_int int64, y float32)."""
    t = unpack2(packed, K)
    y_int = accumulate(xq, t)
    return y_int, rescale(y_int, eta, gamma)


def bitlinear(W, x):
    """The whole layer on fp32 inputs: returns a dict of every intermediate."""
    packed, gamma, t = pack_weights(W)
    xq, eta, xsum = quant_act(x)
    y_int, y = forward(xq, eta, packed, gamma, np.asarray(W).shape[1])
    return dict(packed=packed, gamma=gamma, t=t, xq=xq, eta=eta, xsum=xsum,
                y_int=y_int, y=y)

"""The decode kernel's launch-shape model is host logic: checked here on the
CPU (no GPU) through bitlinear_decode_shape_for with B200's 148 SMs.

Invariants every shape must keep (the kernel relies on them), and the
shapes the model picks for the decode_3b matrices, which a forced-shape
sweep on the GPU measured as the fastest.
"""
import ctypes

import pytest

from ternary_weight_linear_04_b200 import _lib
from ternary_weight_linear_04_b200 import build as libbuild

FIELDS = ("G", "RB", "teams", "nwj", "rpc", "grid", "bpc", "stages", "x_staged", "smem")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.lib()


def shape(L, M, K, N, fused=1, sms=148):
    buf = (ctypes.c_int32 * 10)()
    st = L.bitlinear_decode_shape_for(M, K, N, fused, sms, buf)
    return st, dict(zip(FIELDS, list(buf)))


SHAPES = [(M, K, N) for M in (1, 2, 3, 4)
          for K, N in ((64, 5), (256, 256), (3200, 8640), (8640, 3200), (8192, 8192), (8192, 1024),
                       (8192, 28672), (28672, 8192), (4096, 11008), (16384, 77))]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_shape_invariants(L, M, K, N):
    mt = 1 if M == 1 else (2 if M == 2 else 4)
    st, g = shape(L, M, K, N)
    if K * mt > 131072:
        assert st == _lib.BL_ERR_UNSUPPORTED
        return
    assert st == _lib.BL_OK, st
    assert 1 <= g["G"] <= 16 and g["teams"] == 16 // g["G"]
    assert g["RB"] in (1, 2, 4, 8, 16) and g["RB"] * mt <= 16
    assert 32 * g["G"] * g["nwj"] >= K // 16                  # every packed word has a lane
    assert g["rpc"] * g["grid"] >= N and (g["grid"] - 1) * g["rpc"] < N
    assert g["grid"] <= max(148, N)
    blocks = -(-g["rpc"] // g["RB"])
    if g["G"] > 1:
        assert blocks <= 64                                   # reduction slots per CTA
    assert 1 <= g["bpc"] <= blocks and 1 <= g["stages"] <= 8
    assert g["smem"] <= 227 * 1024
    # shared memory = x~ slots + staged activations + ring + tail, all accounted for
    slots = mt * 32 * g["G"] * g["nwj"] * 16
    ring = g["stages"] * g["bpc"] * g["RB"] * (K // 4)
    assert g["smem"] >= slots + ring
    if g["x_staged"]:
        assert g["smem"] >= slots + ring + M * K * 2


def test_decode_3b_shapes_are_the_measured_best(L):
    """A forced-shape sweep on B200 measured G=1, RB=4 (K=3200) and G=1,
    RB=2 (K=8640) as the fastest for one token; the model picks them."""
    _, a = shape(L, 1, 3200, 8640)
    _, b = shape(L, 1, 8640, 3200)
    assert (a["G"], a["RB"]) == (1, 4) and (b["G"], b["RB"]) == (1, 2)
    # and the whole share of a CTA fits the ring: the weights are prefetched
    assert a["bpc"] * a["stages"] * a["RB"] >= a["rpc"]
    assert b["bpc"] * b["stages"] * b["RB"] >= b["rpc"]


def test_fewer_sms_more_rows_per_cta(L):
    _, a = shape(L, 1, 3200, 8640, sms=148)
    _, b = shape(L, 1, 3200, 8640, sms=74)
    assert b["rpc"] > a["rpc"] and b["grid"] <= 74


def test_bad_arguments(L):
    assert shape(L, 1, 3200, 8640, sms=0)[0] == _lib.BL_ERR_INVALID_ARG
    assert shape(L, 1, 3200, 0)[0] == _lib.BL_ERR_INVALID_ARG
    assert shape(L, 5, 3200, 8640)[0] == _lib.BL_ERR_UNSUPPORTED
    buf = (ctypes.c_int32 * 10)()
    assert L.bitlinear_decode_shape_for(1, 3200, 8640, 1, 148, None) == _lib.BL_ERR_INVALID_ARG


def test_register_kernel_shape_picks():
    """The one-token register-resident kernel: decode_3b's matrices take it
    (K=3200 -> N=8640: 4 rows per warp, 7 words per lane, 59 rows per CTA;
    K=8640 -> N=3200: 2 rows per warp, 17 words per lane, 22 rows per CTA),
    and shapes beyond its register budget or 64 rows per CTA do not."""
    L = _lib.lib()

    def reg(K, N, sms=148):
        buf = (ctypes.c_int32 * 4)()
        st = L.bitlinear_decode_reg_shape(K, N, sms, buf)
        return None if st == _lib.BL_ERR_UNSUPPORTED else (st, list(buf))

    assert reg(3200, 8640) == (_lib.BL_OK, [4, 7, 59, 147])
    assert reg(8640, 3200) == (_lib.BL_OK, [2, 17, 22, 146])
    assert reg(8192, 1024) == (_lib.BL_OK, [1, 16, 7, 147])
    assert reg(8192, 28672) is None        # 194 rows per CTA
    assert reg(28672, 8192) is None        # 56 rows per CTA: 4 rows per warp, more than 8 words per lane
    assert reg(3232, 100) is None          # K not a multiple of 64
    for K in range(64, 16384 + 1, 64):
        for N in (1, 148, 2368, 2369, 4736, 9472, 9473):
            r = reg(K, N)
            if r is None:
                continue
            rb, nj, rpc, grid = r[1]
            assert rb in (1, 2, 4) and rpc <= 16 * rb and rb * nj <= 34
            assert 512 * nj >= K and rpc * grid >= N and (grid - 1) * rpc < N


def test_multi_token_register_kernel_shape_picks():
    """The register-resident kernel for 2..8 tokens (x~ given): the rows of
    the one-token geometry, 2, 4 or 8 token slots, RB * MT <= 32, and the
    smallest instantiated word count that covers K."""
    L = _lib.lib()

    def regm(M, K, N, sms=148):
        buf = (ctypes.c_int32 * 5)()
        st = L.bitlinear_decode_regm_shape(M, K, N, sms, buf)
        return None if st == _lib.BL_ERR_UNSUPPORTED else (st, list(buf))

    assert regm(4, 3200, 8640) == (_lib.BL_OK, [4, 4, 7, 59, 147])
    assert regm(3, 8640, 3200) == (_lib.BL_OK, [4, 2, 17, 22, 146])
    assert regm(2, 3200, 8640) == (_lib.BL_OK, [2, 4, 7, 59, 147])
    assert regm(2, 8192, 1024) == (_lib.BL_OK, [2, 1, 17, 7, 147])
    assert regm(1, 3200, 8640) is None     # one token: the fused kernel
    assert regm(5, 3200, 8640) == (_lib.BL_OK, [8, 4, 7, 59, 147])
    assert regm(8, 8640, 3200) == (_lib.BL_OK, [8, 2, 17, 22, 146])
    assert regm(9, 3200, 8640) is None     # more than 8 tokens
    assert regm(4, 8192, 28672) is None    # 194 rows per CTA
    assert regm(4, 3232, 100) is None      # K not a multiple of 64
    buf = (ctypes.c_int32 * 5)()
    assert L.bitlinear_decode_regm_shape(4, 3200, 8640, 0, buf) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_decode_regm_shape(4, 3200, 8640, 148, None) == _lib.BL_ERR_INVALID_ARG
    for M in (2, 3, 4, 5, 8):
        for K in range(64, 16384 + 1, 64):
            for N in (1, 148, 2368, 2369, 4736, 9472, 9473):
                r = regm(M, K, N)
                if r is None:
                    continue
                mt, rb, nj, rpc, grid = r[1]
                assert mt == (2 if M == 2 else (4 if M <= 4 else 8)) and rb in (1, 2, 4) and rb * mt <= 32
                assert nj in {1: (2, 4, 7, 8, 12, 17, 24), 2: (2, 4, 7, 8, 12, 17), 4: (2, 4, 7, 8)}[rb]
                assert rpc <= 16 * rb and 512 * nj >= K and rpc * grid >= N and (grid - 1) * rpc < N


def test_warp_mma_kernel_shape_picks():
    """The warp-MMA decode kernel for 9..16 tokens (x~ given): the rows of the
    one-token geometry, blocks of 16 rows (RBK), 16 / RBK parts of K, the
    smallest instantiated step count covering K, 16 token slots, and
    the activation slots plus partial tiles within one CTA's shared memory;
    up to 8 tokens the register kernel runs instead."""
    L = _lib.lib()

    def mma(M, K, N, sms=148):
        buf = (ctypes.c_int32 * 7)()
        st = L.bitlinear_decode_mma_shape(M, K, N, sms, buf)
        return None if st == _lib.BL_ERR_UNSUPPORTED else (st, list(buf))

    assert mma(16, 3200, 8640) == (_lib.BL_OK, [16, 4, 4, 13, 59, 147, 69632])
    assert mma(16, 8640, 3200) == (_lib.BL_OK, [16, 2, 8, 17, 22, 146, 156672])
    assert mma(9, 3200, 8640) == (_lib.BL_OK, [16, 4, 4, 13, 59, 147, 69632])
    assert mma(8, 3200, 8640) is None       # 8 tokens: the register kernel
    assert mma(17, 3200, 8640) is None      # more than 16 tokens: the tensor-core kernel
    assert mma(16, 8192, 8192) is None      # 32 steps per warp: beyond the register budget
    assert mma(16, 8192, 28672) is None     # 194 rows per CTA
    assert mma(12, 3232, 100) is None       # K not a multiple of 64
    buf = (ctypes.c_int32 * 7)()
    assert L.bitlinear_decode_mma_shape(12, 3200, 8640, 0, buf) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_decode_mma_shape(12, 3200, 8640, 148, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_decode_mma(2) == _lib.BL_ERR_INVALID_ARG
    for M in (9, 12, 16):
        for K in range(64, 24576 + 1, 64):
            for N in (1, 148, 2368, 2369, 4736, 9472, 9473):
                r = mma(M, K, N)
                if r is None:
                    continue
                slots, rbk, kp, ns, rpc, grid, smem = r[1]
                assert slots == 16 and rbk * kp == 16
                assert ns in (4, 9, 13, 17, 24) and kp * ns * 64 >= K and rpc <= 16 * rbk
                assert rpc * grid >= N and (grid - 1) * rpc < N and smem + 1024 <= 227 * 1024

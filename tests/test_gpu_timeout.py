"""The bounded-wait failure path, on a GPU, without a fault.

A separate build of the library (BL_TEST_HOOKS: every mbarrier wait gives up
after 1 ms, and bitlinear_test_set_fault(1) makes one unpack warp of the
tensor-core kernel withhold its arrival on the first stage's barrier) runs
one forward whose MMA-issuing thread then waits on a barrier that nothing
completes.  The wait runs out; the kernel records BL_ERR_TIMEOUT in the
library's device error word, drains the copies it had issued, frees its
tensor memory and returns without writing y.  The host reads the status
with bitlinear_device_error, and the next call (hook off) is bit-exact again
on the same context.  Nothing traps, faults or hangs: every wait is bounded.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import native as orc
from ternary_weight_linear_04_b200 import _lib
from ternary_weight_linear_04_b200 import build as libbuild
from ternary_weight_linear_04_b200 import inputs

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p
I64 = ctypes.c_int64


@pytest.fixture(scope="module")
def hooks():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    path = libbuild.build_test_hooks()
    L = ctypes.CDLL(path)
    L.bitlinear_forward_path.restype = ctypes.c_int
    L.bitlinear_forward_path.argtypes = [P, P, P, I64, I64, P, P, I64, P, ctypes.c_int, P,
                                         ctypes.c_int, ctypes.c_uint, P]
    L.bitlinear_test_set_fault.restype = ctypes.c_int
    L.bitlinear_test_set_fault.argtypes = [ctypes.c_int]
    L.bitlinear_set_tc_split.restype = ctypes.c_int
    L.bitlinear_set_tc_split.argtypes = [ctypes.c_int]
    L.bitlinear_device_error.restype = ctypes.c_int
    L.bitlinear_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), P]
    yield L
    L.bitlinear_test_set_fault(0)
    L.bitlinear_set_tc_split(0)


def _device_error(L):
    code = ctypes.c_int32(-1)
    assert L.bitlinear_device_error(ctypes.byref(code), None) == _lib.BL_OK
    return code.value


def test_withheld_arrival_times_out_and_the_next_call_is_exact(hooks):
    L = hooks
    M, K, N = 16, 1024, 256
    W, x = inputs.make_case(4711, M, K, N, act_dtype="bf16")
    packed, gamma, _ = orc.pack_weights(W)
    xq, eta, xsum = orc.quant_act(x)
    want_i, want_y = orc.forward(xq, eta, packed, gamma, K, N)
    d = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in
         dict(xq=xq, eta=eta, xsum=xsum.astype(np.int32), packed=packed,
              gamma=np.array([gamma], np.float32)).items()}
    y = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    yi = torch.zeros((M, N), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()

    def call():
        st = L.bitlinear_forward_path(P(d["xq"].data_ptr()), P(d["eta"].data_ptr()),
                                      P(d["xsum"].data_ptr()), M, K, P(d["packed"].data_ptr()),
                                      P(d["gamma"].data_ptr()), N, P(y.data_ptr()), _lib.BL_F32,
                                      P(yi.data_ptr()), _lib.BL_PATH_TCGEN05, 0, None)
        assert st == _lib.BL_OK
        torch.cuda.synchronize()

    assert L.bitlinear_set_tc_split(1) == _lib.BL_OK  # one CTA per tile: no cluster barriers
    assert _device_error(L) == _lib.BL_OK
    assert L.bitlinear_test_set_fault(1) == _lib.BL_OK
    call()
    assert _device_error(L) == _lib.BL_ERR_TIMEOUT
    assert torch.all(y == 7.0), "an aborted kernel must not write its output"
    assert _device_error(L) == _lib.BL_OK  # read and cleared
    assert L.bitlinear_test_set_fault(0) == _lib.BL_OK
    call()
    assert _device_error(L) == _lib.BL_OK
    np.testing.assert_array_equal(yi.cpu().numpy(), want_i)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), want_y.view(np.uint32))

"""The allocation-free packing entry point against the ordinary one.

bitlinear_pack_weights_noalloc serves callers that may not allocate device
memory themselves (a host framework that owns all device memory, or a path
that must not call cudaMalloc); it keeps its 2 KB pack scratch (exponent
buckets, an fp64 sum and its decision flag) in a device array inside the
library instead of a caller buffer.  Its packed bytes and gamma must equal
bitlinear_pack_weights' bit for bit, on consecutive calls (the shared scratch
must start from zero each time), also when a matrix needs the exact buckets
between two that do not.  This file is collected
last so that a run stopping at its first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from ternary_weight_linear_04_b200 import _lib
from ternary_weight_linear_04_b200 import build as libbuild
from ternary_weight_linear_04_b200 import inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _pack_both(L, W, stream):
    N, K = W.shape
    dev = W.device
    P = (K + 3) // 4
    ref_packed = torch.empty((N, P), dtype=torch.uint8, device=dev)
    ref_gamma = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(int(L.bitlinear_pack_workspace_bytes()), dtype=torch.uint8, device=dev)
    assert L.bitlinear_pack_weights(_p(W), N, K, _p(ref_packed), _p(ref_gamma), _p(ws), stream) == 0
    packed = torch.full((N, P), 0xAB, dtype=torch.uint8, device=dev)
    gamma = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    assert L.bitlinear_pack_weights_noalloc(_p(W), N, K, _p(packed), _p(gamma), stream) == 0
    torch.cuda.synchronize()
    return packed.cpu(), gamma.cpu(), ref_packed.cpu(), ref_gamma.cpu()


def test_noalloc_pack_matches_pack_on_consecutive_calls():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU test"
    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    mid = np.zeros(8 * 64, np.float32)  # mean |W| on an fp32 rounding midpoint: exact buckets
    mid[:64] = 1.0
    mid[64:128] = -(2.0 ** -24)
    cases = [inputs.make_case(31, 1, 4096, 1000, w_dist="laplace")[0],
             np.random.default_rng(5).permutation(mid).reshape(8, 64),
             inputs.make_case(32, 1, 3200, 777)[0]]
    for W in cases:  # two calls in a row: the second must not see the first's sums
        Wd = torch.from_numpy(W).cuda()
        packed, gamma, ref_packed, ref_gamma = _pack_both(L, Wd, stream)
        assert gamma.numpy().view(np.uint32)[0] == ref_gamma.numpy().view(np.uint32)[0]
        assert torch.equal(packed, ref_packed)


def test_noalloc_pack_rejects_oversize_and_bad_arguments():
    L = _lib.lib()
    fake = ctypes.c_void_p(256)
    assert L.bitlinear_pack_weights_noalloc(fake, 1 << 21, 1 << 20, fake, fake, None) == _lib.BL_ERR_UNSUPPORTED
    assert L.bitlinear_pack_weights_noalloc(None, 4, 4, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_pack_weights_noalloc(fake, 0, 4, fake, fake, None) == _lib.BL_ERR_INVALID_ARG

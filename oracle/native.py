"""ctypes front end of the scalar C oracle (``bitlinear_oracle.c``).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Same definitions as
``oracle.reference``, written independently in C; used for shapes too large
for the NumPy twin and for the timed CPU baseline.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_absmean_gamma.argtypes = [_ptr, _i64, _ptr, _ptr]
        L.oracle_ternarise_pack.argtypes = [_ptr, _i64, _i64, ctypes.c_float, _ptr, _ptr]
        L.oracle_quant_act.argtypes = [_ptr, _i64, _i64, _ptr, _ptr, _ptr, ctypes.c_int]
        L.oracle_forward.argtypes = [_ptr, _ptr, _i64, _i64, _ptr, ctypes.c_float, _i64,
                                     _ptr, _ptr, ctypes.c_int]
        L.oracle_forward_at.argtypes = [_ptr, _ptr, _i64, _i64, _ptr, ctypes.c_float, _i64,
                                        _ptr, _ptr, _i64, _ptr, _ptr]
        L.oracle_f32_to_bf16.argtypes = [_ptr, _ptr, _i64]
        L.oracle_f32_to_bf16.restype = None
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError("oracle %s failed with code %d" % (what, rc))


def max_threads():
    return int(lib().oracle_max_threads())


def absmean_gamma(W):
    W = np.ascontiguousarray(W, dtype=np.float32)
    g = np.zeros(1, np.float32)
    s = np.zeros(1, np.float64)
    _check(lib().oracle_absmean_gamma(_p(W), W.size, _p(g), _p(s)), "absmean_gamma")
    return np.float32(g[0]), float(s[0])


def ternarise_pack(W, gamma, want_ternary=False):
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    packed = np.zeros((N, (K + 3) // 4), np.uint8)
    t = np.zeros((N, K), np.int8) if want_ternary else None
    _check(lib().oracle_ternarise_pack(_p(W), N, K, ctypes.c_float(gamma), _p(packed),
                                       _p(t) if t is not None else None), "ternarise_pack")
    return packed, t


def pack_weights(W, want_ternary=False):
    gamma, _ = absmean_gamma(W)
    packed, t = ternarise_pack(W, gamma, want_ternary)
    return packed, gamma, t


def quant_act(x, nthreads=0):
    x = np.ascontiguousarray(x, dtype=np.float32)
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    eta = np.zeros(M, np.float32)
    xsum = np.zeros(M, np.int32)
    _check(lib().oracle_quant_act(_p(x), M, K, _p(xq), _p(eta), _p(xsum), nthreads), "quant_act")
    return xq, eta, xsum


def forward(xq, eta, packed, gamma, K, N, nthreads=0, want_y_int=True):
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    eta = np.ascontiguousarray(eta, dtype=np.float32)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    M = xq.shape[0]
    y_int = np.zeros((M, N), np.int32) if want_y_int else None
    y = np.zeros((M, N), np.float32)
    _check(lib().oracle_forward(_p(xq), _p(eta), M, K, _p(packed), ctypes.c_float(gamma), N,
                                _p(y_int) if y_int is not None else None, _p(y), nthreads),
           "forward")
    return y_int, y


def forward_at(xq, eta, packed, gamma, K, N, ms, ns):
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    eta = np.ascontiguousarray(eta, dtype=np.float32)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y_int = np.zeros(ms.size, np.int32)
    y = np.zeros(ms.size, np.float32)
    _check(lib().oracle_forward_at(_p(xq), _p(eta), xq.shape[0], K, _p(packed),
                                   ctypes.c_float(gamma), N, _p(ms), _p(ns), ms.size,
                                   _p(y_int), _p(y)), "forward_at")
    return y_int, y


def f32_to_bf16_bits(y):
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.zeros(y.shape, np.uint16)
    lib().oracle_f32_to_bf16(_p(y), _p(out), y.size)
    return out

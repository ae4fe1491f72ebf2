"""Loads ``libbitlinear.so`` and declares the C ABI of ``include/bitlinear.h``.

The library is built in-tree by ``ternary_weight_linear_04_b200.build`` (or
``__graft_entry__.build()``).  There is no fallback: if the library is
missing or fails to load, every call raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitlinear.so")

BL_OK, BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED, BL_ERR_ALIGNMENT, BL_ERR_CUDA, BL_ERR_TIMEOUT = range(6)
BL_F32, BL_BF16 = 0, 1
BL_PATH_AUTO, BL_PATH_GEMV, BL_PATH_TCGEN05, BL_PATH_GENERIC = range(4)
BL_FLAG_WEIGHTS_STATIC = 1

# name -> (restype, argtypes); every symbol include/bitlinear.h declares.
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
SIGNATURES = {
    "bitlinear_status_str": (ctypes.c_char_p, [_I]),
    "bitlinear_version": (ctypes.c_char_p, []),
    "bitlinear_packed_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "bitlinear_pack_workspace_bytes": (ctypes.c_size_t, []),
    "bitlinear_pack_weights": (_I, [_P, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_absmean_buckets": (_I, [_P, _I64, _I64, _P, _P]),
    "bitlinear_gamma_from_buckets": (_I, [_P, _I64, _P, _P]),
    "bitlinear_ternarise_pack": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "bitlinear_pack_weights_noalloc": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "bitlinear_quant_act": (_I, [_P, _I, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_rmsnorm_quant_act": (_I, [_P, _I, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_forward": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _I64, _P, _I, _P, _P]),
    "bitlinear_forward_path": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _I64, _P, _I, _P, _I,
                                    ctypes.c_uint, _P]),
    "bitlinear_linear": (_I, [_P, _I, _I64, _I64, _P, _P, _I64, _P, _I, _P, _P, _P, _P,
                              ctypes.c_uint, _P]),
    "bitlinear_select_path": (_I, [_I64, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_device_error": (_I, [_P, _P]),
    "bitlinear_decode_shape": (_I, [_I64, _I64, _I64, _I, _P]),
    "bitlinear_decode_shape_for": (_I, [_I64, _I64, _I64, _I, _I, _P]),
    "bitlinear_decode_reg_shape": (_I, [_I64, _I64, _I, _P]),
    "bitlinear_decode_regm_shape": (_I, [_I64, _I64, _I64, _I, _P]),
    "bitlinear_decode_mma_shape": (_I, [_I64, _I64, _I64, _I, _P]),
    "bitlinear_set_decode_mma": (_I, [_I]),
    "bitlinear_set_decode_reg": (_I, [_I]),
    "bitlinear_set_decode_shape": (_I, [_I, _I]),
    "bitlinear_set_tc_split": (_I, [_I]),
    "bitlinear_linear_group": (_I, [_P, _I, _I64, _I64, _I, _P, _P, _P, _P, _I, ctypes.c_uint, _P]),
    "bitlinear_packed3_stride": (_I64, [_I64]),
    "bitlinear_pack_weights3": (_I, [_P, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_forward3": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _I64, _P, _I, _P, _P]),
}

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_str(status), status))


def lib():
    """The loaded library; raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libbitlinear.so is not built (%s); run ternary_weight_linear_04_b200.build.build() "
                "or __graft_entry__.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_str(status):
    return lib().bitlinear_status_str(int(status)).decode()


def check(status, what):
    if status != BL_OK:
        raise BitLinearError(status, what)

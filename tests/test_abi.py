"""The C-ABI library loads without a GPU, exports every symbol its header
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from ternary_weight_linear_04_b200 import _lib
from ternary_weight_linear_04_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    syms = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            text = open(os.path.join(ROOT, "include", name)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            syms |= set(re.findall(r"\b(bitlinear_\w+)\s*\(", text))
    return syms


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.lib()


def test_library_exports_every_declared_symbol(L):
    syms = header_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(L, s), s
    assert set(_lib.SIGNATURES) == syms


def test_host_only_queries(L):
    assert L.bitlinear_packed_bytes(3, 5) == 3 * 2
    assert L.bitlinear_packed_bytes(8640, 3200) == 8640 * 800
    assert L.bitlinear_packed_bytes(0, 5) == 0
    assert L.bitlinear_pack_workspace_bytes() == 2048 + 16  # buckets, fp64 sum, flag
    assert L.bitlinear_version().decode().count(".") == 2
    for st in range(6):
        assert len(L.bitlinear_status_str(st)) > 0


def test_bad_arguments_are_rejected_without_a_launch(L):
    P = ctypes.c_void_p
    fake = P(256)  # never dereferenced: validation fails first
    assert L.bitlinear_pack_weights(None, 4, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_pack_weights(fake, 0, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_pack_weights(fake, 4, -1, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_pack_weights(fake, 1 << 21, 1 << 20, fake, fake, fake, None) == _lib.BL_ERR_UNSUPPORTED
    assert L.bitlinear_pack_weights(P(258), 4, 4, fake, fake, fake, None) == _lib.BL_ERR_ALIGNMENT
    assert L.bitlinear_quant_act(None, 0, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_quant_act(None, 0, 0, 4, None, None, None, None) == _lib.BL_OK
    assert L.bitlinear_quant_act(fake, 7, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_quant_act(fake, 0, -1, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_quant_act(fake, 0, 1, 0, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_quant_act(P(257), 1, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_ALIGNMENT
    assert L.bitlinear_quant_act(fake, 0, 0, 4, fake, fake, fake, None) == _lib.BL_OK  # M = 0: no-op
    ab, gb, tp = L.bitlinear_absmean_buckets, L.bitlinear_gamma_from_buckets, L.bitlinear_ternarise_pack
    assert ab(None, 4, 4, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert ab(fake, 0, 4, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert ab(fake, 1 << 21, 1 << 20, fake, None) == _lib.BL_ERR_UNSUPPORTED
    assert ab(fake, (1 << 20) + 1, 1 << 20, fake, None) == _lib.BL_ERR_UNSUPPORTED  # one row past N*K = 2^40
    assert ab(fake, 4, 4, P(260), None) == _lib.BL_ERR_ALIGNMENT
    assert gb(None, 16, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert gb(fake, 0, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert gb(fake, (1 << 40) + 1, fake, None) == _lib.BL_ERR_UNSUPPORTED
    assert gb(P(260), 16, fake, None) == _lib.BL_ERR_ALIGNMENT
    assert tp(fake, 4, 4, None, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert tp(fake, 4, -1, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert tp(fake, 1 << 21, 1 << 20, fake, fake, None) == _lib.BL_ERR_UNSUPPORTED
    assert tp(P(258), 4, 4, fake, fake, None) == _lib.BL_ERR_ALIGNMENT
    rq = L.bitlinear_rmsnorm_quant_act
    assert rq(None, 1, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert rq(None, 1, 0, 4, None, None, None, None) == _lib.BL_OK
    assert rq(fake, 7, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert rq(fake, 1, -1, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert rq(fake, 1, 1, 0, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert rq(fake, 0, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_UNSUPPORTED  # fp32 input
    assert rq(fake, 1, 1, (1 << 24) + 1, fake, fake, fake, None) == _lib.BL_ERR_UNSUPPORTED
    assert rq(P(257), 1, 1, 4, fake, fake, fake, None) == _lib.BL_ERR_ALIGNMENT
    assert rq(fake, 1, 1, 4, fake, P(258), fake, None) == _lib.BL_ERR_ALIGNMENT
    fwd = L.bitlinear_forward
    assert fwd(None, fake, fake, 1, 64, fake, fake, 8, fake, 0, None, None) == _lib.BL_ERR_INVALID_ARG
    assert fwd(fake, fake, fake, 1, 0, fake, fake, 8, fake, 0, None, None) == _lib.BL_ERR_INVALID_ARG
    assert fwd(fake, fake, fake, 1, 64, fake, fake, 0, fake, 0, None, None) == _lib.BL_ERR_INVALID_ARG
    assert fwd(fake, fake, fake, 1, 64, fake, fake, 8, fake, 9, None, None) == _lib.BL_ERR_INVALID_ARG
    assert fwd(fake, fake, fake, 1, 1 << 25, fake, fake, 8, fake, 0, None, None) == _lib.BL_ERR_UNSUPPORTED
    assert fwd(fake, P(258), fake, 1, 64, fake, fake, 8, fake, 0, None, None) == _lib.BL_ERR_ALIGNMENT
    assert fwd(fake, fake, fake, 0, 64, fake, fake, 8, fake, 0, None, None) == _lib.BL_OK
    assert fwd(None, None, None, 0, 64, fake, fake, 8, None, 0, None, None) == _lib.BL_OK
    assert fwd(None, None, None, 0, 64, None, fake, 8, None, 0, None, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_forward_path(fake, fake, fake, 1, 64, fake, fake, 8, fake, 0, None, 9, 0,
                                    None) == _lib.BL_ERR_INVALID_ARG
    lin = L.bitlinear_linear
    assert lin(fake, 0, 1, 64, None, fake, 8, fake, 0, None, None, None, None, 0, None) == _lib.BL_ERR_INVALID_ARG
    assert lin(fake, 3, 1, 64, fake, fake, 8, fake, 0, None, None, None, None, 0, None) == _lib.BL_ERR_INVALID_ARG
    assert lin(None, 0, 0, 64, fake, fake, 8, None, 0, None, None, None, None, 0, None) == _lib.BL_OK
    # a prefill-sized batch needs the caller's x~ scratch
    assert lin(fake, 1, 64, 64, fake, fake, 8, fake, 1, None, None, None, None, 0, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_device_error(None, None) == _lib.BL_ERR_INVALID_ARG
    shape = (ctypes.c_int32 * 10)()
    assert L.bitlinear_decode_shape(1, 3200, 8640, 1, None) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_decode_shape(1, 3200, 0, 1, shape) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_decode_shape(5, 3200, 8640, 1, shape) == _lib.BL_ERR_UNSUPPORTED   # M > 4
    assert L.bitlinear_decode_shape(1, 3232, 8640, 1, shape) == _lib.BL_ERR_UNSUPPORTED   # K % 64
    assert L.bitlinear_decode_shape(4, 65536, 64, 1, shape) == _lib.BL_ERR_UNSUPPORTED    # K * M'
    assert L.bitlinear_set_decode_shape(17, 0) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_decode_shape(-1, 0) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_decode_shape(0, 3) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_decode_shape(0, 32) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_decode_shape(0, 0) == _lib.BL_OK
    assert L.bitlinear_set_tc_split(-1) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_tc_split(9) == _lib.BL_ERR_INVALID_ARG
    assert L.bitlinear_set_tc_split(0) == _lib.BL_OK
    grp = L.bitlinear_linear_group
    arr1 = (ctypes.c_void_p * 1)(fake)
    n1 = (ctypes.c_int64 * 1)(64)
    assert grp(fake, 1, 1, 64, 0, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_INVALID_ARG  # nseg 0
    assert grp(fake, 1, 1, 64, 5, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_INVALID_ARG  # nseg 5
    assert grp(fake, 1, 1, 64, 1, None, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_INVALID_ARG
    assert grp(fake, 1, 1, 64, 1, arr1, arr1, (ctypes.c_int64 * 1)(0), arr1, 1, 0, None) == _lib.BL_ERR_INVALID_ARG
    assert grp(fake, 0, 1, 64, 1, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_UNSUPPORTED  # f32 x
    assert grp(fake, 1, 5, 64, 1, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_UNSUPPORTED  # M > 4
    assert grp(fake, 1, 1, 96, 1, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_UNSUPPORTED  # K % 64
    assert grp(P(257), 1, 1, 64, 1, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_ERR_ALIGNMENT
    assert grp(None, 1, 0, 64, 1, arr1, arr1, n1, arr1, 1, 0, None) == _lib.BL_OK  # M = 0
    assert [L.bitlinear_packed3_stride(K) for K in (0, 1, 80, 81, 3200, 8192)] == [0, 16, 16, 32, 640, 1648]
    p3 = L.bitlinear_pack_weights3
    assert p3(None, 4, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert p3(fake, 0, 4, fake, fake, fake, None) == _lib.BL_ERR_INVALID_ARG
    assert p3(P(258), 4, 4, fake, fake, fake, None) == _lib.BL_ERR_ALIGNMENT
    f3 = L.bitlinear_forward3
    assert f3(fake, fake, fake, 1, 0, fake, fake, 8, fake, 0, None, None) == _lib.BL_ERR_INVALID_ARG
    assert f3(fake, fake, fake, 1, 64, None, fake, 8, fake, 0, None, None) == _lib.BL_ERR_INVALID_ARG
    assert f3(fake, fake, fake, 1, 64, fake, fake, 8, fake, 7, None, None) == _lib.BL_ERR_INVALID_ARG
    assert f3(fake, fake, fake, 1, 1 << 20, fake, fake, 8, fake, 0, None, None) == _lib.BL_ERR_UNSUPPORTED
    assert f3(fake, fake, fake, 1, 64, P(264), fake, 8, fake, 0, None, None) == _lib.BL_ERR_ALIGNMENT
    assert f3(None, None, None, 0, 64, fake, fake, 8, None, 0, None, None) == _lib.BL_OK


def test_path_selection_is_host_logic(L):
    P = ctypes.c_void_p
    a = P(1 << 20)
    sel = L.bitlinear_select_path
    assert sel(1, 4096, 4096, a, a, a, None) == _lib.BL_PATH_GEMV
    assert sel(1, 28672, 8192, a, a, a, None) == _lib.BL_PATH_GEMV      # K * M' <= 131072
    assert sel(4, 65536, 64, a, a, a, None) == _lib.BL_PATH_TCGEN05     # K * M' > 131072
    assert sel(2048, 4096, 11008, a, a, a, None) == _lib.BL_PATH_TCGEN05
    assert sel(1, 4095, 4096, a, a, a, None) == _lib.BL_PATH_GENERIC      # ragged K
    assert sel(1, 4096, 4096, P((1 << 20) + 8), a, a, None) == _lib.BL_PATH_GENERIC  # misaligned


def test_product_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        _lib.lib()


def test_product_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "ternary_weight_linear_04_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in re.sub(r"#.*|//.*", "", text).lower() or f == "inputs.py", f

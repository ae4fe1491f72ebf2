"""The C ABI from plain C: include/bitlinear.h compiles as strict C99
(-Wall -Wextra -pedantic -Werror), a C program links libbitlinear.so, and the
host-only calls it makes return what the same calls return through ctypes.
No GPU is needed: every call used here returns before any device work."""
import ctypes
import os
import shutil
import subprocess
import tempfile

import pytest

from ternary_weight_linear_04_b200 import _lib
from ternary_weight_linear_04_b200 import build as libbuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def client_output():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib = libbuild.build()
    d = tempfile.mkdtemp(prefix="c_client_")
    exe = os.path.join(d, "client")
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "c_abi_client.c"),
                    "-L", libdir, "-lbitlinear", "-Wl,-rpath," + libdir, "-o", exe],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60).stdout
    shutil.rmtree(d, ignore_errors=True)
    lines = {}
    for line in out.splitlines():
        key, _, rest = line.partition(" ")
        lines.setdefault(key, []).append(rest)
    return lines


def test_header_is_strict_c99_and_links(client_output):
    assert client_output["version"][0].count(".") == 2


def test_host_calls_agree_with_ctypes(client_output):
    L = _lib.lib()
    assert client_output["version"][0] == L.bitlinear_version().decode()
    for line in client_output["status_str"]:
        code, text = line.split(" ", 1)
        assert text == L.bitlinear_status_str(int(code)).decode()
    assert client_output["packed_bytes"][0].split() == [str(8640 * 800), str(3 * 2)]
    assert client_output["workspace_bytes"][0] == str(L.bitlinear_pack_workspace_bytes())
    assert client_output["packed3_stride"][0].split() == [str(L.bitlinear_packed3_stride(3200)),
                                                          str(L.bitlinear_packed3_stride(1))]
    shape = (ctypes.c_int32 * 10)()
    st = L.bitlinear_decode_shape_for(1, 3200, 8640, 1, 148, shape)
    assert client_output["decode_shape_for"][0].split() == [str(st)] + [str(v) for v in shape]


def test_argument_errors_from_c(client_output):
    assert client_output["quant_act_null"][0] == str(_lib.BL_ERR_INVALID_ARG)
    assert client_output["quant_act_empty"][0] == str(_lib.BL_OK)
    assert client_output["forward_badk"][0] == str(_lib.BL_ERR_INVALID_ARG)
    assert client_output["rmsnorm_f32"][0] == str(_lib.BL_ERR_UNSUPPORTED)

"""Build ``libbitlinear.so`` (the C-ABI CUDA library) in-tree with nvcc.

Compiles ``csrc/bitlinear.cu`` for sm_100a only; the result sits next to
this file so it travels with the package.  Rebuilds when any source or the
public header is newer than the library.
"""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libbitlinear.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "bitlinear.h")])


# The fault-injection variant used only by the timeout test: the same
# sources with BL_TEST_HOOKS (1 ms wait limit, bitlinear_test_set_fault).
TEST_HOOKS_LIB = os.path.join(HERE, "libbitlinear_testhooks.so")


def needs_build(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force=False, verbose=False, extra=(), lib=LIB):
    if not force and not needs_build(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC, *FLAGS, *extra, "-I", INCLUDE, os.path.join(CSRC, "bitlinear.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build_test_hooks(force=False):
    """Builds the fault-injection variant (tests only; never loaded by the package)."""
    return build(force=force, extra=("-DBL_TEST_HOOKS",), lib=TEST_HOOKS_LIB)


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose=True, extra=sys.argv[1:]))

"""BitNet b1.58 BitLinear forward on one NVIDIA B200 (sm_100a).

The compute lives in ``libbitlinear.so`` (CUDA, C ABI in
``include/bitlinear.h``); this package is its thin Python binding.
Importing it does not load the library; the first call does, and fails
loudly if the library is not built.
"""
__version__ = "0.1.0"


def __getattr__(name):
    if name in ("pack_weights", "quant_act", "forward", "linear", "BitLinear", "packed_bytes",
                "select_path", "device_error"):
        from . import bitlinear
        return getattr(bitlinear, name)
    raise AttributeError(name)

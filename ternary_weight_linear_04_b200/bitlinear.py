"""Python binding of the BitLinear C ABI (``include/bitlinear.h``).

Argument marshalling only: torch supplies device memory and the current
CUDA stream; every step of the layer runs in the library's CUDA kernels.
Names follow the C entry points: ``pack_weights``, ``quant_act``,
``forward`` (plus ``BitLinear``, a small holder of one packed matrix).
"""
import ctypes

import torch

from . import _lib
from ._lib import check

PATHS = {"auto": _lib.BL_PATH_AUTO, "gemv": _lib.BL_PATH_GEMV,
         "tcgen05": _lib.BL_PATH_TCGEN05, "generic": _lib.BL_PATH_GENERIC}
PATH_NAMES = {v: k for k, v in PATHS.items()}
_DTYPES = {torch.float32: _lib.BL_F32, torch.bfloat16: _lib.BL_BF16}


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def packed_bytes(N, K):
    return int(_lib.lib().bitlinear_packed_bytes(N, K))


def _pack_workspace(workspace, dev):
    """The caller's pack scratch, checked for size, or a new one."""
    need = int(_lib.lib().bitlinear_pack_workspace_bytes())
    if workspace is None:
        return torch.empty(need, dtype=torch.uint8, device=dev)
    _require_cuda(workspace)
    if workspace.numel() * workspace.element_size() < need or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous buffer of at least %d bytes" % need)
    return workspace


def pack_weights(W, stream=None, workspace=None, packed=None, gamma=None):
    """fp32 latent weights (N x K, CUDA) -> (packed uint8 N x ceil(K/4), gamma fp32[1])."""
    _require_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    L = _lib.lib()
    dev = W.device
    if packed is None:
        packed = torch.empty((N, (K + 3) // 4), dtype=torch.uint8, device=dev)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=dev)
    workspace = _pack_workspace(workspace, dev)
    check(L.bitlinear_pack_weights(_ptr(W), N, K, _ptr(packed), _ptr(gamma), _ptr(workspace),
                                   _stream(stream)), "bitlinear_pack_weights")
    return packed, gamma


def absmean_buckets(W, stream=None, out=None):
    """Exact |W| exponent buckets of a row shard (fp32 N x K, CUDA) -> int64[256]
    (uint64 totals in two's complement; sum them over shards with an int64
    all-reduce)."""
    _require_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    b = out if out is not None else torch.empty(256, dtype=torch.int64, device=W.device)
    check(_lib.lib().bitlinear_absmean_buckets(_ptr(W), N, K, _ptr(b), _stream(stream)),
          "bitlinear_absmean_buckets")
    return b


def gamma_from_buckets(buckets, count, stream=None, out=None):
    """gamma (fp32[1]) from bucket totals of a whole matrix of `count` elements."""
    _require_cuda(buckets)
    if buckets.dtype != torch.int64 or buckets.numel() != 256:
        raise ValueError("buckets must be 256 int64 values")
    g = out if out is not None else torch.empty(1, dtype=torch.float32, device=buckets.device)
    check(_lib.lib().bitlinear_gamma_from_buckets(_ptr(buckets), int(count), _ptr(g),
                                                  _stream(stream)), "bitlinear_gamma_from_buckets")
    return g


def ternarise_pack(W, gamma, stream=None, out=None):
    """Rows of W (fp32 N x K, CUDA) ternarised with a given gamma and packed
    (uint8 N x ceil(K/4))."""
    _require_cuda(W, gamma)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    p = out if out is not None else torch.empty((N, (K + 3) // 4), dtype=torch.uint8,
                                                 device=W.device)
    check(_lib.lib().bitlinear_ternarise_pack(_ptr(W), N, K, _ptr(gamma), _ptr(p), _stream(stream)),
          "bitlinear_ternarise_pack")
    return p


def quant_act(x, stream=None, out=None):
    """Activations (M x K, fp32 or bf16, CUDA) -> (xq int8 M x K, eta fp32 M, xsum int32 M)."""
    _require_cuda(x)
    if x.dim() != 2 or x.dtype not in _DTYPES:
        raise ValueError("x must be a 2-D float32 or bfloat16 tensor")
    M, K = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty((M, K), dtype=torch.int8, device=dev),
               torch.empty(M, dtype=torch.float32, device=dev),
               torch.empty(M, dtype=torch.int32, device=dev))
    xq, eta, xsum = out
    check(_lib.lib().bitlinear_quant_act(_ptr(x), _DTYPES[x.dtype], M, K, _ptr(xq), _ptr(eta),
                                         _ptr(xsum), _stream(stream)), "bitlinear_quant_act")
    return xq, eta, xsum


def rmsnorm_quant_act(x, stream=None, out=None):
    """RMSNorm (no affine, eps 1e-6) fused with the per-token quantiser.
    Activations (M x K, bf16, CUDA) -> (xq int8 M x K, eta fp32 M, xsum int32 M)
    of the normalised rows."""
    _require_cuda(x)
    if x.dim() != 2 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    M, K = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty((M, K), dtype=torch.int8, device=dev),
               torch.empty(M, dtype=torch.float32, device=dev),
               torch.empty(M, dtype=torch.int32, device=dev))
    xq, eta, xsum = out
    check(_lib.lib().bitlinear_rmsnorm_quant_act(_ptr(x), _DTYPES[x.dtype], M, K, _ptr(xq),
                                                 _ptr(eta), _ptr(xsum), _stream(stream)),
          "bitlinear_rmsnorm_quant_act")
    return xq, eta, xsum


def forward(xq, eta, xsum, packed, gamma, N, out_dtype=torch.bfloat16, want_int=False,
            path="auto", stream=None, out=None, out_int=None, weights_static=False):
    """Integer accumulation + rescale.  Returns y (M x N), or (y, y_int) if want_int.
    weights_static: packed/gamma are not written by pending work on the stream
    (lets the decode kernel start streaming them early)."""
    _require_cuda(xq, eta, xsum, packed, gamma)
    M, K = xq.shape
    if packed.shape != (N, (K + 3) // 4):
        raise ValueError("packed shape %s does not match N=%d, K=%d" % (tuple(packed.shape), N, K))
    dev = xq.device
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=dev)
    y_int = out_int
    if want_int and y_int is None:
        y_int = torch.empty((M, N), dtype=torch.int32, device=dev)
    check(_lib.lib().bitlinear_forward_path(
        _ptr(xq), _ptr(eta), _ptr(xsum), M, K, _ptr(packed), _ptr(gamma), N, _ptr(y),
        _DTYPES[y.dtype], _ptr(y_int), PATHS[path],
        _lib.BL_FLAG_WEIGHTS_STATIC if weights_static else 0, _stream(stream)), "bitlinear_forward")
    return (y, y_int) if want_int else y


def fused_decode_ok(M, K):
    """Whether bitlinear_linear runs its single fused decode kernel for (M, K)
    with bf16 activations: one or two tokens (the same rule as the library;
    otherwise it needs x~ scratch)."""
    mt = 1 if M <= 1 else 2
    return 1 <= M <= 2 and K >= 64 and K % 64 == 0 and K * mt <= 131072


DECODE_SHAPE_FIELDS = ("team_warps", "rows_per_block", "teams", "words_per_lane", "rows_per_cta",
                       "ctas", "blocks_per_stage", "stages", "x_staged", "smem_bytes")


def decode_shape(M, K, N, fused=True):
    """The decode kernel's launch shape for (M, K, N) on the current device,
    as a dict (see bitlinear_decode_shape)."""
    buf = (ctypes.c_int32 * len(DECODE_SHAPE_FIELDS))()
    check(_lib.lib().bitlinear_decode_shape(M, K, N, 1 if fused else 0, buf), "bitlinear_decode_shape")
    return dict(zip(DECODE_SHAPE_FIELDS, list(buf)))


def decode_reg_shape(K, N, sms=None):
    """Shape of the one-token register-resident kernel of bitlinear_linear for
    (K, N) as a dict, or None when that kernel does not take the layer.  sms
    defaults to the current device's SM count."""
    if sms is None:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    buf = (ctypes.c_int32 * 4)()
    st = _lib.lib().bitlinear_decode_reg_shape(K, N, sms, buf)
    if st == _lib.BL_ERR_UNSUPPORTED:
        return None
    check(st, "bitlinear_decode_reg_shape")
    return dict(zip(("rows_per_warp", "words_per_lane", "rows_per_cta", "ctas"), list(buf)))


def decode_regm_shape(M, K, N, sms=None):
    """Shape of the register-resident kernel for 2..8 tokens with x~ given,
    as a dict, or None when that kernel does not take (M, K, N).  sms
    defaults to the current device's SM count."""
    if sms is None:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    buf = (ctypes.c_int32 * 5)()
    st = _lib.lib().bitlinear_decode_regm_shape(M, K, N, sms, buf)
    if st == _lib.BL_ERR_UNSUPPORTED:
        return None
    check(st, "bitlinear_decode_regm_shape")
    return dict(zip(("token_slots", "rows_per_warp", "words_per_lane", "rows_per_cta", "ctas"), list(buf)))


def decode_mma_shape(M, K, N, sms=None):
    """Shape of the warp-MMA decode kernel for 9..16 tokens with x~ given, as
    a dict, or None when that kernel does not take (M, K, N).  sms defaults
    to the current device's SM count."""
    if sms is None:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    buf = (ctypes.c_int32 * 7)()
    st = _lib.lib().bitlinear_decode_mma_shape(M, K, N, sms, buf)
    if st == _lib.BL_ERR_UNSUPPORTED:
        return None
    check(st, "bitlinear_decode_mma_shape")
    return dict(zip(("token_slots", "row_blocks", "k_parts", "k_steps", "rows_per_cta", "ctas",
                     "smem_bytes"), list(buf)))


def set_decode_mma(enable=True):
    """Turn the warp-MMA decode kernel on (default) or off for later launches
    in this process."""
    check(_lib.lib().bitlinear_set_decode_mma(1 if enable else 0), "bitlinear_set_decode_mma")


def set_decode_reg(enable=True):
    """Turn the register-resident kernels (one token fused; 2..8 tokens with
    x~ given) on (default) or off for later launches in this process (off:
    the shared-memory decode kernel)."""
    check(_lib.lib().bitlinear_set_decode_reg(1 if enable else 0), "bitlinear_set_decode_reg")


def set_tc_split(k_split=0):
    """Force the K split (CTAs per cluster) of the tensor-core kernel for later
    launches in this process (0 = the library's choice)."""
    check(_lib.lib().bitlinear_set_tc_split(k_split), "bitlinear_set_tc_split")


def set_decode_shape(team_warps=0, rows_per_block=0):
    """Force the decode kernel's team width and row-block height for later
    launches in this process (0 = the library's choice)."""
    check(_lib.lib().bitlinear_set_decode_shape(team_warps, rows_per_block), "bitlinear_set_decode_shape")


def linear(x, packed, gamma, N, out_dtype=torch.bfloat16, want_quant=False, want_int=False,
           weights_static=False, stream=None, out=None, scratch=None):
    """The whole per-token layer (quantise + accumulate + rescale) in one call.
    Returns y, plus (xq, eta, xsum) if want_quant and y_int if want_int."""
    _require_cuda(x, packed, gamma)
    if x.dim() != 2 or x.dtype not in _DTYPES:
        raise ValueError("x must be a 2-D float32 or bfloat16 tensor")
    M, K = x.shape
    if packed.shape != (N, (K + 3) // 4):
        raise ValueError("packed shape %s does not match N=%d, K=%d" % (tuple(packed.shape), N, K))
    dev = x.device
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=dev)
    decode = fused_decode_ok(M, K) and x.dtype == torch.bfloat16
    if scratch is not None:
        xq, eta, xsum = scratch
    elif want_quant or not decode:
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        eta = torch.empty(M, dtype=torch.float32, device=dev)
        xsum = torch.empty(M, dtype=torch.int32, device=dev)
    else:
        xq = eta = xsum = None
    y_int = torch.empty((M, N), dtype=torch.int32, device=dev) if want_int else None
    check(_lib.lib().bitlinear_linear(
        _ptr(x), _DTYPES[x.dtype], M, K, _ptr(packed), _ptr(gamma), N, _ptr(y), _DTYPES[y.dtype],
        _ptr(xq), _ptr(eta), _ptr(xsum), _ptr(y_int),
        _lib.BL_FLAG_WEIGHTS_STATIC if weights_static else 0, _stream(stream)), "bitlinear_linear")
    out_ = (y,)
    if want_quant:
        out_ += ((xq, eta, xsum),)
    if want_int:
        out_ += (y_int,)
    return out_[0] if len(out_) == 1 else out_


def linear_group(x, packed, gamma, out_dtype=torch.bfloat16, weights_static=False, stream=None,
                 out=None):
    """bitlinear_linear_group: the per-token layer for up to 4 matrices that
    share the activations x (bf16 M x K, M <= 4), in one launch.  packed and
    gamma are lists (one per matrix); returns the list of outputs."""
    _require_cuda(x, *packed, *gamma)
    if x.dim() != 2 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    M, K = x.shape
    n = len(packed)
    if n != len(gamma) or not 1 <= n <= 4:
        raise ValueError("one gamma per packed matrix, 1 to 4 matrices")
    Ns = [p.shape[0] for p in packed]
    for p in packed:
        if p.shape[1] != (K + 3) // 4:
            raise ValueError("packed shape %s does not match K=%d" % (tuple(p.shape), K))
    ys = out if out is not None else [torch.empty((M, N), dtype=out_dtype, device=x.device) for N in Ns]
    arr = ctypes.c_void_p * n
    check(_lib.lib().bitlinear_linear_group(
        _ptr(x), _lib.BL_BF16, M, K, n, arr(*[_ptr(p) for p in packed]), arr(*[_ptr(g) for g in gamma]),
        (ctypes.c_int64 * n)(*Ns), arr(*[_ptr(y) for y in ys]), _DTYPES[ys[0].dtype],
        _lib.BL_FLAG_WEIGHTS_STATIC if weights_static else 0, _stream(stream)), "bitlinear_linear_group")
    return ys


def packed3_stride(K):
    """Row stride (bytes) of the base-3 layout."""
    return int(_lib.lib().bitlinear_packed3_stride(K))


def pack_weights3(W, stream=None, workspace=None):
    """bitlinear_pack_weights3: (packed3 N x stride uint8, gamma) on W's device."""
    _require_cuda(W)
    N, K = W.shape
    dev = W.device
    packed3 = torch.empty((N, packed3_stride(K)), dtype=torch.uint8, device=dev)
    gamma = torch.empty(1, dtype=torch.float32, device=dev)
    ws = _pack_workspace(workspace, dev)
    check(_lib.lib().bitlinear_pack_weights3(_ptr(W), N, K, _ptr(packed3), _ptr(gamma), _ptr(ws),
                                             _stream(stream)), "bitlinear_pack_weights3")
    return packed3, gamma


def forward3(xq, eta, xsum, packed3, gamma, N, out_dtype=torch.float32, want_int=False,
             stream=None, out=None):
    """bitlinear_forward3: the accumulate + rescale on base-3 packed weights."""
    _require_cuda(xq, eta, xsum, packed3, gamma)
    M, K = xq.shape
    if packed3.shape != (N, packed3_stride(K)):
        raise ValueError("packed3 shape %s does not match N=%d, K=%d" % (tuple(packed3.shape), N, K))
    y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=xq.device)
    y_int = torch.empty((M, N), dtype=torch.int32, device=xq.device) if want_int else None
    check(_lib.lib().bitlinear_forward3(_ptr(xq), _ptr(eta), _ptr(xsum), M, K, _ptr(packed3), _ptr(gamma),
                                        N, _ptr(y), _DTYPES[y.dtype], _ptr(y_int), _stream(stream)),
          "bitlinear_forward3")
    return (y, y_int) if want_int else y


def select_path(M, K, N, xq, packed, y, y_int=None):
    return PATH_NAMES[int(_lib.lib().bitlinear_select_path(M, K, N, _ptr(xq), _ptr(packed),
                                                           _ptr(y), _ptr(y_int)))]


def device_error(stream=None):
    code = ctypes.c_int32(0)
    check(_lib.lib().bitlinear_device_error(ctypes.byref(code), _stream(stream)),
          "bitlinear_device_error")
    return int(code.value)


class BitLinear:
    """One packed ternary matrix and its gamma, applied to activations.

    ``BitLinear.from_latent(W)`` packs fp32 latent weights (N x K) once;
    calling the object quantises x (M x K) per token and runs the integer
    accumulate + rescale.  With ``rmsnorm=True`` the tokens are first
    RMS-normalised (no affine weight, eps 1e-6; bf16 x), as BitLinear158.forward
    does in [Production] "2. Absmax Dynamic Activation Quantization"."""

    def __init__(self, packed, gamma, in_features, out_features, rmsnorm=False):
        self.packed, self.gamma = packed, gamma
        self.in_features, self.out_features = in_features, out_features
        self.rmsnorm = rmsnorm

    @classmethod
    def from_latent(cls, W, stream=None, rmsnorm=False):
        packed, gamma = pack_weights(W, stream=stream)
        return cls(packed, gamma, W.shape[1], W.shape[0], rmsnorm=rmsnorm)

    def __call__(self, x, out_dtype=torch.bfloat16, stream=None):
        if self.rmsnorm:
            xq, eta, xsum = rmsnorm_quant_act(x, stream=stream)
            return forward(xq, eta, xsum, self.packed, self.gamma, self.out_features,
                           out_dtype=out_dtype, stream=stream, weights_static=True)
        return linear(x, self.packed, self.gamma, self.out_features, out_dtype=out_dtype,
                      weights_static=True, stream=stream)

// bitlinear.cu -- C ABI of the BitLinear library: argument checks, kernel
// selection and launches.  Declarations and the contract of every entry
// point are in include/bitlinear.h.  All kernels live in this one
// translation unit (the .cuh files) so the device error word needs no
// relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>

#include "bitlinear.h"
#include "common.cuh"
#include "decode.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "pack.cuh"
#include "quant.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kGemvMaxM = 4;  // largest token count the CUDA-core decode kernel takes

// Tokens rounded up to the decode kernel's widths (1, 2, 4).
inline int decode_mt(int64_t M) { return M <= 1 ? 1 : (M <= 2 ? 2 : 4); }

// Whether the decode kernel takes (M, K): K % 64 == 0, M <= 4 and
// K * MT <= 32768 (each thread stages at most 8 words x MT tokens of
// activations, 32 KB of shared memory per CTA).
inline bool decode_ok(int64_t M, int64_t K) {
  return M >= 1 && M <= kGemvMaxM && K % 64 == 0 && K * decode_mt(M) <= 32768;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bl_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous kernel on the stream finishes; every such kernel calls
// griddepcontrol.wait before it reads anything an earlier kernel wrote.
template <typename... KArgs, typename... Args>
bl_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return BL_ERR_CUDA;
  }
  return launch_status();
}

// Once per device: is it an sm_100 part, and how many SMs does it have.
struct DeviceInfo {
  int checked = 0;
  int ok = 0;
  int sms = 148;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

bl_status device_info(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BL_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.sms = count > 0 ? count : 148;
    d.checked = 1;
  }
  if (sms) *sms = d.sms;
  return d.ok ? BL_OK : BL_ERR_UNSUPPORTED;
}

// Once per device and kernel: raise the dynamic shared memory limit and ask
// for the largest shared-memory carveout.  Every kernel of the library uses
// the same carveout, so CTAs of consecutive kernels can share an SM (the
// carveout of an SM only changes while it is idle), which is what lets a
// kernel launched with programmatic dependent launch start early.
template <typename Kern>
bool ensure_smem(Kern kern, size_t bytes, int* done_flags) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (done_flags[dev] >= static_cast<int>(bytes) && done_flags[dev] > 0) return true;
  if (bytes > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return false;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return false;
  done_flags[dev] = bytes > 0 ? static_cast<int>(bytes) : 1;
  return true;
}

// ------------------------------------------------------------ tensor maps

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major uint8 matrix rows x cols (cols contiguous), box box_rows x
// box_cols bytes; out-of-bounds elements read as zero.
bool make_tmap_u8(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, uint32_t box_cols, bool swizzle128) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ launchers

// Decode kernel (M <= 4 tokens): one CTA per SM, each owning a contiguous
// block of rows, so the next kernel's CTA fits beside it under programmatic
// dependent launch.  XT = activation type when the quantiser is fused, or
// bl::DecNoFuse when x~ is given.
template <int MT, typename XT, typename OutT>
bl_status launch_decode_kernel(const bl::DecodeArgs& a0, int sms, cudaStream_t st) {
  static int smem_done[kMaxDevices] = {0};
  bl::DecodeArgs a = a0;
  const int64_t P = a.K / 4;
  const int64_t nwj = (a.K / 16 + bl::kDecColThreads - 1) / bl::kDecColThreads;
  int64_t rps = bl::kDecStageTarget / P;  // rows per stage (one chunk)
  if (rps > 32 / MT) rps = 32 / MT;
  if (rps < 1) rps = 1;
  // One CTA per SM, unless that would give a CTA more chunks than its
  // reduction slots hold.
  int64_t grid = sms;
  const int64_t min_grid = (a.N + rps * bl::kDecMaxChunks - 1) / (rps * bl::kDecMaxChunks);
  if (grid < min_grid) grid = min_grid;
  if (grid > a.N) grid = a.N;
  a.rows_per_cta = static_cast<int>((a.N + grid - 1) / grid);
  grid = (a.N + a.rows_per_cta - 1) / a.rows_per_cta;
  if (rps > a.rows_per_cta) rps = a.rows_per_cta;
  a.rows_per_stage = static_cast<int>(rps);
  const int64_t chunks = (a.rows_per_cta + rps - 1) / rps;
  if (chunks > bl::kDecMaxChunks || grid > 0x7FFFFFFF) return BL_ERR_UNSUPPORTED;
  int64_t stages = bl::kDecSmemBudget / (rps * P);
  if (stages > bl::kDecMaxStages) stages = bl::kDecMaxStages;
  if (stages > chunks) stages = chunks;
  if (stages < 1) stages = 1;
  a.stages = static_cast<int>(stages);
  constexpr int64_t kXElem = std::is_same<XT, bl::DecNoFuse>::value ? 1 : 2;
  const size_t smem = static_cast<size_t>(nwj * MT * bl::kDecColThreads * 16) +
                      static_cast<size_t>((MT * a.K * kXElem + 127) & ~int64_t{127}) +
                      static_cast<size_t>(stages * rps * P) + sizeof(bl::DecTail);
  auto kern = bl::k_decode<MT, XT, OutT>;
  if (!ensure_smem(kern, 227 * 1024, smem_done)) return BL_ERR_CUDA;
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(bl::kDecThreads), smem, st, a);
}

template <typename XT, typename OutT>
bl_status launch_decode(const bl::DecodeArgs& a, int sms, cudaStream_t st) {
  if (!decode_ok(a.M, a.K)) return BL_ERR_UNSUPPORTED;
  switch (decode_mt(a.M)) {
    case 1: return launch_decode_kernel<1, XT, OutT>(a, sms, st);
    case 2: return launch_decode_kernel<2, XT, OutT>(a, sms, st);
    default: return launch_decode_kernel<4, XT, OutT>(a, sms, st);
  }
}

template <typename OutT>
bl_status launch_generic(const int8_t* xq, const float* eta, int64_t M, int64_t K,
                         const uint8_t* packed, const float* gamma, int64_t N, void* y,
                         int32_t* y_int, int sms, cudaStream_t st) {
  const int64_t mblocks = (M + 7) / 8;
  for (int64_t mb0 = 0; mb0 < mblocks; mb0 += 65535) {
    const int64_t mb = (mblocks - mb0) < 65535 ? (mblocks - mb0) : 65535;
    int64_t ctas = (N + 7) / 8;
    if (ctas > static_cast<int64_t>(sms) * 16) ctas = static_cast<int64_t>(sms) * 16;
    dim3 grid(static_cast<unsigned>(ctas), static_cast<unsigned>(mb));
    const int64_t m_off = mb0 * 8;
    static int carve_done[kMaxDevices] = {0};
    if (!ensure_smem(bl::k_gemv_generic<OutT>, 0, carve_done)) return BL_ERR_CUDA;
    const bl_status s = launch_pdl(
        bl::k_gemv_generic<OutT>, grid, dim3(256), 0, st, xq + m_off * K, eta + m_off, M - m_off,
        K, packed, gamma, N, static_cast<void*>(static_cast<char*>(y) + m_off * N * sizeof(OutT)),
        y_int ? y_int + m_off * N : static_cast<int32_t*>(nullptr));
    if (s != BL_OK) return s;
  }
  return BL_OK;
}

template <int BM, typename OutT>
bl_status launch_tc_bm(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                       const uint8_t* packed, const float* gamma, int N, void* y, int32_t* y_int,
                       cudaStream_t st) {
  using Cfg = bl::TcCfg<BM>;
  static int smem_done[kMaxDevices] = {0};
  auto kern = bl::k_gemm_tc<BM, OutT>;
  if (!ensure_smem(kern, Cfg::kSmem, smem_done)) return BL_ERR_CUDA;
  CUtensorMap tm_x, tm_w;
  if (!make_tmap_u8(&tm_x, xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K), BM, bl::kTcBK, true))
    return BL_ERR_CUDA;
  if (!make_tmap_u8(&tm_w, packed, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 4),
                    bl::kTcBN, bl::kTcBK / 4, false))
    return BL_ERR_CUDA;
  dim3 grid((N + bl::kTcBN - 1) / bl::kTcBN, (M + BM - 1) / BM);
  if (grid.y > 65535) return BL_ERR_UNSUPPORTED;
  return launch_pdl(kern, grid, dim3(bl::kTcThreads), Cfg::kSmem, st, tm_x, tm_w, eta, xsum, gamma,
                    M, K, N, y, y_int);
}

template <typename OutT>
bl_status launch_tc(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                    const uint8_t* packed, const float* gamma, int N, void* y, int32_t* y_int,
                    cudaStream_t st) {
  if (M <= 16) return launch_tc_bm<16, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, st);
  if (M <= 32) return launch_tc_bm<32, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, st);
  if (M <= 64) return launch_tc_bm<64, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, st);
  if (M <= 128) return launch_tc_bm<128, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, st);
  return launch_tc_bm<256, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, st);
}

bool fast_layout_ok(int64_t K, const void* xq, const void* packed, const void* y, const void* y_int) {
  return (K % 64 == 0) && aligned(xq, 16) && aligned(packed, 16) && aligned(y, 16) &&
         (y_int == nullptr || aligned(y_int, 16));
}

bl_path select_path(int64_t M, int64_t K, const void* xq, const void* packed, const void* y,
                    const void* y_int) {
  if (!fast_layout_ok(K, xq, packed, y, y_int) || K > (1 << 30)) return BL_PATH_GENERIC;
  if (decode_ok(M, K)) return BL_PATH_GEMV;
  return BL_PATH_TCGEN05;
}

bl_status forward_impl(const int8_t* xq, const float* eta, const int32_t* xsum, int64_t M,
                       int64_t K, const uint8_t* packed, const float* gamma, int64_t N, void* y,
                       bl_dtype ydt, int32_t* y_int, bl_path path, unsigned flags, void* stream) {
  if (M < 0 || K < 1 || N < 1) return BL_ERR_INVALID_ARG;
  if (ydt != BL_F32 && ydt != BL_BF16) return BL_ERR_INVALID_ARG;
  if (path < BL_PATH_AUTO || path > BL_PATH_GENERIC) return BL_ERR_INVALID_ARG;
  if (!packed || !gamma) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;  // empty batch: the M-sized buffers may be NULL
  if (!xq || !eta || !xsum || !y) return BL_ERR_INVALID_ARG;
  if (127 * K >= (int64_t{1} << 31)) return BL_ERR_UNSUPPORTED;
  if (!aligned(eta, 4) || !aligned(xsum, 4) || !aligned(gamma, 4) ||
      (y_int && !aligned(y_int, 4)) || !aligned(y, ydt == BL_F32 ? 4 : 2))
    return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  if (path == BL_PATH_AUTO) path = select_path(M, K, xq, packed, y, y_int);
  const cudaStream_t s = as_stream(stream);
  if (path == BL_PATH_GEMV) {
    if (!fast_layout_ok(K, xq, packed, y, y_int) || !decode_ok(M, K) ||
        N > INT32_MAX / 2)
      return BL_ERR_UNSUPPORTED;
    bl::DecodeArgs a = {};
    a.x = xq; a.eta = eta; a.xsum = xsum; a.M = (int)M; a.K = (int)K; a.N = (int)N;
    a.packed = packed; a.gamma = gamma; a.y = y; a.y_int = y_int;
    a.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
    return ydt == BL_F32 ? launch_decode<bl::DecNoFuse, float>(a, sms, s)
                         : launch_decode<bl::DecNoFuse, __nv_bfloat16>(a, sms, s);
  }
  if (path == BL_PATH_TCGEN05) {
    if (!fast_layout_ok(K, xq, packed, y, y_int) || M > INT32_MAX / 2 || N > INT32_MAX / 2 ||
        K > (1 << 30))
      return BL_ERR_UNSUPPORTED;
    return ydt == BL_F32
               ? launch_tc<float>(xq, eta, xsum, (int)M, (int)K, packed, gamma, (int)N, y, y_int, s)
               : launch_tc<__nv_bfloat16>(xq, eta, xsum, (int)M, (int)K, packed, gamma, (int)N, y,
                                          y_int, s);
  }
  return ydt == BL_F32
             ? launch_generic<float>(xq, eta, M, K, packed, gamma, N, y, y_int, sms, s)
             : launch_generic<__nv_bfloat16>(xq, eta, M, K, packed, gamma, N, y, y_int, sms, s);
}

}  // namespace

extern "C" {

const char* bitlinear_status_str(bl_status status) {
  switch (status) {
    case BL_OK: return "ok";
    case BL_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or dtype)";
    case BL_ERR_UNSUPPORTED: return "unsupported (size beyond limits, layout, or not an sm_100 GPU)";
    case BL_ERR_ALIGNMENT: return "pointer alignment requirement not met";
    case BL_ERR_CUDA: return "CUDA runtime error";
    case BL_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

const char* bitlinear_version(void) { return "0.1.0"; }

size_t bitlinear_packed_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 1) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>((K + 3) / 4);
}

size_t bitlinear_pack_workspace_bytes(void) { return bl::kBuckets * sizeof(unsigned long long); }

bl_status bitlinear_pack_weights(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                 float* gamma, void* workspace, void* stream) {
  if (!W || !packed || !gamma || !workspace) return BL_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(workspace, 8) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  auto* buckets = static_cast<unsigned long long*>(workspace);
  bl::k_zero_u64<<<1, 256, 0, s>>>(buckets, bl::kBuckets);
  if ((st = launch_status()) != BL_OK) return st;
  const int64_t count = N * K;
  int64_t ctas = (count / 4 + 255) / 256;
  if (ctas > static_cast<int64_t>(sms) * 8) ctas = static_cast<int64_t>(sms) * 8;
  if (ctas < 1) ctas = 1;
  bl::k_absmean_buckets<<<static_cast<int>(ctas), 256, 0, s>>>(W, count, buckets);
  if ((st = launch_status()) != BL_OK) return st;
  bl::k_gamma_finalize<<<1, 32, 0, s>>>(buckets, count, gamma);
  if ((st = launch_status()) != BL_OK) return st;
  const int64_t bytes = N * ((K + 3) / 4);
  int64_t pctas = (bytes + 255) / 256;
  if (pctas > static_cast<int64_t>(sms) * 32) pctas = static_cast<int64_t>(sms) * 32;
  bl::k_ternarise_pack2<<<static_cast<int>(pctas), 256, 0, s>>>(W, N, K, gamma, packed);
  return launch_status();
}

}  // extern "C"

// ------------------------------------------------------------ allocation-free packing
//
// Scratch for bitlinear_pack_weights_noalloc: the 256 exponent buckets of
// the exact |W| sum (2048 bytes), in a file-scope device array instead of a
// caller buffer.  Every GPU that loads the library holds one copy until the
// process exits.  In host code the array's name is only a host-side stand-in
// for the symbol, so its device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
namespace {

static __device__ __align__(256) unsigned long long g_pack_scratch[bl::kBuckets];

unsigned long long* g_pack_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_pack_scratch_mu;

bl_status pack_scratch_address(unsigned long long** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_pack_scratch_mu);
  if (!g_pack_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pack_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return BL_ERR_CUDA;
    }
    g_pack_scratch_ptr[dev] = static_cast<unsigned long long*>(p);
  }
  *out = g_pack_scratch_ptr[dev];
  return BL_OK;
}

}  // namespace

extern "C" {

bl_status bitlinear_pack_weights_noalloc(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                         float* gamma, void* stream) {
  if (!W || !packed || !gamma) return BL_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  // The fixed 2048-byte scratch holds 64-bit bucket sums of 24-bit
  // mantissas: exact for fewer than 2^40 weights.
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  unsigned long long* buckets = nullptr;
  if ((st = pack_scratch_address(&buckets)) != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  // The shared array keeps the previous call's sums: clear it first.
  bl::k_zero_u64<<<1, 256, 0, s>>>(buckets, bl::kBuckets);
  if ((st = launch_status()) != BL_OK) return st;
  const int64_t count = N * K;
  int64_t ctas = (count / 4 + 255) / 256;
  if (ctas > static_cast<int64_t>(sms) * 8) ctas = static_cast<int64_t>(sms) * 8;
  if (ctas < 1) ctas = 1;
  bl::k_absmean_buckets<<<static_cast<int>(ctas), 256, 0, s>>>(W, count, buckets);
  if ((st = launch_status()) != BL_OK) return st;
  bl::k_gamma_finalize<<<1, 32, 0, s>>>(buckets, count, gamma);
  if ((st = launch_status()) != BL_OK) return st;
  const int64_t bytes = N * ((K + 3) / 4);
  int64_t pctas = (bytes + 255) / 256;
  if (pctas > static_cast<int64_t>(sms) * 32) pctas = static_cast<int64_t>(sms) * 32;
  bl::k_ternarise_pack2<<<static_cast<int>(pctas), 256, 0, s>>>(W, N, K, gamma, packed);
  return launch_status();
}

bl_status bitlinear_quant_act(const void* x, bl_dtype xdt, int64_t M, int64_t K, int8_t* xq,
                              float* eta, int32_t* xsum, void* stream) {
  if (M < 0 || K < 1) return BL_ERR_INVALID_ARG;
  if (xdt != BL_F32 && xdt != BL_BF16) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;  // empty batch: the buffers may be NULL
  if (!x || !xq || !eta || !xsum) return BL_ERR_INVALID_ARG;
  if (!aligned(x, xdt == BL_F32 ? 4 : 2) || !aligned(eta, 4) || !aligned(xsum, 4))
    return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  int64_t ctas = M;
  if (ctas > static_cast<int64_t>(sms) * 64) ctas = static_cast<int64_t>(sms) * 64;
  if (xdt == BL_BF16) {
    const int vec = (K % 8 == 0) && aligned(x, 16) && aligned(xq, 8);
    static int carve_done[kMaxDevices] = {0};
    if (!ensure_smem(bl::k_quant_act<__nv_bfloat16>, 0, carve_done)) return BL_ERR_CUDA;
    return launch_pdl(bl::k_quant_act<__nv_bfloat16>, dim3(static_cast<unsigned>(ctas)), dim3(256),
                      0, s, static_cast<const __nv_bfloat16*>(x), M, K, vec, xq, eta, xsum);
  }
  const int vec = (K % 4 == 0) && aligned(x, 16) && aligned(xq, 4);
  static int carve_done_f[kMaxDevices] = {0};
  if (!ensure_smem(bl::k_quant_act<float>, 0, carve_done_f)) return BL_ERR_CUDA;
  return launch_pdl(bl::k_quant_act<float>, dim3(static_cast<unsigned>(ctas)), dim3(256), 0, s,
                    static_cast<const float*>(x), M, K, vec, xq, eta, xsum);
}

bl_status bitlinear_forward(const int8_t* xq, const float* eta, const int32_t* xsum, int64_t M,
                            int64_t K, const uint8_t* packed, const float* gamma, int64_t N,
                            void* y, bl_dtype ydt, int32_t* y_int, void* stream) {
  return forward_impl(xq, eta, xsum, M, K, packed, gamma, N, y, ydt, y_int, BL_PATH_AUTO, 0u, stream);
}

bl_status bitlinear_forward_path(const int8_t* xq, const float* eta, const int32_t* xsum,
                                 int64_t M, int64_t K, const uint8_t* packed, const float* gamma,
                                 int64_t N, void* y, bl_dtype ydt, int32_t* y_int, bl_path path,
                                 unsigned flags, void* stream) {
  return forward_impl(xq, eta, xsum, M, K, packed, gamma, N, y, ydt, y_int, path, flags, stream);
}

bl_status bitlinear_linear(const void* x, bl_dtype xdt, int64_t M, int64_t K, const uint8_t* packed,
                           const float* gamma, int64_t N, void* y, bl_dtype ydt, int8_t* xq,
                           float* eta, int32_t* xsum, int32_t* y_int, unsigned flags,
                           void* stream) {
  if (M < 0 || K < 1 || N < 1) return BL_ERR_INVALID_ARG;
  if ((xdt != BL_F32 && xdt != BL_BF16) || (ydt != BL_F32 && ydt != BL_BF16))
    return BL_ERR_INVALID_ARG;
  if (!packed || !gamma) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!x || !y) return BL_ERR_INVALID_ARG;
  if (127 * K >= (int64_t{1} << 31)) return BL_ERR_UNSUPPORTED;
  const bool fused = decode_ok(M, K) && xdt == BL_BF16 &&
                     aligned(x, 16) && aligned(packed, 16) && aligned(y, 16) &&
                     (!y_int || aligned(y_int, 16)) && (!xq || aligned(xq, 16)) &&
                     (!eta || aligned(eta, 4)) && (!xsum || aligned(xsum, 4)) && N <= INT32_MAX / 2;
  if (!fused) {
    // Two kernels: quantise into the caller's x~ buffers, then accumulate.
    if (!xq || !eta || !xsum) return BL_ERR_INVALID_ARG;
    bl_status st = bitlinear_quant_act(x, xdt, M, K, xq, eta, xsum, stream);
    if (st != BL_OK) return st;
    return forward_impl(xq, eta, xsum, M, K, packed, gamma, N, y, ydt, y_int, BL_PATH_AUTO, flags,
                        stream);
  }
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  bl::DecodeArgs a = {};
  a.x = x; a.M = (int)M; a.K = (int)K; a.N = (int)N;
  a.packed = packed; a.gamma = gamma; a.y = y; a.y_int = y_int;
  a.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
  a.xq_out = xq; a.eta_out = eta; a.xsum_out = xsum;
  const cudaStream_t s = as_stream(stream);
  return ydt == BL_F32 ? launch_decode<__nv_bfloat16, float>(a, sms, s)
                       : launch_decode<__nv_bfloat16, __nv_bfloat16>(a, sms, s);
}

bl_path bitlinear_select_path(int64_t M, int64_t K, int64_t N, const void* xq, const void* packed,
                              const void* y, const void* y_int) {
  (void)N;
  return select_path(M, K, xq, packed, y, y_int);
}

bl_status bitlinear_device_error(int32_t* code, void* stream) {
  if (!code) return BL_ERR_INVALID_ARG;
  const cudaStream_t s = as_stream(stream);
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, bl::g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbolAsync(bl::g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  *code = v == 0 ? BL_OK : static_cast<int32_t>(v);
  return BL_OK;
}

}  // extern "C"

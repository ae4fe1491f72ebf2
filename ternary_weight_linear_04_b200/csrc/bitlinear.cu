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

#include "bitlinear.h"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "pack.cuh"
#include "quant.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kGemvMaxM = 8;          // largest token count the CUDA-core kernel takes
constexpr int kGemvAutoMaxM = 4;      // auto dispatch: above this, tensor cores
constexpr int64_t kGemvMaxSmem = 200 * 1024;

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bl_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
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

// Raise a kernel's dynamic shared memory limit once per device.
template <typename Kern>
bool ensure_smem(Kern kern, size_t bytes, int* done_flags) {
  if (bytes <= 48 * 1024) return true;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (done_flags[dev] >= static_cast<int>(bytes)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return false;
  done_flags[dev] = static_cast<int>(bytes);
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

template <int MT, int R, typename OutT>
bl_status launch_gemv_swar(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                           const uint8_t* packed, const float* gamma, int N, void* y,
                           int32_t* y_int, int sms, cudaStream_t st) {
  static int smem_done[kMaxDevices] = {0};
  const size_t smem = static_cast<size_t>(MT) * K;
  auto kern = bl::k_gemv_swar<MT, R, OutT>;
  if (!ensure_smem(kern, smem, smem_done)) return BL_ERR_CUDA;
  const int warps_per_cta = 8;
  int64_t ctas = (static_cast<int64_t>(N) + warps_per_cta * R - 1) / (warps_per_cta * R);
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  if (ctas > cap) ctas = cap;
  kern<<<static_cast<int>(ctas), 256, smem, st>>>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int);
  return launch_status();
}

template <int MT, typename OutT>
bl_status gemv_pick_r(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                      const uint8_t* packed, const float* gamma, int N, void* y, int32_t* y_int,
                      int sms, cudaStream_t st) {
  // Enough warp tasks to fill every SM twice over with 8-warp CTAs.
  const int64_t want = static_cast<int64_t>(sms) * 16;
  if (N / 4 >= want)
    return launch_gemv_swar<MT, 4, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
  if (N / 2 >= want)
    return launch_gemv_swar<MT, 2, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
  return launch_gemv_swar<MT, 1, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
}

template <typename OutT>
bl_status launch_gemv(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                      const uint8_t* packed, const float* gamma, int N, void* y, int32_t* y_int,
                      int sms, cudaStream_t st) {
  if (M <= 1) return gemv_pick_r<1, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
  if (M <= 2) return gemv_pick_r<2, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
  if (M <= 4) return gemv_pick_r<4, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
  return gemv_pick_r<8, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, st);
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
    bl::k_gemv_generic<OutT><<<grid, 256, 0, st>>>(xq + m_off * K, eta + m_off, M - m_off, K,
                                                    packed, gamma, N,
                                                    static_cast<char*>(y) + m_off * N * sizeof(OutT),
                                                    y_int ? y_int + m_off * N : nullptr);
    const bl_status s = launch_status();
    if (s != BL_OK) return s;
  }
  return BL_OK;
}

template <int BM, typename OutT>
bl_status launch_tc_bm(const int8_t* xq, const float* eta, int M, int K, const uint8_t* packed,
                       const float* gamma, int N, void* y, int32_t* y_int, cudaStream_t st) {
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
  kern<<<grid, 192, Cfg::kSmem, st>>>(tm_x, tm_w, eta, gamma, M, K, N, y, y_int);
  return launch_status();
}

template <typename OutT>
bl_status launch_tc(const int8_t* xq, const float* eta, int M, int K, const uint8_t* packed,
                    const float* gamma, int N, void* y, int32_t* y_int, cudaStream_t st) {
  if (M <= 16) return launch_tc_bm<16, OutT>(xq, eta, M, K, packed, gamma, N, y, y_int, st);
  if (M <= 32) return launch_tc_bm<32, OutT>(xq, eta, M, K, packed, gamma, N, y, y_int, st);
  if (M <= 64) return launch_tc_bm<64, OutT>(xq, eta, M, K, packed, gamma, N, y, y_int, st);
  if (M <= 128) return launch_tc_bm<128, OutT>(xq, eta, M, K, packed, gamma, N, y, y_int, st);
  return launch_tc_bm<256, OutT>(xq, eta, M, K, packed, gamma, N, y, y_int, st);
}

bool fast_layout_ok(int64_t K, const void* xq, const void* packed, const void* y, const void* y_int) {
  return (K % 64 == 0) && aligned(xq, 16) && aligned(packed, 16) && aligned(y, 16) &&
         (y_int == nullptr || aligned(y_int, 16));
}

bl_path select_path(int64_t M, int64_t K, const void* xq, const void* packed, const void* y,
                    const void* y_int) {
  if (!fast_layout_ok(K, xq, packed, y, y_int) || K > (1 << 30)) return BL_PATH_GENERIC;
  if (M <= kGemvAutoMaxM && static_cast<int64_t>(M) * K <= kGemvMaxSmem) return BL_PATH_GEMV;
  return BL_PATH_TCGEN05;
}

bl_status forward_impl(const int8_t* xq, const float* eta, const int32_t* xsum, int64_t M,
                       int64_t K, const uint8_t* packed, const float* gamma, int64_t N, void* y,
                       bl_dtype ydt, int32_t* y_int, bl_path path, void* stream) {
  if (!xq || !eta || !xsum || !packed || !gamma || !y) return BL_ERR_INVALID_ARG;
  if (M < 0 || K < 1 || N < 1) return BL_ERR_INVALID_ARG;
  if (ydt != BL_F32 && ydt != BL_BF16) return BL_ERR_INVALID_ARG;
  if (path < BL_PATH_AUTO || path > BL_PATH_GENERIC) return BL_ERR_INVALID_ARG;
  if (127 * K >= (int64_t{1} << 31)) return BL_ERR_UNSUPPORTED;
  if (!aligned(eta, 4) || !aligned(xsum, 4) || !aligned(gamma, 4) ||
      (y_int && !aligned(y_int, 4)) || !aligned(y, ydt == BL_F32 ? 4 : 2))
    return BL_ERR_ALIGNMENT;
  if (M == 0) return BL_OK;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  if (path == BL_PATH_AUTO) path = select_path(M, K, xq, packed, y, y_int);
  const cudaStream_t s = as_stream(stream);
  if (path == BL_PATH_GEMV) {
    if (!fast_layout_ok(K, xq, packed, y, y_int) || M > kGemvMaxM ||
        M * K > kGemvMaxSmem || N > INT32_MAX / 2)
      return BL_ERR_UNSUPPORTED;
    return ydt == BL_F32
               ? launch_gemv<float>(xq, eta, xsum, (int)M, (int)K, packed, gamma, (int)N, y, y_int, sms, s)
               : launch_gemv<__nv_bfloat16>(xq, eta, xsum, (int)M, (int)K, packed, gamma, (int)N, y,
                                            y_int, sms, s);
  }
  if (path == BL_PATH_TCGEN05) {
    if (!fast_layout_ok(K, xq, packed, y, y_int) || M > INT32_MAX / 2 || N > INT32_MAX / 2 ||
        K > (1 << 30))
      return BL_ERR_UNSUPPORTED;
    return ydt == BL_F32
               ? launch_tc<float>(xq, eta, (int)M, (int)K, packed, gamma, (int)N, y, y_int, s)
               : launch_tc<__nv_bfloat16>(xq, eta, (int)M, (int)K, packed, gamma, (int)N, y, y_int, s);
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

bl_status bitlinear_quant_act(const void* x, bl_dtype xdt, int64_t M, int64_t K, int8_t* xq,
                              float* eta, int32_t* xsum, void* stream) {
  if (!x || !xq || !eta || !xsum) return BL_ERR_INVALID_ARG;
  if (M < 0 || K < 1) return BL_ERR_INVALID_ARG;
  if (xdt != BL_F32 && xdt != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!aligned(x, xdt == BL_F32 ? 4 : 2) || !aligned(eta, 4) || !aligned(xsum, 4))
    return BL_ERR_ALIGNMENT;
  if (M == 0) return BL_OK;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  int64_t ctas = M;
  if (ctas > static_cast<int64_t>(sms) * 64) ctas = static_cast<int64_t>(sms) * 64;
  if (xdt == BL_BF16) {
    const int vec = (K % 8 == 0) && aligned(x, 16) && aligned(xq, 8);
    bl::k_quant_act<__nv_bfloat16><<<static_cast<int>(ctas), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), M, K, vec, xq, eta, xsum);
  } else {
    const int vec = (K % 4 == 0) && aligned(x, 16) && aligned(xq, 4);
    bl::k_quant_act<float><<<static_cast<int>(ctas), 256, 0, s>>>(static_cast<const float*>(x), M,
                                                                   K, vec, xq, eta, xsum);
  }
  return launch_status();
}

bl_status bitlinear_forward(const int8_t* xq, const float* eta, const int32_t* xsum, int64_t M,
                            int64_t K, const uint8_t* packed, const float* gamma, int64_t N,
                            void* y, bl_dtype ydt, int32_t* y_int, void* stream) {
  return forward_impl(xq, eta, xsum, M, K, packed, gamma, N, y, ydt, y_int, BL_PATH_AUTO, stream);
}

bl_status bitlinear_forward_path(const int8_t* xq, const float* eta, const int32_t* xsum,
                                 int64_t M, int64_t K, const uint8_t* packed, const float* gamma,
                                 int64_t N, void* y, bl_dtype ydt, int32_t* y_int, bl_path path,
                                 void* stream) {
  return forward_impl(xq, eta, xsum, M, K, packed, gamma, N, y, ydt, y_int, path, stream);
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

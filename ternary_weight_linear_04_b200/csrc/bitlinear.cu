// bitlinear.cu -- C ABI of the BitLinear library: argument checks, kernel
// selection and launches.  Declarations and the contract of every entry
// point are in include/bitlinear.h.  All kernels live in this one
// translation unit (the .cuh files) so the device error word needs no
// relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <utility>

#include "bitlinear.h"
#include "common.cuh"
#include "decode.cuh"
#include "decode_reg.cuh"
#include "decode_mma.cuh"
#include "base3.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "pack.cuh"
#include "quant.cuh"
#include "rmsnorm_rows.cuh"
#include "rmsnorm.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kGemvMaxM = 4;  // largest token count the CUDA-core decode kernel takes
constexpr int kFusedMaxM = 2;  // largest token count bitlinear_linear fuses into one kernel

// Tokens rounded up to the decode kernel's widths (1, 2, 4).
inline int decode_mt(int64_t M) { return M <= 1 ? 1 : (M <= 2 ? 2 : 4); }

// Whether the decode kernel takes (M, K): K % 64 == 0, M <= 4 and
// K * MT <= 131072 (the quantised activations of all MT tokens sit in
// shared memory, K * MT bytes, beside at least one ring stage).
inline bool decode_ok(int64_t M, int64_t K) {
  return M >= 1 && M <= kGemvMaxM && K >= 64 && K % 64 == 0 && K * decode_mt(M) <= 131072;
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

// The same, as thread-block clusters of `cluster_z` CTAs along grid z.
template <typename... KArgs, typename... Args>
bl_status launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, unsigned cluster_z, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = cluster_z;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
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
  // The default limit (48 KB) covers static and dynamic shared memory
  // together: raise the dynamic limit whenever the sum would pass it.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  if (bytes + fa.sharedSizeBytes > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess) {
    (void)cudaGetLastError();  // do not leave the error for the next launch check
    return false;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
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
// range of rows, small enough that the next kernel's CTA fits beside it
// under programmatic dependent launch.
//
// The shape of the work inside a CTA -- G warps per team splitting K, RB
// rows per block -- is picked here by a small cost model in SM cycles: the
// largest of (instructions / 4 issue slots, dp4a / 2 per cycle, shared
// memory wavefronts, and 2 x one warp's own instruction stream), with the
// padding words (32*G*nwj >= K/16) and padding rows (blocks of RB) counted.
// When the CTA's rows do not fit the ring (the weights stream while the
// kernel runs), the stages must also keep enough copies in flight and
// enough warps busy: a stage holds whole blocks, only the teams owning
// them work on it, and `stages` stages cover the load latency.
struct DecGeom {
  int G = 1, teams = 16, nwj = 1, RB = 1;
  int rows_per_cta = 1, grid = 1, bpc = 1, stages = 1, x_staged = 0;
  size_t smem = 0;
};

constexpr size_t kDecTwoCtaSmem = 113 * 1024;  // two CTAs per SM (228 KB less 1 KB each)
constexpr size_t kDecMaxSmem = 227 * 1024;
constexpr int64_t kDecRingBytes = 64 * 1024;
constexpr int64_t kDecStageTarget = 32 * 1024;
constexpr double kDecLoadLatency = 2000.0;  // cycles from a stage's copy request to its arrival

inline bool rb_allowed(int MT, int RB) { return RB * MT <= 16; }

// Shape forced by bitlinear_set_decode_shape (0 = chosen by the model).
std::atomic<int> g_force_G{0}, g_force_RB{0};
// bitlinear_set_decode_reg: 0 turns the register-resident kernels off (one
// token fused with the quantiser; 2..8 tokens with x~ given).
std::atomic<int> g_decode_reg{1};

bool decode_geometry(int MT, int64_t M, int64_t K, int64_t N, int sms, int64_t xelem,
                     DecGeom* out) {
  const int64_t NW = K / 16, P = K / 4;
  const int fG = g_force_G.load(std::memory_order_relaxed);
  const int fRB = g_force_RB.load(std::memory_order_relaxed);
  int64_t grid = N < sms ? N : sms;
  int64_t rpc = (N + grid - 1) / grid;
  grid = (N + rpc - 1) / rpc;
  double best = 1e30;
  bool found = false;
  for (int RB = 1; RB <= 16; RB *= 2) {
    if (!rb_allowed(MT, RB) || (fRB && RB != fRB)) continue;
    const int V = RB * MT;
    const int alu = V <= 8 ? 5 : 7;
    const int64_t nblocks = (rpc + RB - 1) / RB;
    for (int G = 1; G <= 16; ++G) {
      if (fG && G != fG) continue;
      const int teams = 16 / G;
      if (G > 1 && nblocks > bl::kDecMaxBlocks) continue;
      const int64_t nwj = (NW + 32 * G - 1) / (32 * G);
      const int64_t bpt = (nblocks + teams - 1) / teams;
      // per warp and block: x~ loads, weight loads, plane split, dp4a, loop
      const double per_block = nwj * (MT + RB + alu * RB + 4.0 * V + 3) + 2.0 * V + 8 +
                               (G > 1 ? 10 : 0);
      const double warp_blocks = static_cast<double>(nblocks) * G;
      const double t_issue = warp_blocks * per_block / 4.0;
      const double t_dp4a = warp_blocks * nwj * 4.0 * V / 2.0;
      const double t_lsu = warp_blocks * nwj * (4.0 * MT + RB);
      const double t_warp = 2.0 * bpt * per_block;
      double cost = t_issue;
      if (t_dp4a > cost) cost = t_dp4a;
      if (t_lsu > cost) cost = t_lsu;
      if (t_warp > cost) cost = t_warp;
      // shared memory: slots + ring of at least one block + tail
      const int64_t slots = static_cast<int64_t>(MT) * 32 * G * nwj * 16;
      const int64_t blk = RB * P;
      const int64_t tail = static_cast<int64_t>(sizeof(bl::DecTail));
      if (slots + blk + tail > static_cast<int64_t>(kDecMaxSmem)) continue;
      // streaming: chunks of bpc blocks, `st` of them in flight
      int64_t bpc = kDecStageTarget / blk;
      if (bpc < 1) bpc = 1;
      if (bpc > nblocks) bpc = nblocks;
      const int64_t chunks = (nblocks + bpc - 1) / bpc;
      int64_t ring = static_cast<int64_t>(kDecTwoCtaSmem) - slots - tail;
      if (ring > kDecRingBytes) ring = kDecRingBytes;
      if (ring < bpc * blk) ring = bpc * blk;
      int64_t st = ring / (bpc * blk);
      if (st > bl::kDecMaxStages) st = bl::kDecMaxStages;
      if (st > chunks) st = chunks;
      if (chunks > st) {
        // A stage is refilled only after every warp has passed it, so the
        // chunks go through one after another; a chunk takes as long as its
        // busiest warp (a lone warp issues well below one instruction per
        // cycle: 2.5 cycles per instruction) or the SM's issue slots.
        const double t_chunk_warp = 2.5 * std::ceil(static_cast<double>(bpc) / teams) * per_block;
        const double t_chunk_issue = static_cast<double>(bpc) * G * per_block / 4.0;
        const double t_chunk = t_chunk_warp > t_chunk_issue ? t_chunk_warp : t_chunk_issue;
        const double per_chunk_load = (kDecLoadLatency + t_chunk) / st;
        const double t_stream =
            kDecLoadLatency + chunks * (t_chunk > per_chunk_load ? t_chunk : per_chunk_load);
        if (t_stream > cost) cost = t_stream;
      }
      if (cost < best * 0.999) {
        best = cost;
        found = true;
        out->G = G; out->teams = teams; out->nwj = static_cast<int>(nwj); out->RB = RB;
      }
    }
  }
  if (!found) return false;
  // ring: whole blocks per stage, about kDecStageTarget per stage
  const int64_t blk = out->RB * P;
  const int64_t nblocks = (rpc + out->RB - 1) / out->RB;
  int64_t bpc = kDecStageTarget / blk;
  if (bpc < 1) bpc = 1;
  if (bpc > nblocks) bpc = nblocks;
  const int64_t chunks = (nblocks + bpc - 1) / bpc;
  const int64_t slots = static_cast<int64_t>(MT) * 32 * out->G * out->nwj * 16;
  const int64_t tail = static_cast<int64_t>(sizeof(bl::DecTail));
  const int64_t xbytes = ((M * K * xelem) + 127) & ~int64_t{127};
  int64_t ring = kDecRingBytes;
  // stay within two CTAs per SM when the slots allow it
  if (slots + tail + bpc * blk <= static_cast<int64_t>(kDecTwoCtaSmem) &&
      slots + tail + ring > static_cast<int64_t>(kDecTwoCtaSmem))
    ring = static_cast<int64_t>(kDecTwoCtaSmem) - slots - tail;
  if (slots + tail + ring > static_cast<int64_t>(kDecMaxSmem))
    ring = static_cast<int64_t>(kDecMaxSmem) - slots - tail;
  int64_t stages = ring / (bpc * blk);
  if (stages > bl::kDecMaxStages) stages = bl::kDecMaxStages;
  if (stages > chunks) stages = chunks;
  if (stages < 1) stages = 1;
  size_t smem = static_cast<size_t>(slots + stages * bpc * blk + tail);
  int x_staged = 0;
  const size_t limit = smem <= kDecTwoCtaSmem ? kDecTwoCtaSmem : kDecMaxSmem;
  if (smem + static_cast<size_t>(xbytes) <= limit) {
    smem += static_cast<size_t>(xbytes);
    x_staged = 1;
  }
  if (smem > kDecMaxSmem) return false;
  out->rows_per_cta = static_cast<int>(rpc);
  out->grid = static_cast<int>(grid);
  out->bpc = static_cast<int>(bpc);
  out->stages = static_cast<int>(stages);
  out->x_staged = x_staged;
  out->smem = smem;
  return true;
}

template <int MT, int RB, typename XT, typename OutT>
bl_status launch_decode_rb(const bl::DecodeArgs& a, const DecGeom& g, cudaStream_t st) {
  static int smem_done[kMaxDevices] = {0};
  auto kern = bl::k_decode<MT, RB, XT, OutT>;
  if (!ensure_smem(kern, static_cast<int>(kDecMaxSmem), smem_done)) return BL_ERR_CUDA;
  return launch_pdl(kern, dim3(static_cast<unsigned>(g.grid)), dim3(bl::kDecThreads), g.smem, st,
                    a);
}

template <int MT, typename XT, typename OutT>
bl_status launch_decode_kernel(const bl::DecodeArgs& a0, int sms, cudaStream_t st) {
  constexpr int64_t kXElem = std::is_same<XT, bl::DecNoFuse>::value ? 1 : 2;
  DecGeom g;
  // a group of matrices sharing the activations: shape from the summed rows
  int64_t n_total = a0.N;
  if (a0.nseg > 0) {
    n_total = 0;
    for (int s = 0; s < a0.nseg; ++s) n_total += a0.seg_N[s];
  }
  if (!decode_geometry(MT, a0.M, a0.K, n_total, sms, kXElem, &g)) return BL_ERR_UNSUPPORTED;
  bl::DecodeArgs a = a0;
  if (a0.nseg > 0) {  // whole CTAs per matrix, the same rows per CTA for all of them
    int64_t cta = 0;
    for (int s = 0; s < a0.nseg; ++s) {
      a.seg_cta0[s] = static_cast<int>(cta);
      cta += (a0.seg_N[s] + g.rows_per_cta - 1) / g.rows_per_cta;
    }
    a.seg_cta0[a0.nseg] = static_cast<int>(cta);
    if (cta > 0x7FFFFFFF) return BL_ERR_UNSUPPORTED;
    g.grid = static_cast<int>(cta);
  }
  a.rows_per_cta = g.rows_per_cta;
  a.blocks_per_chunk = g.bpc;
  a.stages = g.stages;
  a.team_warps = g.G;
  a.teams = g.teams;
  a.nwj = g.nwj;
  a.x_staged = g.x_staged;
  switch (g.RB) {
    case 1: return launch_decode_rb<MT, 1, XT, OutT>(a, g, st);
    case 2: return launch_decode_rb<MT, 2, XT, OutT>(a, g, st);
    case 4: return launch_decode_rb<MT, 4, XT, OutT>(a, g, st);
    case 8:
      if constexpr (MT <= 2) return launch_decode_rb<MT, 8, XT, OutT>(a, g, st);
      break;
    case 16:
      if constexpr (MT == 1) return launch_decode_rb<MT, 16, XT, OutT>(a, g, st);
      break;
  }
  return BL_ERR_UNSUPPORTED;
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

// One-token layer with the CTA's weights in registers (decode_reg.cuh):
// 16 warps of RB rows each, NJ 32-bit words per lane and row.  Applies when
// one CTA per SM leaves at most 64 rows per CTA and the weight registers
// (RB * NJ) stay within the 64-register budget; the instantiated word
// counts cover the common layer widths (K <= 512 NJ, the smallest that fits
// is taken; the unused words are predicated off).
struct RegGeom {
  int RB = 0, NJ = 0, rows_per_cta = 0, grid = 0;
};

constexpr int kRegNJ1[] = {2, 4, 7, 8, 12, 16, 17, 24};
constexpr int kRegNJ2[] = {2, 4, 7, 8, 12, 17};
constexpr int kRegNJ4[] = {2, 4, 7, 8};

bool reg_decode_geometry(int64_t K, int64_t N, int sms, RegGeom* g) {
  if (K < 64 || K % 64 != 0 || N < 1 || N > INT32_MAX / 2) return false;
  int64_t grid = N < sms ? N : sms;
  const int64_t rpc = (N + grid - 1) / grid;
  grid = (N + rpc - 1) / rpc;
  const int RB = rpc <= 16 ? 1 : (rpc <= 32 ? 2 : (rpc <= 64 ? 4 : 0));
  if (RB == 0) return false;
  const int64_t need = (K / 16 + 31) / 32;
  const int* list = RB == 1 ? kRegNJ1 : (RB == 2 ? kRegNJ2 : kRegNJ4);
  const int n = RB == 1 ? 8 : (RB == 2 ? 6 : 4);
  int NJ = 0;
  for (int i = 0; i < n && !NJ; ++i)
    if (list[i] >= need) NJ = list[i];
  if (!NJ) return false;
  g->RB = RB;
  g->NJ = NJ;
  g->rows_per_cta = static_cast<int>(rpc);
  g->grid = static_cast<int>(grid);
  return true;
}

template <int RB, int NJ>
bl_status launch_decode_reg_nj(const bl::RegDecodeArgs& a, const RegGeom& g, cudaStream_t st) {
  static int done[kMaxDevices] = {0};
  auto kern = bl::k_decode_reg<RB, NJ>;
  if (!ensure_smem(kern, 0, done)) return BL_ERR_CUDA;
  return launch_pdl(kern, dim3(static_cast<unsigned>(g.grid)), dim3(bl::kRegThreads),
                    static_cast<size_t>(32 * NJ * 16), st, a);
}

bl_status launch_decode_reg(const bl::RegDecodeArgs& a, const RegGeom& g, cudaStream_t st) {
#define BL_REG_CASE(R, J) \
  if (g.RB == R && g.NJ == J) return launch_decode_reg_nj<R, J>(a, g, st);
  BL_REG_CASE(1, 2) BL_REG_CASE(1, 4) BL_REG_CASE(1, 7) BL_REG_CASE(1, 8) BL_REG_CASE(1, 12)
  BL_REG_CASE(1, 16) BL_REG_CASE(1, 17) BL_REG_CASE(1, 24)
  BL_REG_CASE(2, 2) BL_REG_CASE(2, 4) BL_REG_CASE(2, 7) BL_REG_CASE(2, 8) BL_REG_CASE(2, 12)
  BL_REG_CASE(2, 17)
  BL_REG_CASE(4, 2) BL_REG_CASE(4, 4) BL_REG_CASE(4, 7) BL_REG_CASE(4, 8)
#undef BL_REG_CASE
  return BL_ERR_UNSUPPORTED;
}

// Register-resident kernel for 2..8 tokens with x~ given (decode_reg.cuh):
// the rows of the one-token geometry (one CTA per SM, RB rows per warp), MT
// = 2, 4 or 8 token slots (RB * MT <= 32), and the smallest instantiated
// word count NJ that covers K.  The instantiated (MT, RB, NJ) keep weights,
// RB * MT accumulators and two activation slots in registers with no spills
// (ptxas).
struct RegMGeom {
  int MT = 0, RB = 0, NJ = 0, rows_per_cta = 0, grid = 0;
};

constexpr int kRegMNJ1[] = {2, 4, 7, 8, 12, 17, 24};
constexpr int kRegMNJ2[] = {2, 4, 7, 8, 12, 17};
constexpr int kRegMNJ4[] = {2, 4, 7, 8};

bool regm_geometry(int64_t M, int64_t K, int64_t N, int sms, RegMGeom* g) {
  if (M < 2 || M > bl::kRegMultiMaxMT) return false;
  RegGeom g1;
  if (!reg_decode_geometry(K, N, sms, &g1)) return false;
  const int MT = M <= 2 ? 2 : (M <= 4 ? 4 : 8);
  if (g1.RB * MT > 32) return false;
  const int64_t need = (K / 16 + 31) / 32;
  const int* list = g1.RB == 1 ? kRegMNJ1 : (g1.RB == 2 ? kRegMNJ2 : kRegMNJ4);
  const int n = g1.RB == 1 ? 7 : (g1.RB == 2 ? 6 : 4);
  int NJ = 0;
  for (int i = 0; i < n && !NJ; ++i)
    if (list[i] >= need) NJ = list[i];
  if (!NJ) return false;
  g->MT = MT;
  g->RB = g1.RB;
  g->NJ = NJ;
  g->rows_per_cta = g1.rows_per_cta;
  g->grid = g1.grid;
  return true;
}

template <int MT, int RB, int NJ, bool FUSE>
bl_status launch_decode_regm_nj(const bl::RegMultiArgs& a, const RegMGeom& g, cudaStream_t st) {
  static int done[kMaxDevices] = {0};
  auto kern = bl::k_decode_regm<MT, RB, NJ, FUSE>;
  const size_t smem = static_cast<size_t>(MT) * 32 * NJ * 16;
  if (!ensure_smem(kern, smem, done)) return BL_ERR_CUDA;
  return launch_pdl(kern, dim3(static_cast<unsigned>(g.grid)), dim3(bl::kRegThreads), smem, st, a);
}

// fuse: the CTA quantises bf16 x itself (bitlinear_linear, two tokens);
// otherwise x~ is given.
bl_status launch_decode_regm(const bl::RegMultiArgs& a, const RegMGeom& g, bool fuse, cudaStream_t st) {
#define BL_REGM_CASE(T, R, J)                                                        \
  if (g.MT == T && g.RB == R && g.NJ == J) {                                         \
    if constexpr (T == 2)                                                            \
      if (fuse) return launch_decode_regm_nj<T, R, J, true>(a, g, st);               \
    return fuse ? BL_ERR_UNSUPPORTED : launch_decode_regm_nj<T, R, J, false>(a, g, st); \
  }
#define BL_REGM_MT(T)                                                                              \
  BL_REGM_CASE(T, 1, 2) BL_REGM_CASE(T, 1, 4) BL_REGM_CASE(T, 1, 7) BL_REGM_CASE(T, 1, 8)          \
  BL_REGM_CASE(T, 1, 12) BL_REGM_CASE(T, 1, 17) BL_REGM_CASE(T, 1, 24)                             \
  BL_REGM_CASE(T, 2, 2) BL_REGM_CASE(T, 2, 4) BL_REGM_CASE(T, 2, 7) BL_REGM_CASE(T, 2, 8)          \
  BL_REGM_CASE(T, 2, 12) BL_REGM_CASE(T, 2, 17)                                                    \
  BL_REGM_CASE(T, 4, 2) BL_REGM_CASE(T, 4, 4) BL_REGM_CASE(T, 4, 7) BL_REGM_CASE(T, 4, 8)
  BL_REGM_MT(2)
  BL_REGM_MT(4)
  BL_REGM_MT(8)
#undef BL_REGM_MT
#undef BL_REGM_CASE
  return BL_ERR_UNSUPPORTED;
}

// Warp-MMA decode kernel for 9..16 tokens with x~ given (decode_mma.cuh):
// the rows of the one-token geometry (one CTA per SM), RBK blocks of 16
// rows, KP = 16 / RBK parts of K per block, NS steps of 64 K per warp (the
// smallest instantiated value that covers K), 8, 16 or 32 token slots, and
// the activation slots plus partial tiles within the shared memory of one CTA.
struct MmaGeom {
  int NT8 = 0, RBK = 0, NS = 0, rows_per_cta = 0, grid = 0;
  size_t smem = 0;
};

constexpr int kMmaNS[] = {4, 9, 13, 17, 24};
std::atomic<int> g_decode_mma{1};  // bitlinear_set_decode_mma

bool mma_geometry(int64_t M, int64_t K, int64_t N, int sms, MmaGeom* g) {
  if (M <= bl::kRegMultiMaxMT || M > bl::kMmaMaxTokens) return false;
  if (K < 64 || K % 64 != 0 || N < 1 || N > INT32_MAX / 2 || sms < 1) return false;
  // one CTA per SM, the rows split evenly (at most 64 per CTA)
  int64_t grid = N < sms ? N : sms;
  const int64_t rpc = (N + grid - 1) / grid;
  grid = (N + rpc - 1) / rpc;
  if (rpc > 64) return false;
  RegGeom g1;
  g1.rows_per_cta = static_cast<int>(rpc);
  g1.grid = static_cast<int>(grid);
  const int rbk = g1.rows_per_cta <= 16 ? 1 : (g1.rows_per_cta <= 32 ? 2 : 4);
  const int64_t need = (K / 64 + (16 / rbk) - 1) / (16 / rbk);
  int ns = 0;
  for (int v : kMmaNS)
    if (!ns && v >= need) ns = v;
  if (!ns) return false;
  const int nt8 = 2;
  const size_t smem = bl::mma_decode_smem(nt8, rbk, static_cast<int>(K));
  if (smem + 1024 > kDecMaxSmem) return false;
  g->NT8 = nt8;
  g->RBK = rbk;
  g->NS = ns;
  g->rows_per_cta = g1.rows_per_cta;
  g->grid = g1.grid;
  g->smem = smem;
  return true;
}

template <int NT8, int RBK, int NS>
bl_status launch_decode_mma_ns(const bl::MmaDecodeArgs& a, const MmaGeom& g, cudaStream_t st) {
  static int done[kMaxDevices] = {0};
  auto kern = bl::k_decode_mma<NT8, RBK, NS>;
  if (!ensure_smem(kern, g.smem, done)) return BL_ERR_CUDA;
  return launch_pdl(kern, dim3(static_cast<unsigned>(g.grid)), dim3(bl::kMmaThreads), g.smem, st, a);
}

bl_status launch_decode_mma(const bl::MmaDecodeArgs& a, const MmaGeom& g, cudaStream_t st) {
#define BL_MMA_CASE(T, R, S) \
  if (g.NT8 == T && g.RBK == R && g.NS == S) return launch_decode_mma_ns<T, R, S>(a, g, st);
#define BL_MMA_R(T, R) \
  BL_MMA_CASE(T, R, 4) BL_MMA_CASE(T, R, 9) BL_MMA_CASE(T, R, 13) BL_MMA_CASE(T, R, 17) BL_MMA_CASE(T, R, 24)
#define BL_MMA_T(T) BL_MMA_R(T, 1) BL_MMA_R(T, 2) BL_MMA_R(T, 4)
  BL_MMA_T(2)
#undef BL_MMA_T
#undef BL_MMA_R
#undef BL_MMA_CASE
  return BL_ERR_UNSUPPORTED;
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

// Base-3 accumulate: shared memory of one launch (table, activation slots
// of mt tokens, per-token scale and sum), and the launch itself.  The
// attribute cache is per kernel instantiation (each k_gemv3<MT, OutT> has
// its own static flags), so every instantiation gets its own raised
// shared-memory limit and carveout.
inline int64_t g3_smem(int mt, int64_t S) { return 2048 + static_cast<int64_t>(mt) * S * 8 + 64; }

template <int MT, typename OutT>
bl_status launch_gemv3(const bl::G3Launch& L, unsigned grid, cudaStream_t st) {
  static int done[kMaxDevices] = {0};
  auto kern = bl::k_gemv3<MT, OutT>;
  const size_t smem = static_cast<size_t>(g3_smem(MT, L.S));
  if (!ensure_smem(kern, smem, done)) return BL_ERR_CUDA;
  return launch_pdl(kern, dim3(grid), dim3(32 * bl::kG3Warps), smem, st, L.xq, L.eta, L.xsum, L.M,
                    L.K, L.S, L.packed3, L.gamma, L.N, L.y, L.y_int);
}

// K split of the tensor-core kernel: when the output tiles cannot fill the
// GPU (few tokens), CTAs split K in clusters of up to 8 and add their
// partial tiles in distributed shared memory.  floor(SMs / tiles) splits
// (the whole grid in one wave of one CTA per SM; measured faster than
// filling both CTA slots of the small token tiles), at least two K tiles of
// 128 per CTA, and no more partial tiles than CTA 0's stage memory holds.
std::atomic<int> g_force_split{0};

template <int BM>
int tc_split(int64_t tiles, int64_t K, int sms) {
  const int64_t KT = (K + bl::kTcBK - 1) / bl::kTcBK;
  const int forced = g_force_split.load(std::memory_order_relaxed);
  int64_t ks = forced > 0 ? forced : (tiles >= sms ? 1 : sms / tiles);
  if (forced <= 0 && ks > KT / 2) ks = KT / 2;
  if (ks > KT) ks = KT;
  if (ks > bl::TcCfg<BM>::kMaxSplit) ks = bl::TcCfg<BM>::kMaxSplit;
  if (ks < 1) ks = 1;
  return static_cast<int>(ks);
}

template <int BM, typename OutT>
bl_status launch_tc_bm(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                       const uint8_t* packed, const float* gamma, int N, void* y, int32_t* y_int,
                       int sms, int wstatic, cudaStream_t st) {
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
  const int ks = tc_split<BM>(grid.x * grid.y, K, sms);
  if (ks <= 1)
    return launch_pdl(kern, grid, dim3(bl::kTcThreads), Cfg::kSmem, st, tm_x, tm_w, eta, xsum,
                      gamma, M, K, N, y, y_int, 1, wstatic);
  grid.z = static_cast<unsigned>(ks);
  return launch_pdl_cluster(kern, grid, dim3(bl::kTcThreads), Cfg::kSmem, st,
                            static_cast<unsigned>(ks), tm_x, tm_w, eta, xsum, gamma, M, K, N, y,
                            y_int, ks, wstatic);
}

template <typename OutT>
bl_status launch_tc(const int8_t* xq, const float* eta, const int32_t* xsum, int M, int K,
                    const uint8_t* packed, const float* gamma, int N, void* y, int32_t* y_int,
                    int sms, int ws, cudaStream_t st) {
  if (M <= 16) return launch_tc_bm<16, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, ws, st);
  if (M <= 32) return launch_tc_bm<32, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, ws, st);
  if (M <= 64) return launch_tc_bm<64, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, ws, st);
  if (M <= 128) return launch_tc_bm<128, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, ws, st);
  return launch_tc_bm<256, OutT>(xq, eta, xsum, M, K, packed, gamma, N, y, y_int, sms, ws, st);
}

bool fast_layout_ok(int64_t K, const void* xq, const void* packed, const void* y, const void* y_int) {
  return (K % 64 == 0) && aligned(xq, 16) && aligned(packed, 16) && aligned(y, 16) &&
         (y_int == nullptr || aligned(y_int, 16));
}

// sms < 1: the device is unknown (the register kernel is not considered).
bl_path select_path(int64_t M, int64_t K, int64_t N, int sms, const void* xq, const void* packed,
                    const void* y, const void* y_int) {
  if (!fast_layout_ok(K, xq, packed, y, y_int) || K > (1 << 30)) return BL_PATH_GENERIC;
  if (decode_ok(M, K)) return BL_PATH_GEMV;
  if (sms >= 1 && g_decode_reg.load(std::memory_order_relaxed) != 0 &&
      g_force_G.load(std::memory_order_relaxed) == 0 &&
      g_force_RB.load(std::memory_order_relaxed) == 0) {
    MmaGeom gm;
    if (g_decode_mma.load(std::memory_order_relaxed) != 0 && mma_geometry(M, K, N, sms, &gm))
      return BL_PATH_GEMV;  // 9..16 tokens: the warp-MMA kernel
    RegMGeom mg;
    if (M <= bl::kRegMultiMaxMT && regm_geometry(M, K, N, sms, &mg))
      return BL_PATH_GEMV;  // 5..8 tokens: the register-resident kernel
  }
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
  if (path == BL_PATH_AUTO) path = select_path(M, K, N, sms, xq, packed, y, y_int);
  const cudaStream_t s = as_stream(stream);
  if (path == BL_PATH_GEMV) {
    if (!fast_layout_ok(K, xq, packed, y, y_int) || N > INT32_MAX / 2) return BL_ERR_UNSUPPORTED;
    // 2..8 tokens: the register-resident kernel when the CTA's share fits
    // (and no shape is forced for the shared-memory kernel, which takes up
    // to 4 tokens).
    const bool reg_on = M >= 2 && g_decode_reg.load(std::memory_order_relaxed) != 0 &&
                        g_force_G.load(std::memory_order_relaxed) == 0 &&
                        g_force_RB.load(std::memory_order_relaxed) == 0;
    MmaGeom gm;
    if (reg_on && g_decode_mma.load(std::memory_order_relaxed) != 0 && mma_geometry(M, K, N, sms, &gm)) {
      bl::MmaDecodeArgs r = {};
      r.xq = xq; r.eta = eta; r.xsum = xsum;
      r.M = static_cast<int>(M); r.K = static_cast<int>(K); r.N = static_cast<int>(N);
      r.packed = packed; r.gamma = gamma; r.y = y;
      r.y_bf16 = ydt == BL_BF16 ? 1 : 0;
      r.y_int = y_int;
      r.rows_per_cta = gm.rows_per_cta;
      r.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
      return launch_decode_mma(r, gm, s);
    }
    RegMGeom mg;
    if (reg_on && regm_geometry(M, K, N, sms, &mg)) {
      bl::RegMultiArgs r = {};
      r.xq = xq; r.eta = eta; r.xsum = xsum;
      r.M = static_cast<int>(M); r.K = static_cast<int>(K); r.N = static_cast<int>(N);
      r.packed = packed; r.gamma = gamma; r.y = y;
      r.y_bf16 = ydt == BL_BF16 ? 1 : 0;
      r.y_int = y_int;
      r.rows_per_cta = mg.rows_per_cta;
      r.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
      return launch_decode_regm(r, mg, false, s);
    }
    if (!decode_ok(M, K)) return BL_ERR_UNSUPPORTED;
    bl::DecodeArgs a = {};
    a.x = xq; a.eta = eta; a.xsum = xsum; a.M = (int)M; a.K = (int)K; a.N = (int)N;
    a.packed = packed; a.gamma = gamma; a.y = y; a.y_int = y_int;
    a.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
    return ydt == BL_F32 ? launch_decode<bl::DecNoFuse, float>(a, sms, s)
                         : launch_decode<bl::DecNoFuse, __nv_bfloat16>(a, sms, s);
  }
  if (path == BL_PATH_TCGEN05) {
    const int ws = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
    if (!fast_layout_ok(K, xq, packed, y, y_int) || M > INT32_MAX / 2 || N > INT32_MAX / 2 ||
        K > (1 << 30))
      return BL_ERR_UNSUPPORTED;
    return ydt == BL_F32
               ? launch_tc<float>(xq, eta, xsum, (int)M, (int)K, packed, gamma, (int)N, y, y_int,
                                  sms, ws, s)
               : launch_tc<__nv_bfloat16>(xq, eta, xsum, (int)M, (int)K, packed, gamma, (int)N, y,
                                          y_int, sms, ws, s);
  }
  return ydt == BL_F32
             ? launch_generic<float>(xq, eta, M, K, packed, gamma, N, y, y_int, sms, s)
             : launch_generic<__nv_bfloat16>(xq, eta, M, K, packed, gamma, N, y, y_int, sms, s);
}

template <int NT, int CV>
bl_status launch_quant_bf16_nt(const __nv_bfloat16* x, int64_t M, int64_t K, int8_t* xq, float* eta,
                               int32_t* xsum, dim3 grid, cudaStream_t s) {
  static int done[kMaxDevices] = {0};
  if (!ensure_smem(bl::k_quant_bf16<NT, CV>, 0, done)) return BL_ERR_CUDA;
  return launch_pdl(bl::k_quant_bf16<NT, CV>, grid, dim3(NT), 0, s, x, M, K, xq, eta, xsum);
}

// bf16 rows streamed through shared memory (k_rmsnorm_rows): S row buffers
// per CTA (3, or 2 when three would leave less than two CTAs per SM) and as
// many persistent CTAs per SM as fit in 200 KB of its shared memory and its
// registers, at most 8.
struct RowsGeom {
  int stages = 0, grid = 0;
  size_t smem = 0;
};

bool rows_stream_geometry(int64_t M, int64_t K, int sms, RowsGeom* g) {
  if (M < 1 || K < 8 || K % 8 != 0 || sms < 1) return false;
  const int64_t row = 2 * K;
  const int64_t budget = 200 * 1024;
  int stages = 3;
  int64_t per_sm = budget / (stages * row);
  if (per_sm < 2) {
    stages = 2;
    per_sm = budget / (stages * row);
  }
  if (per_sm < 1) return false;
  if (per_sm > 8) per_sm = 8;
  g->stages = stages;
  g->smem = static_cast<size_t>(stages * row);
  g->grid = static_cast<int>(M < sms * per_sm ? M : sms * per_sm);
  return true;
}

// Launches a row-streaming kernel (k_rmsnorm_rows): persistent, so no more
// CTAs than are resident at once.
template <typename Kern>
bl_status launch_rows_stream(Kern kern, int* done, const __nv_bfloat16* x, int64_t M, int64_t K,
                             int8_t* xq, float* eta, int32_t* xsum, const RowsGeom& g, int sms,
                             cudaStream_t s) {
  if (!ensure_smem(kern, g.smem, done)) return BL_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, bl::kRowsThreads, g.smem) !=
          cudaSuccess ||
      per_sm < 1) {
    (void)cudaGetLastError();
    return BL_ERR_CUDA;
  }
  const int64_t cap = static_cast<int64_t>(sms) * per_sm;
  const int64_t grid = g.grid < cap ? g.grid : cap;
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(bl::kRowsThreads), g.smem, s, x,
                    M, K, g.stages, xq, eta, xsum);
}

// bf16 rows with 16-byte vectors.  A few rows (decode, latency): one
// vector per thread and the fewest threads that cover the row (up to 1024),
// then 1024 threads with four vectors each.  Many rows: four vectors per
// thread and the fewest threads that cover the row (128 threads for
// K <= 4096), longer rows read again past 32768 values.  (Streaming the
// rows through shared memory, as k_rmsnorm_rows does, measured slower
// here: 12.3 against 9.8 us for 2048 x 4096, the per-row block reductions
// of 8 warps outweighing the copies kept in flight.)
bl_status launch_quant_bf16(const __nv_bfloat16* x, int64_t M, int64_t K, int8_t* xq, float* eta,
                            int32_t* xsum, bool wide, dim3 grid, cudaStream_t s) {
  if (wide) {
    if (K <= 1024) return launch_quant_bf16_nt<128, 1>(x, M, K, xq, eta, xsum, grid, s);
    if (K <= 2048) return launch_quant_bf16_nt<256, 1>(x, M, K, xq, eta, xsum, grid, s);
    if (K <= 4096) return launch_quant_bf16_nt<512, 1>(x, M, K, xq, eta, xsum, grid, s);
    if (K <= 8192) return launch_quant_bf16_nt<1024, 1>(x, M, K, xq, eta, xsum, grid, s);
    return launch_quant_bf16_nt<1024, 4>(x, M, K, xq, eta, xsum, grid, s);
  }
  if (K <= 4096) return launch_quant_bf16_nt<128, 4>(x, M, K, xq, eta, xsum, grid, s);
  if (K <= 8192) return launch_quant_bf16_nt<256, 4>(x, M, K, xq, eta, xsum, grid, s);
  if (K <= 16384) return launch_quant_bf16_nt<512, 4>(x, M, K, xq, eta, xsum, grid, s);
  return launch_quant_bf16_nt<1024, 4>(x, M, K, xq, eta, xsum, grid, s);
}

// Workspace of the single-matrix pack: the 256 exponent buckets (2048
// bytes), then the fp64 sum of |W| (8 bytes) and the decision flag (4, +4).
constexpr size_t kPackWorkspaceBytes = bl::kBuckets * 8 + 16;

// gamma of one whole matrix (count = N*K weights) into *gamma: the fp64 sum
// of |W| and its proof (k_absmean_f64, k_gamma_decide); the exact buckets
// (k_absmean_buckets, k_gamma_finalize) run only when the proof fails,
// their CTAs returning at once otherwise.  ws = kPackWorkspaceBytes of
// scratch; everything is cleared first.
bl_status pack_gamma(const float* W, int64_t count, unsigned long long* ws, float* gamma, int sms,
                     cudaStream_t s) {
  unsigned long long* buckets = ws;
  double* acc = reinterpret_cast<double*>(ws + bl::kBuckets);
  int* decided = reinterpret_cast<int*>(ws + bl::kBuckets + 1);
  bl::k_zero_u64<<<1, 256, 0, s>>>(ws, static_cast<int>(kPackWorkspaceBytes / 8));
  bl_status st = launch_status();
  if (st != BL_OK) return st;
  int64_t ctas = (count / 4 + 255) / 256;
  if (ctas > static_cast<int64_t>(sms) * 8) ctas = static_cast<int64_t>(sms) * 8;
  if (ctas < 1) ctas = 1;
  bl::k_absmean_f64<<<static_cast<int>(ctas), 256, 0, s>>>(W, count, acc);
  if ((st = launch_status()) != BL_OK) return st;
  // Tree height: a thread's adds (at most count / threads + 5, whether or
  // not W allows 16-byte loads), 5 butterfly levels, 7 adds over the warps,
  // one atomic add per CTA.
  const int64_t threads = ctas * 256;
  const int64_t h = (count + threads - 1) / threads + 5 + 5 + 7 + ctas;
  bl::k_gamma_decide<<<1, 32, 0, s>>>(acc, count, h, gamma, decided);
  if ((st = launch_status()) != BL_OK) return st;
  bl::k_absmean_buckets<<<static_cast<int>(ctas), 256, 0, s>>>(W, count, buckets, decided);
  if ((st = launch_status()) != BL_OK) return st;
  bl::k_gamma_finalize<<<1, 32, 0, s>>>(buckets, count, gamma, decided);
  return launch_status();
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

bl_status bitlinear_linear_group(const void* x, bl_dtype xdt, int64_t M, int64_t K, int nseg,
                                 const uint8_t* const* packed, const float* const* gamma,
                                 const int64_t* N, void* const* y, bl_dtype ydt, unsigned flags,
                                 void* stream) {
  if (nseg < 1 || nseg > bl::kDecMaxSeg || !packed || !gamma || !N || !y) return BL_ERR_INVALID_ARG;
  if (M < 0 || K < 1) return BL_ERR_INVALID_ARG;
  if ((xdt != BL_F32 && xdt != BL_BF16) || (ydt != BL_F32 && ydt != BL_BF16))
    return BL_ERR_INVALID_ARG;
  for (int s = 0; s < nseg; ++s) {
    if (!packed[s] || !gamma[s] || N[s] < 1) return BL_ERR_INVALID_ARG;
    if (M > 0 && !y[s]) return BL_ERR_INVALID_ARG;
  }
  if (M == 0) return BL_OK;
  if (!x) return BL_ERR_INVALID_ARG;
  if (xdt != BL_BF16 || !decode_ok(M, K)) return BL_ERR_UNSUPPORTED;
  if (!aligned(x, 16)) return BL_ERR_ALIGNMENT;
  for (int s = 0; s < nseg; ++s) {
    if (N[s] > INT32_MAX / 2) return BL_ERR_UNSUPPORTED;
    if (!aligned(packed[s], 16) || !aligned(y[s], 16) || !aligned(gamma[s], 4)) return BL_ERR_ALIGNMENT;
  }
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  bl::DecodeArgs a = {};
  a.x = x; a.M = static_cast<int>(M); a.K = static_cast<int>(K);
  a.N = static_cast<int>(N[0]); a.packed = packed[0]; a.gamma = gamma[0]; a.y = y[0];
  a.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
  a.nseg = nseg;
  for (int s = 0; s < nseg; ++s) {
    a.seg_packed[s] = packed[s];
    a.seg_gamma[s] = gamma[s];
    a.seg_y[s] = y[s];
    a.seg_N[s] = static_cast<int>(N[s]);
  }
  const cudaStream_t cs = as_stream(stream);
  return ydt == BL_F32 ? launch_decode<__nv_bfloat16, float>(a, sms, cs)
                       : launch_decode<__nv_bfloat16, __nv_bfloat16>(a, sms, cs);
}

bl_status bitlinear_decode_shape_for(int64_t M, int64_t K, int64_t N, int fused, int sms,
                                     int32_t* shape) {
  if (!shape || N < 1 || sms < 1) return BL_ERR_INVALID_ARG;
  if (!decode_ok(M, K) || N > INT32_MAX / 2) return BL_ERR_UNSUPPORTED;
  DecGeom g;
  if (!decode_geometry(decode_mt(M), M, K, N, sms, fused ? 2 : 1, &g)) return BL_ERR_UNSUPPORTED;
  shape[0] = g.G;
  shape[1] = g.RB;
  shape[2] = g.teams;
  shape[3] = g.nwj;
  shape[4] = g.rows_per_cta;
  shape[5] = g.grid;
  shape[6] = g.bpc;
  shape[7] = g.stages;
  shape[8] = g.x_staged;
  shape[9] = static_cast<int32_t>(g.smem);
  return BL_OK;
}

bl_status bitlinear_decode_shape(int64_t M, int64_t K, int64_t N, int fused, int32_t* shape) {
  if (!shape || N < 1) return BL_ERR_INVALID_ARG;
  if (!decode_ok(M, K) || N > INT32_MAX / 2) return BL_ERR_UNSUPPORTED;
  int sms = 148;
  const bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  DecGeom g;
  if (!decode_geometry(decode_mt(M), M, K, N, sms, fused ? 2 : 1, &g)) return BL_ERR_UNSUPPORTED;
  shape[0] = g.G;
  shape[1] = g.RB;
  shape[2] = g.teams;
  shape[3] = g.nwj;
  shape[4] = g.rows_per_cta;
  shape[5] = g.grid;
  shape[6] = g.bpc;
  shape[7] = g.stages;
  shape[8] = g.x_staged;
  shape[9] = static_cast<int32_t>(g.smem);
  return BL_OK;
}

bl_status bitlinear_decode_mma_shape(int64_t M, int64_t K, int64_t N, int sms, int32_t* shape) {
  if (!shape || K < 1 || N < 1 || sms < 1) return BL_ERR_INVALID_ARG;
  MmaGeom g;
  if (!mma_geometry(M, K, N, sms, &g)) return BL_ERR_UNSUPPORTED;
  shape[0] = 8 * g.NT8;
  shape[1] = g.RBK;
  shape[2] = 16 / g.RBK;
  shape[3] = g.NS;
  shape[4] = g.rows_per_cta;
  shape[5] = g.grid;
  shape[6] = static_cast<int32_t>(g.smem);
  return BL_OK;
}

bl_status bitlinear_set_decode_mma(int enable) {
  if (enable != 0 && enable != 1) return BL_ERR_INVALID_ARG;
  g_decode_mma.store(enable, std::memory_order_relaxed);
  return BL_OK;
}

bl_status bitlinear_decode_regm_shape(int64_t M, int64_t K, int64_t N, int sms, int32_t* shape) {
  if (!shape || K < 1 || N < 1 || sms < 1) return BL_ERR_INVALID_ARG;
  RegMGeom g;
  if (!regm_geometry(M, K, N, sms, &g)) return BL_ERR_UNSUPPORTED;
  shape[0] = g.MT;
  shape[1] = g.RB;
  shape[2] = g.NJ;
  shape[3] = g.rows_per_cta;
  shape[4] = g.grid;
  return BL_OK;
}

bl_status bitlinear_decode_reg_shape(int64_t K, int64_t N, int sms, int32_t* shape) {
  if (!shape || K < 1 || N < 1 || sms < 1) return BL_ERR_INVALID_ARG;
  RegGeom g;
  if (!reg_decode_geometry(K, N, sms, &g)) return BL_ERR_UNSUPPORTED;
  shape[0] = g.RB;
  shape[1] = g.NJ;
  shape[2] = g.rows_per_cta;
  shape[3] = g.grid;
  return BL_OK;
}

bl_status bitlinear_set_decode_reg(int enable) {
  if (enable != 0 && enable != 1) return BL_ERR_INVALID_ARG;
  g_decode_reg.store(enable, std::memory_order_relaxed);
  return BL_OK;
}

bl_status bitlinear_set_tc_split(int k_split) {
  if (k_split < 0 || k_split > 8) return BL_ERR_INVALID_ARG;
  g_force_split.store(k_split, std::memory_order_relaxed);
  return BL_OK;
}

bl_status bitlinear_set_decode_shape(int team_warps, int rows_per_block) {
  if (team_warps < 0 || team_warps > 16) return BL_ERR_INVALID_ARG;
  if (rows_per_block < 0 || rows_per_block > 16 || (rows_per_block & (rows_per_block - 1)) != 0)
    return BL_ERR_INVALID_ARG;
  g_force_G.store(team_warps, std::memory_order_relaxed);
  g_force_RB.store(rows_per_block, std::memory_order_relaxed);
  return BL_OK;
}

const char* bitlinear_version(void) { return "0.1.0"; }

size_t bitlinear_packed_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 1) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>((K + 3) / 4);
}

size_t bitlinear_pack_workspace_bytes(void) { return kPackWorkspaceBytes; }

bl_status bitlinear_absmean_buckets(const float* W, int64_t N, int64_t K, void* buckets,
                                   void* stream) {
  if (!W || !buckets) return BL_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(buckets, 8)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  auto* b = static_cast<unsigned long long*>(buckets);
  bl::k_zero_u64<<<1, 256, 0, s>>>(b, bl::kBuckets);
  if ((st = launch_status()) != BL_OK) return st;
  const int64_t count = N * K;
  int64_t ctas = (count / 4 + 255) / 256;
  if (ctas > static_cast<int64_t>(sms) * 8) ctas = static_cast<int64_t>(sms) * 8;
  if (ctas < 1) ctas = 1;
  bl::k_absmean_buckets<<<static_cast<int>(ctas), 256, 0, s>>>(W, count, b, nullptr);
  return launch_status();
}

bl_status bitlinear_gamma_from_buckets(const void* buckets, int64_t count, float* gamma,
                                       void* stream) {
  if (!buckets || !gamma || count < 1) return BL_ERR_INVALID_ARG;
  if (count > (int64_t{1} << 40)) return BL_ERR_UNSUPPORTED;  // bucket totals stay below 2^64
  if (!aligned(buckets, 8) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  const bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  bl::k_gamma_finalize<<<1, 32, 0, as_stream(stream)>>>(
      static_cast<const unsigned long long*>(buckets), count, gamma, nullptr);
  return launch_status();
}

bl_status bitlinear_ternarise_pack(const float* W, int64_t N, int64_t K, const float* gamma,
                                   uint8_t* packed, void* stream) {
  if (!W || !gamma || !packed) return BL_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  const bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const int64_t bytes = N * ((K + 3) / 4);
  int64_t pctas = (bytes + 255) / 256;
  if (pctas > static_cast<int64_t>(sms) * 32) pctas = static_cast<int64_t>(sms) * 32;
  bl::k_ternarise_pack2<<<static_cast<int>(pctas), 256, 0, as_stream(stream)>>>(W, N, K, gamma,
                                                                                packed);
  return launch_status();
}

bl_status bitlinear_pack_weights(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                 float* gamma, void* workspace, void* stream) {
  if (!W || !packed || !gamma || !workspace) return BL_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(workspace, 8) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  if ((st = pack_gamma(W, N * K, static_cast<unsigned long long*>(workspace), gamma, sms,
                       as_stream(stream))) != BL_OK)
    return st;
  return bitlinear_ternarise_pack(W, N, K, gamma, packed, stream);
}

bl_status bitlinear_rmsnorm_quant_act(const void* x, bl_dtype xdt, int64_t M, int64_t K,
                                      int8_t* xq, float* eta, int32_t* xsum, void* stream) {
  if (M < 0 || K < 1 || (xdt != BL_F32 && xdt != BL_BF16)) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!x || !xq || !eta || !xsum) return BL_ERR_INVALID_ARG;
  if (xdt != BL_BF16) return BL_ERR_UNSUPPORTED;  // the exact sum of squares needs bf16 inputs
  if (K > (int64_t{1} << 24)) return BL_ERR_UNSUPPORTED;  // keeps xsum within int32
  if (!aligned(x, 2) || !aligned(eta, 4) || !aligned(xsum, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const int vec = (K % 8 == 0 && aligned(x, 16) && aligned(xq, 8)) ? 1 : 0;
  // Rows with 16-byte vectors up to K = 51200: streamed through shared
  // memory, the sum of squares in fp64 with a proof (k_rmsnorm_rows); the
  // rest: one CTA per row, the sum of squares exact (k_rmsnorm_quant).
  RowsGeom g;
  if (vec && rows_stream_geometry(M, K, sms, &g)) {
    static int done_rows[kMaxDevices] = {0};
    return launch_rows_stream(bl::k_rmsnorm_rows, done_rows, static_cast<const __nv_bfloat16*>(x), M, K,
                              xq, eta, xsum, g, sms, as_stream(stream));
  }
  static int carve_done[kMaxDevices] = {0};
  if (!ensure_smem(bl::k_rmsnorm_quant, 0, carve_done)) return BL_ERR_CUDA;
  const int64_t ctas = M < static_cast<int64_t>(sms) * 8 ? M : static_cast<int64_t>(sms) * 8;
  return launch_pdl(bl::k_rmsnorm_quant, dim3(static_cast<unsigned>(ctas)), dim3(256), 0,
                    as_stream(stream), static_cast<const __nv_bfloat16*>(x), M, K, vec, xq, eta,
                    xsum);
}

int64_t bitlinear_packed3_stride(int64_t K) {
  if (K < 1) return 0;
  return 16 * ((((K + 4) / 5) + 15) / 16);
}

bl_status bitlinear_pack_weights3(const float* W, int64_t N, int64_t K, uint8_t* packed3,
                                  float* gamma, void* workspace, void* stream) {
  if (!W || !packed3 || !gamma || !workspace) return BL_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(workspace, 8) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  if ((st = pack_gamma(W, N * K, static_cast<unsigned long long*>(workspace), gamma, sms, s)) != BL_OK)
    return st;
  const int64_t S = bitlinear_packed3_stride(K);
  int64_t pctas = (N * S + 255) / 256;
  if (pctas > static_cast<int64_t>(sms) * 32) pctas = static_cast<int64_t>(sms) * 32;
  bl::k_ternarise_pack3<<<static_cast<int>(pctas), 256, 0, s>>>(W, N, K, S, gamma, packed3);
  return launch_status();
}

bl_status bitlinear_forward3(const int8_t* xq, const float* eta, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* packed3, const float* gamma, int64_t N,
                             void* y, bl_dtype ydt, int32_t* y_int, void* stream) {
  if (M < 0 || K < 1 || N < 1) return BL_ERR_INVALID_ARG;
  if (ydt != BL_F32 && ydt != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!packed3 || !gamma) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!xq || !eta || !xsum || !y) return BL_ERR_INVALID_ARG;
  const int64_t S = bitlinear_packed3_stride(K);
  // shared memory: the 2 KB table + 8-byte activation slots per group of
  // five per token; tokens per launch 4, 2 or 1, the most that fit
  const int64_t limit = static_cast<int64_t>(kDecMaxSmem);
  if (K > (1 << 30) || N > INT32_MAX / 2 || g3_smem(1, S) > limit) return BL_ERR_UNSUPPORTED;
  const int mt_max = g3_smem(4, S) <= limit ? 4 : (g3_smem(2, S) <= limit ? 2 : 1);
  if (!aligned(packed3, 16) || !aligned(eta, 4) || !aligned(xsum, 4) || !aligned(gamma, 4) ||
      (y_int && !aligned(y_int, 4)) || !aligned(y, ydt == BL_F32 ? 4 : 2))
    return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t cs = as_stream(stream);
  const size_t esz = ydt == BL_F32 ? 4 : 2;
  int64_t ctas = (N + bl::kG3Warps * bl::kG3Rows - 1) / (bl::kG3Warps * bl::kG3Rows);
  if (ctas > static_cast<int64_t>(sms) * 8) ctas = static_cast<int64_t>(sms) * 8;
  for (int64_t m0 = 0; m0 < M; m0 += mt_max) {
    const int mc = static_cast<int>(M - m0 < mt_max ? M - m0 : mt_max);
    const int mt = mc <= 1 ? 1 : (mc <= 2 ? 2 : 4);
    const int8_t* xq_m = xq + m0 * K;
    void* y_m = static_cast<char*>(y) + m0 * N * esz;
    int32_t* yi_m = y_int ? y_int + m0 * N : nullptr;
    const bl::G3Launch L = {xq_m, eta + m0, xsum + m0, mc, static_cast<int>(K), static_cast<int>(S),
                            packed3, gamma, static_cast<int>(N), y_m, yi_m};
    const unsigned grid = static_cast<unsigned>(ctas);
    if (ydt == BL_F32)
      st = mt == 1 ? launch_gemv3<1, float>(L, grid, cs)
                   : (mt == 2 ? launch_gemv3<2, float>(L, grid, cs) : launch_gemv3<4, float>(L, grid, cs));
    else
      st = mt == 1 ? launch_gemv3<1, __nv_bfloat16>(L, grid, cs)
                   : (mt == 2 ? launch_gemv3<2, __nv_bfloat16>(L, grid, cs)
                              : launch_gemv3<4, __nv_bfloat16>(L, grid, cs));
    if (st != BL_OK) return st;
  }
  return BL_OK;
}

}  // extern "C"

// ------------------------------------------------------------ allocation-free packing
//
// Scratch for bitlinear_pack_weights_noalloc: the pack workspace (the 256
// exponent buckets of the exact |W| sum, the fp64 sum and its decision flag;
// 2064 bytes), in a file-scope device array instead of a caller buffer.  Every GPU that loads the library holds one copy until the
// process exits.  In host code the array's name is only a host-side stand-in
// for the symbol, so its device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
namespace {

static __device__ __align__(256) unsigned long long g_pack_scratch[kPackWorkspaceBytes / 8];

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
  // The fixed scratch holds 64-bit bucket sums of 24-bit mantissas: exact
  // for up to 2^40 weights.
  if (N > (int64_t{1} << 40) / K) return BL_ERR_UNSUPPORTED;
  if (!aligned(W, 4) || !aligned(gamma, 4)) return BL_ERR_ALIGNMENT;
  int sms = 148;
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  unsigned long long* scratch = nullptr;
  if ((st = pack_scratch_address(&scratch)) != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  const int64_t count = N * K;
  if ((st = pack_gamma(W, count, scratch, gamma, sms, s)) != BL_OK) return st;
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
  // bf16 rows with 16-byte vectors: k_quant_bf16 (launch_quant_bf16).  The
  // rest: a few rows (decode) 1024 threads per row, the whole row in
  // registers for K <= 16384, one read; many rows 256 threads per row.
  const bool wide = M <= 64;
  const dim3 grid(static_cast<unsigned>(ctas));
  if (xdt == BL_BF16) {
    const int vec = (K % 8 == 0) && aligned(x, 16) && aligned(xq, 8);
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    if (vec) return launch_quant_bf16(xb, M, K, xq, eta, xsum, wide, grid, s);
    if (wide) {
      static int done_w[kMaxDevices] = {0};
      if (!ensure_smem(bl::k_quant_act<__nv_bfloat16, 1024>, 0, done_w)) return BL_ERR_CUDA;
      return launch_pdl(bl::k_quant_act<__nv_bfloat16, 1024>, grid, dim3(1024), 0, s, xb, M, K, vec, xq,
                        eta, xsum);
    }
    static int carve_done[kMaxDevices] = {0};
    if (!ensure_smem(bl::k_quant_act<__nv_bfloat16, 256>, 0, carve_done)) return BL_ERR_CUDA;
    return launch_pdl(bl::k_quant_act<__nv_bfloat16, 256>, grid, dim3(256), 0, s, xb, M, K, vec, xq,
                      eta, xsum);
  }
  const int vec = (K % 4 == 0) && aligned(x, 16) && aligned(xq, 4);
  const auto* xf = static_cast<const float*>(x);
  if (wide) {
    static int done_wf[kMaxDevices] = {0};
    if (!ensure_smem(bl::k_quant_act<float, 1024>, 0, done_wf)) return BL_ERR_CUDA;
    return launch_pdl(bl::k_quant_act<float, 1024>, grid, dim3(1024), 0, s, xf, M, K, vec, xq, eta,
                      xsum);
  }
  static int carve_done_f[kMaxDevices] = {0};
  if (!ensure_smem(bl::k_quant_act<float, 256>, 0, carve_done_f)) return BL_ERR_CUDA;
  return launch_pdl(bl::k_quant_act<float, 256>, grid, dim3(256), 0, s, xf, M, K, vec, xq, eta,
                    xsum);
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
  // One fused launch for one or two bf16 tokens (a register-resident kernel
  // when it takes the layer, else the shared-memory kernel); from three
  // tokens on the quantiser kernel, then the accumulate.
  int sms = 148;
  // Two bf16 tokens whose layer the register kernel takes: one fused launch
  // (every CTA quantises both rows itself), x~ / eta / xsum optional.  From
  // three tokens on, quantising every row in every CTA costs more than the
  // separate quantiser launch (decode_3b layer step, fused against two
  // kernels: M = 3 17.1 / 14.7 us, M = 4 18.3 / 15.7 us, M = 8 29.4 / 20.6 us).
  RegMGeom fmg;
  if (M == 2 && xdt == BL_BF16 && device_info(&sms) == BL_OK &&
      g_decode_reg.load(std::memory_order_relaxed) != 0 &&
      g_force_G.load(std::memory_order_relaxed) == 0 &&
      g_force_RB.load(std::memory_order_relaxed) == 0 && aligned(x, 16) && aligned(packed, 16) &&
      aligned(y, 16) && (!y_int || aligned(y_int, 16)) && (!xq || aligned(xq, 16)) &&
      (!eta || aligned(eta, 4)) && (!xsum || aligned(xsum, 4)) &&
      regm_geometry(M, K, N, sms, &fmg)) {
    bl::RegMultiArgs r = {};
    r.x = static_cast<const __nv_bfloat16*>(x);
    r.xq_out = xq; r.eta_out = eta; r.xsum_out = xsum;
    r.M = static_cast<int>(M); r.K = static_cast<int>(K); r.N = static_cast<int>(N);
    r.packed = packed; r.gamma = gamma; r.y = y;
    r.y_bf16 = ydt == BL_BF16 ? 1 : 0;
    r.y_int = y_int;
    r.rows_per_cta = fmg.rows_per_cta;
    r.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
    return launch_decode_regm(r, fmg, true, as_stream(stream));
  }
  const bool fused = M <= kFusedMaxM && decode_ok(M, K) && xdt == BL_BF16 &&
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
  bl_status st = device_info(&sms);
  if (st != BL_OK) return st;
  const cudaStream_t s = as_stream(stream);
  // One token: the register-resident kernel when the CTA's share fits (and
  // no decode shape is forced for the shared-memory kernel).
  RegGeom rg;
  if (M == 1 && g_decode_reg.load(std::memory_order_relaxed) != 0 &&
      g_force_G.load(std::memory_order_relaxed) == 0 &&
      g_force_RB.load(std::memory_order_relaxed) == 0 && reg_decode_geometry(K, N, sms, &rg)) {
    bl::RegDecodeArgs r = {};
    r.x = static_cast<const __nv_bfloat16*>(x);
    r.K = static_cast<int>(K);
    r.N = static_cast<int>(N);
    r.packed = packed;
    r.gamma = gamma;
    r.y = y;
    r.y_bf16 = ydt == BL_BF16 ? 1 : 0;
    r.y_int = y_int;
    r.rows_per_cta = rg.rows_per_cta;
    r.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
    r.xq_out = xq;
    r.eta_out = eta;
    r.xsum_out = xsum;
    return launch_decode_reg(r, rg, s);
  }
  bl::DecodeArgs a = {};
  a.x = x; a.M = (int)M; a.K = (int)K; a.N = (int)N;
  a.packed = packed; a.gamma = gamma; a.y = y; a.y_int = y_int;
  a.weights_static = (flags & BL_FLAG_WEIGHTS_STATIC) ? 1 : 0;
  a.xq_out = xq; a.eta_out = eta; a.xsum_out = xsum;
  return ydt == BL_F32 ? launch_decode<__nv_bfloat16, float>(a, sms, s)
                       : launch_decode<__nv_bfloat16, __nv_bfloat16>(a, sms, s);
}

bl_path bitlinear_select_path(int64_t M, int64_t K, int64_t N, const void* xq, const void* packed,
                              const void* y, const void* y_int) {
  int sms = 0;
  if (device_info(&sms) != BL_OK) {
    (void)cudaGetLastError();
    sms = 0;
  }
  return select_path(M, K, N, sms, xq, packed, y, y_int);
}

#ifdef BL_TEST_HOOKS
// Fault-injection build only (not part of the library's interface): 1 makes
// the tensor-core kernel withhold one barrier arrival, so that its bounded
// wait runs out and the kernel returns with BL_ERR_TIMEOUT recorded; 0 turns
// it off.  Synchronous.
bl_status bitlinear_test_set_fault(int what) {
  if (cudaMemcpyToSymbol(bl::g_test_fault, &what, sizeof(int)) != cudaSuccess) return BL_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}
#endif

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

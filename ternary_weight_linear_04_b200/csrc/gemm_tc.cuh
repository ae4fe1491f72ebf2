// gemm_tc.cuh -- tensor-core accumulate kernel (tcgen05, kind::i8, sm_100a).
//
// When many tokens share each weight the accumulation is a dense int8
// contraction, y_int = x~ . W~^T, so it runs on the 5th-generation tensor
// core: 8-bit x 8-bit -> int32 with the accumulator in tensor memory (TMEM).
// The pages give no GPU kernel; the add / subtract / skip of [Production]
// "The MatMul-Free Breakthrough" is what the integer MMA computes exactly
// (all partial sums fit int32), and the rescale of [Production] pipeline
// step 5 is fused into the epilogue.
//
// The MMA consumes the 2-bit codes c = t + 1 in {0, 1, 2} directly as
// unsigned 8-bit values (A operand) against the signed int8 activations
// (B operand), so sum c * x~ = y_int + xsum; the epilogue subtracts the
// quantiser's per-token xsum.  That saves the per-byte sign conversion in
// the unpack, which is what bounds this kernel.
//
// Tile: 128 output features (the MMA's M, operand A = weights) by BM tokens
// (the MMA's N, operand B = activations), K in stages of 128.  Per stage:
//   * warp 0 (one thread) issues two TMA loads: the BM x 128 int8 activation
//     tile (128-byte swizzle, K-major) and the 128 x 32-byte packed weight
//     tile;
//   * warps 2-9 expand the packed codes (each thread: half of one row's 32
//     bytes, i.e. 64 codes) to bytes in natural k order, directly in the
//     128-byte swizzled K-major layout the MMA reads, then fence the
//     generic->async proxy and arrive (one arrival per warp);
//   * warp 1 (one thread) issues four 128 x BM x 32 MMAs and commits the
//     stage back to the producer.
// After the K loop warps 2-9 read the accumulator (one TMEM lane = one
// output feature; the two warps of a lane quarter split the token columns),
// subtract xsum, rescale and store.  Every barrier wait is bounded (see
// common.cuh).  No cluster, no multicast.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace bl {

constexpr int kTcBN = 128;  // features per tile (MMA M)
constexpr int kTcBK = 128;  // K per stage: one 128-byte swizzle row of int8
constexpr int kTcUnpackWarps = 8;
constexpr int kTcThreads = 32 * (2 + kTcUnpackWarps);

template <int BM>
struct TcCfg {
  static constexpr int kStages = BM >= 256 ? 4 : (BM >= 128 ? 5 : 6);
  static constexpr int kABytes = kTcBN * kTcBK;        // unpacked weights
  static constexpr int kBBytes = BM * kTcBK;           // activations
  static constexpr int kPBytes = kTcBN * (kTcBK / 4);  // packed weights
  static constexpr int kTmemCols = BM < 32 ? 32 : BM;
  static constexpr int kBarBytes = 8 * (3 * kStages + 1) + 16 + 8 * BM;
  static constexpr size_t kSmem =
      1024 + static_cast<size_t>(kStages) * (kABytes + kBBytes + kPBytes) + kBarBytes;
};

template <int BM, typename OutT>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
              const float* __restrict__ eta, const int32_t* __restrict__ xsum,
              const float* __restrict__ gamma_p, int M, int K, int N, void* __restrict__ y,
              int32_t* __restrict__ y_int) {
  using Cfg = TcCfg<BM>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = base;
  uint8_t* sB = sA + S * Cfg::kABytes;
  uint8_t* sP = sB + S * Cfg::kBBytes;
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(sP + S * Cfg::kPBytes);
  uint64_t* full_a = full_tma + S;
  uint64_t* empty = full_a + S;
  uint64_t* accum_full = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_scale = reinterpret_cast<float*>(tmem_slot + 4);
  int32_t* s_xsum = reinterpret_cast<int32_t*>(s_scale + BM);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTcBN;
  const int m0 = blockIdx.y * BM;
  const int KT = (K + kTcBK - 1) / kTcBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_tma + s, 1);
      mbar_init(full_a + s, kTcUnpackWarps);
      mbar_init(empty + s, 1);
    }
    mbar_init(accum_full, 1);
    *abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  {
    const float gamma = *gamma_p;
    for (int i = threadIdx.x; i < BM; i += blockDim.x) {
      const bool in = m0 + i < M;
      s_scale[i] = in ? token_scale(eta[m0 + i], gamma) : 0.0f;
      s_xsum[i] = in ? xsum[m0 + i] : 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % S;
        const uint32_t round = static_cast<uint32_t>(kt / S);
        if (kt >= S && !mbar_wait(empty + s, (round - 1) & 1u, abort_flag)) break;
        mbar_arrive_expect_tx(full_tma + s, Cfg::kBBytes + Cfg::kPBytes);
        tma_load_2d(sB + s * Cfg::kBBytes, &tm_x, full_tma + s, kt * kTcBK, m0);
        tma_load_2d(sP + s * Cfg::kPBytes, &tm_w, full_tma + s, kt * (kTcBK / 4), n0);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_i8_u8s8(kTcBN, BM);
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % S;
        const uint32_t par = static_cast<uint32_t>(kt / S) & 1u;
        ok = mbar_wait(full_tma + s, par, abort_flag) && mbar_wait(full_a + s, par, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * Cfg::kABytes);
        const uint32_t b0 = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kTcBK / 32; ++kk)
          tc_mma_i8_ss(tmem_d, make_sw128_kmajor_desc(a0 + 32 * kk),
                       make_sw128_kmajor_desc(b0 + 32 * kk), idesc, (kt | kk) != 0 ? 1u : 0u);
        tc_commit(empty + s);
      }
      if (ok) tc_commit(accum_full);
    }
  } else {
    // ---------------- unpack, then epilogue (warps 2..9)
    const int u = warp - 2;          // 0..7
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;   // weight row (output feature) in the tile
    const int half = u >> 2;         // which half of the row's 32 packed bytes
    const int r8 = row & 7;
    uint8_t* a_row = sA + (row >> 3) * 1024 + r8 * 128;
    bool ok = true;
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % S;
      const uint32_t par = static_cast<uint32_t>(kt / S) & 1u;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(full_tma + s, par, abort_flag));
      if (!ok) break;
      const uint4 p = *reinterpret_cast<const uint4*>(sP + s * Cfg::kPBytes + row * 32 + half * 16);
      const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
      uint8_t* dst = a_row + s * Cfg::kABytes;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = half * 4 + i;  // 16-byte chunk of the 128-byte row
        // word c holds the codes of k = 16c .. 16c+15; byte b bits 2j = k 16c+4b+j
        const uint32_t t0 = pw[i] & 0x03030303u;
        const uint32_t t1 = (pw[i] >> 2) & 0x03030303u;
        const uint32_t t2 = (pw[i] >> 4) & 0x03030303u;
        const uint32_t t3 = (pw[i] >> 6) & 0x03030303u;
        uint32_t o0, o1, o2, o3;
        transpose4x4_bytes(t0, t1, t2, t3, o0, o1, o2, o3);  // natural k order
        *reinterpret_cast<uint4*>(dst + ((c ^ r8) << 4)) = make_uint4(o0, o1, o2, o3);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(full_a + s);
    }
    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(accum_full, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int n = n0 + row;
      const uint32_t t_row = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      constexpr int kColsPerWarp = BM < 32 ? 16 : BM / 2;  // two warps per lane quarter
      const int col0 = (BM < 32) ? 0 : half * kColsPerWarp;
      if (!(BM < 32 && half == 1)) {
#pragma unroll 1
        for (int cc = col0; cc < col0 + kColsPerWarp; cc += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_row + cc, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m0 + cc + j;
            if (m < M && n < N) {
              const int32_t yi = static_cast<int32_t>(v[j]) - s_xsum[cc + j];
              const int64_t o = static_cast<int64_t>(m) * N + n;
              store_out<OutT>(y, o, rescale(yi, s_scale[cc + j]));
              if (y_int) y_int[o] = yi;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, Cfg::kTmemCols);
  }
}

}  // namespace bl

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
//   * warp 0 issues two TMA loads: lane 1 the 128 x 32-byte packed weight
//     tile, lane 0 the BM x 128 int8 activation tile (128-byte swizzle,
//     K-major).  When the caller declares the weights static, the packed
//     tiles of the first S stages are requested before griddepcontrol.wait,
//     overlapping the preceding kernel;
//   * warps 2-9 expand the packed codes (each thread: half of one row's 32
//     bytes, i.e. 64 codes; a warp takes 16 consecutive rows) to bytes in
//     natural k order, directly in the 128-byte swizzled K-major layout the
//     MMA reads, then fence the generic->async proxy and arrive (one
//     arrival per warp);
//   * warp 1 (one thread) issues four 128 x BM x 32 MMAs and commits the
//     stage back (one commit per stage: the MMA thread's issue rate bounds
//     the small token tiles).
// After the K loop warps 2-9 read the accumulator (one TMEM lane = one
// output feature; the two warps of a lane quarter split the token columns),
// subtract xsum, rescale and store.
//
// Split K (few tokens, so fewer tiles than SMs): the launch groups
// `ksplit` CTAs along K into a thread-block cluster; CTA r accumulates K
// tiles [KT*r/ksplit, KT*(r+1)/ksplit) in its own TMEM.  After a cluster
// barrier (every MMA of the cluster done, so the stage memory of CTA 0 is
// free) CTAs 1.. store their int32 partial tiles into CTA 0's stage memory
// through distributed shared memory; after a second barrier CTA 0 adds
// them to its own accumulator and runs the epilogue.  Integer sums, so the
// result does not depend on the split.  Every barrier wait is bounded (see
// common.cuh); the cluster barriers count exited threads as arrived.  No
// multicast.
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
  // few stages for the small token tiles: two CTAs fit per SM
  static constexpr int kStages = BM >= 256 ? 4 : (BM >= 128 ? 5 : (BM >= 64 ? 6 : 4));
  static constexpr int kABytes = kTcBN * kTcBK;        // unpacked weights
  static constexpr int kBBytes = BM * kTcBK;           // activations
  static constexpr int kPBytes = kTcBN * (kTcBK / 4);  // packed weights
  static constexpr size_t kStageRegion =
      static_cast<size_t>(kStages) * (kABytes + kBBytes + kPBytes);
  // largest split whose partial tiles fit in CTA 0's stage memory
  static constexpr int kMaxSplit =
      1 + static_cast<int>(kStageRegion / (static_cast<size_t>(kTcBN) * BM * 4)) > 8
          ? 8
          : 1 + static_cast<int>(kStageRegion / (static_cast<size_t>(kTcBN) * BM * 4));
  static constexpr int kTmemCols = BM < 32 ? 32 : BM;
  static constexpr int kBarBytes = 8 * (4 * kStages + 2) + 16 + 8 * BM;
  static constexpr size_t kSmem = 1024 + kStageRegion + kBarBytes;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static_assert(BM > 32 || kSmem <= 113 * 1024, "two CTAs per SM for the small token tiles");
};

template <int BM, typename OutT>
__global__ void __launch_bounds__(kTcThreads, BM <= 32 ? 2 : 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
              const float* __restrict__ eta, const int32_t* __restrict__ xsum,
              const float* __restrict__ gamma_p, int M, int K, int N, void* __restrict__ y,
              int32_t* __restrict__ y_int, int ksplit, int wstatic) {
  using Cfg = TcCfg<BM>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (the swizzle atom), by pointer arithmetic on the
  // shared array so that every access below stays a shared-memory access
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = base;                    // [S] unpacked weights
  uint8_t* sB = sA + S * Cfg::kABytes;   // [S] activations
  uint8_t* sP = sB + S * Cfg::kBBytes;   // [S] packed weights
  uint64_t* full_a = reinterpret_cast<uint64_t*>(sP + S * Cfg::kPBytes);  // unpacked (8 warps)
  uint64_t* full_p = full_a + S;  // packed weight tile in
  uint64_t* full_b = full_p + S;  // activation tile in
  uint64_t* empty = full_b + S;   // the MMA is done with the stage
  uint64_t* accum_full = empty + S;
  uint64_t* drain = accum_full + 1;  // the MMAs issued before an abort are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_scale = reinterpret_cast<float*>(tmem_slot + 4);
  int32_t* s_xsum = reinterpret_cast<int32_t*>(s_scale + BM);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTcBN;
  const int m0 = blockIdx.y * BM;
  const int KT = (K + kTcBK - 1) / kTcBK;
  const int zr = ksplit > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int kt0 = static_cast<int>(static_cast<int64_t>(KT) * zr / ksplit);
  const int nkt = static_cast<int>(static_cast<int64_t>(KT) * (zr + 1) / ksplit) - kt0;  // >= 1

  auto issue_p = [&](int i) {  // packed weight tile i of this CTA's K range
    const int s = i % S;
    mbar_arrive_expect_tx(full_p + s, Cfg::kPBytes);
    tma_load_2d(sP + s * Cfg::kPBytes, &tm_w, full_p + s, (kt0 + i) * (kTcBK / 4), n0);
  };
  const int p_first = nkt < S ? nkt : S;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_a + s, kTcUnpackWarps);
      mbar_init(full_p + s, 1);
      mbar_init(full_b + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(accum_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    if (wstatic)
      for (int i = 0; i < p_first; ++i) issue_p(i);  // not written by the preceding kernel
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
  bool epi_ok = false;  // unpack warps: the accumulator is complete
  int issued = 0;       // warp 0, lane 0 / 1: activation / packed-weight loads issued

  if (warp == 0) {
    // ---------------- TMA producers: lane 0 activations, lane 1 packed weights
    if (lane == 0) {
      for (int i = 0; i < nkt; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(empty + s, static_cast<uint32_t>(i / S - 1) & 1u, abort_flag)) break;
        mbar_arrive_expect_tx(full_b + s, Cfg::kBBytes);
        tma_load_2d(sB + s * Cfg::kBBytes, &tm_x, full_b + s, (kt0 + i) * kTcBK, m0);
        issued = i + 1;
      }
    } else if (lane == 1) {
      if (!wstatic)
        for (int i = 0; i < p_first; ++i) issue_p(i);
      issued = p_first;
      for (int i = S; i < nkt; ++i) {
        if (!mbar_wait(empty + i % S, static_cast<uint32_t>(i / S - 1) & 1u, abort_flag)) break;
        issue_p(i);
        issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_i8_u8s8(kTcBN, BM);
      // Descriptors of stage 0, advanced by adding to the start-address field
      // (address >> 4 in the low bits; every stage address stays below 2^18,
      // so the field never carries): +S_bytes/16 per stage, +2 per K step of
      // 32 bytes.  Keeps the single issuing thread's work per stage short.
      const uint64_t a_desc0 = make_sw128_kmajor_desc(smem_u32(sA));
      const uint64_t b_desc0 = make_sw128_kmajor_desc(smem_u32(sB));
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % S;
        const uint32_t par = static_cast<uint32_t>(i / S) & 1u;
        ok = mbar_wait(full_b + s, par, abort_flag) && mbar_wait(full_a + s, par, abort_flag);
        if (!ok) {
          if (i > 0) {  // MMAs are in flight: let them finish before TMEM is freed
            tc_commit(drain);
            mbar_drain(drain, 0);
          }
          break;
        }
        tc_fence_after();
        const uint64_t ad = a_desc0 + static_cast<uint64_t>(s * (Cfg::kABytes >> 4));
        const uint64_t bd = b_desc0 + static_cast<uint64_t>(s * (Cfg::kBBytes >> 4));
        tc_mma_i8_ss(tmem_d, ad, bd, idesc, i != 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < kTcBK / 32; ++kk)
          tc_mma_i8_ss(tmem_d, ad + 2 * kk, bd + 2 * kk, idesc, 1u);
        tc_commit(empty + s);
      }
      if (ok) tc_commit(accum_full);
    }
  } else {
    // ---------------- unpack, then epilogue (warps 2..9)
    const int u = warp - 2;            // 0..7
    // thread t = 32u + lane: row t / 2, half t % 2 of the row's 32 packed
    // bytes, so a warp reads 512 contiguous bytes of the packed tile (no
    // bank conflict), and the 16-byte stores of each quarter-warp (rows
    // 4i..4i+3, both halves) land in eight different swizzle chunks
    const int urow = 16 * u + (lane >> 1);  // weight row (output feature) in the tile
    const int uhalf = lane & 1;        // which half of the row's 32 packed bytes
    const int r8 = urow & 7;
    uint8_t* a_row = sA + (urow >> 3) * 1024 + r8 * 128;
    bool ok = true;
    for (int i = 0; i < nkt; ++i) {
      const int s = i % S;
      // the packed tile is in (its load waited for the MMA to free the stage)
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(full_p + s, static_cast<uint32_t>(i / S) & 1u, abort_flag));
      if (!ok) break;
      const uint4 p = *reinterpret_cast<const uint4*>(sP + s * Cfg::kPBytes + urow * 32 + uhalf * 16);
      const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
      uint8_t* dst = a_row + s * Cfg::kABytes;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        const int c = uhalf * 4 + wi;  // 16-byte chunk of the 128-byte row
        // word c holds the codes of k = 16c .. 16c+15; byte b bits 2j = k 16c+4b+j
        const uint32_t t0 = pw[wi] & 0x03030303u;
        const uint32_t t1 = (pw[wi] >> 2) & 0x03030303u;
        const uint32_t t2 = (pw[wi] >> 4) & 0x03030303u;
        const uint32_t t3 = (pw[wi] >> 6) & 0x03030303u;
        uint32_t o0, o1, o2, o3;
        transpose4x4_bytes(t0, t1, t2, t3, o0, o1, o2, o3);  // natural k order
        *reinterpret_cast<uint4*>(dst + ((c ^ r8) << 4)) = make_uint4(o0, o1, o2, o3);
      }
      fence_proxy_async_smem();
      __syncwarp();
#ifdef BL_TEST_HOOKS
      if (g_test_fault == 1 && u == 0 && i == 0) continue;  // a wait that nothing completes
#endif
      if (lane == 0) mbar_arrive(full_a + s);
    }
    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(accum_full, 0, abort_flag));
    epi_ok = ok && __all_sync(0xFFFFFFFFu, *abort_flag == 0);
  }

  // Every role is done and the abort flag is final.  After an abort, the
  // producers wait (bounded) for their last S loads, the only ones that can
  // still be in flight, so no copy lands in shared memory that is reused
  // below or freed at exit.
  __syncwarp();
  __syncthreads();
  if (warp == 0 && lane < 2 && *abort_flag) {
    uint64_t* bars = lane == 0 ? full_b : full_p;
    for (int i = issued > S ? issued - S : 0; i < issued; ++i)
      mbar_drain(bars + i % S, static_cast<uint32_t>(i / S) & 1u);
  }

  // ---------------- epilogue (warps 2..9): one TMEM lane = one output feature
  const bool epi_warp = warp >= 2;
  const int q = warp & 3;
  const int row = q * 32 + lane;
  const int half = (warp - 2) >> 2;
  constexpr int kColsPerWarp = BM < 32 ? 16 : BM / 2;  // two warps per lane quarter
  const int col0 = (BM < 32) ? 0 : half * kColsPerWarp;
  const bool epi_cols = epi_warp && !(BM < 32 && half == 1);
  const uint32_t t_row = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
  // CTA 0's stage memory receives the partial tiles of CTAs 1..ksplit-1:
  // slot r-1, [128 rows][BM columns] int32
  int32_t* part = reinterpret_cast<int32_t*>(sA);
  if (ksplit > 1) {
    __syncwarp();  // the cluster barrier is warp-aligned: reconverge after the role branches
    tc_fence_before();
    cluster_sync_all();  // every MMA of the cluster is done; CTA 0's stages are free
    tc_fence_after();
    if (zr != 0 && epi_cols && epi_ok) {
      int32_t* slot = part + static_cast<size_t>(zr - 1) * kTcBN * BM + static_cast<size_t>(row) * BM;
#pragma unroll 1
      for (int cc = col0; cc < col0 + kColsPerWarp; cc += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(t_row + cc, v);
        tmem_ld_wait();
        const uint32_t dst = cluster_map(slot + cc, 0);
#pragma unroll
        for (int j = 0; j < 16; j += 4) st_cluster_v4(dst + 4 * j, v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    }
    __syncwarp();
    cluster_sync_all();  // the partial tiles are in CTA 0
  }
  if (zr == 0 && epi_cols && epi_ok) {
    tc_fence_after();
    const int n = n0 + row;
#pragma unroll 1
    for (int cc = col0; cc < col0 + kColsPerWarp; cc += 16) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(t_row + cc, v);
      tmem_ld_wait();
      for (int r = 1; r < ksplit; ++r) {
        const int32_t* src = part + static_cast<size_t>(r - 1) * kTcBN * BM + static_cast<size_t>(row) * BM + cc;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const int4 t = *reinterpret_cast<const int4*>(src + j);
          v[j] += static_cast<uint32_t>(t.x);
          v[j + 1] += static_cast<uint32_t>(t.y);
          v[j + 2] += static_cast<uint32_t>(t.z);
          v[j + 3] += static_cast<uint32_t>(t.w);
        }
      }
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
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, Cfg::kTmemCols);
  }
}

}  // namespace bl

// decode.cuh -- decode-time accumulate kernel (a few tokens), CUDA cores,
// packed weights streamed into shared memory by bulk copies (TMA engine).
//
// [Production] "The MatMul-Free Breakthrough" and [Additive] "3. Additive
// Integer Accumulation": y_int[m,n] = sum_{W~=+1} x~ - sum_{W~=-1} x~ (zeros
// skipped); [Production] pipeline step 5: y = y_int * (eta*gamma)/127.
// Optionally fused with the quantiser of [Production] "2. Absmax Dynamic
// Activation Quantization": each CTA quantises the activation rows itself,
// so a decode layer is one kernel.
//
// At a few tokens the layer is a stream over the packed weights (N*K/4
// bytes); the kernel is organised around HBM and around latency:
//   * CTA b owns a contiguous block of rows; one producer warp moves it into
//     a ring of shared-memory stages with cp.async.bulk (one copy per stage,
//     tens of KB in flight per SM, no register cost).  When the caller
//     declares the weights static, the first stages are requested before
//     griddepcontrol.wait, so under programmatic dependent launch the
//     weight stream overlaps the previous kernel.
//   * Two teams of 256 compute threads split every stage's rows; within a
//     team, thread t owns fixed 32-bit columns of every packed row (words t,
//     t+256, ...; a word = 16 codes = 16 activations), the activations for
//     those columns are quantised (or loaded) once into shared slots, and
//     the 32 threads of a warp read 128 consecutive bytes of a row.
//   * Decode is SIMD within a register: a word holds codes c = t + 1 in
//     {0,1,2}; (word >> 2j) & 0x03030303 lines up the j-th code of each byte,
//     and one dp4a against the matching four int8 activations (kept
//     transposed 4x4 within each group of 16) adds sum x~ * c for four of
//     them.  sum x~ * t = sum x~ * c - sum x~, so xsum is subtracted once.
//   * Per stage each thread holds up to 16 row partials; a transposed warp
//     reduction (15 shuffles for 16 values, plus one) leaves one total per
//     lane pair, the 16 warps combine theirs with shared atomics, and the
//     last warp to finish a stage completes its rows (no CTA-wide barrier
//     per stage).  Only the producer lane waits for the preceding grid.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kDecTeams = 2;               // row teams sharing one column ownership
constexpr int kDecColThreads = 256;        // threads per team (own the packed-row columns)
constexpr int kDecComputeWarps = kDecTeams * kDecColThreads / 32;
constexpr int kDecComputeThreads = 32 * kDecComputeWarps;
constexpr int kDecThreads = kDecComputeThreads + 32;  // + producer warp
constexpr int kDecMaxStages = 4;
constexpr int kDecSmemBudget = 64 * 1024;  // stage ring; with the rest, two CTAs fit per SM
constexpr int kDecStageTarget = 32 * 1024;

__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch: wait for the preceding grid (and its memory)
// / allow the next grid to launch.  No-ops when launched without the
// attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void named_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint32_t pack4_i8(int32_t a, int32_t b, int32_t c, int32_t d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | (static_cast<uint32_t>(d) << 24);
}

// x~ given (not fused): the int8 activations themselves.
struct DecNoFuse {};

// 16 bf16 values from shared memory, widened to fp32 exactly.
__device__ __forceinline__ void load16_bf16_smem(const uint8_t* p, float (&f)[16]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint4 b = *reinterpret_cast<const uint4*>(p + 16);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

struct DecodeArgs {
  const void* x;         // activations (fused) or x~ (int8), M x K
  const float* eta;      // not fused: per-token scales
  const int32_t* xsum;   // not fused: per-token sums of x~
  int M, K, N;
  const uint8_t* packed;
  const float* gamma;
  void* y;
  int32_t* y_int;        // optional
  int rows_per_cta;
  int rows_per_stage;    // <= 32 / MT
  int stages;            // <= kDecMaxStages
  int weights_static;
  int8_t* xq_out;        // fused, optional: CTA 0 writes x~, eta, xsum
  float* eta_out;
  int32_t* xsum_out;
};

constexpr int kDecMaxChunks = 64;  // row chunks per CTA (the host sizes the grid to fit)

// Shared memory after the stages: barriers, flags, per-token values and the
// per-chunk reduction slots (32 sums and an arrival counter per chunk).
struct DecTail {
  uint64_t full[kDecMaxStages];
  uint64_t empty[kDecMaxStages];
  uint64_t xfull;  // the activation rows are in xbuf
  int abort_flag;
  float gamma;
  int pad[2];
  float s_max[kDecComputeWarps][8];
  float s_scale[8];
  int32_t s_xsum[8];
  int32_t red[kDecMaxChunks][32];
  int32_t cnt[kDecMaxChunks];
};

// Sum of V values (V = 4, 8, 16 or 32; the first V entries of v) across the
// 32 lanes, transposed: each of log2(V) rounds keeps half of the values (the
// lower or upper half, by one lane bit, starting from bit 4) and adds the
// partner's copy; the remaining rounds are a plain butterfly.  Afterwards
// lane l holds the warp total of value l >> (5 - log2 V).
template <int N, int HALF, int L>
__device__ __forceinline__ void transpose_sum_round(int32_t (&v)[L], int lane) {
  if constexpr (HALF >= 1) {
    if constexpr (N > 1) {
      const bool upper = (lane & HALF) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const int32_t send = upper ? v[i] : v[i + N / 2];
        const int32_t keep = upper ? v[i + N / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, HALF);
      }
      transpose_sum_round<N / 2, HALF / 2, L>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], HALF);
      transpose_sum_round<1, HALF / 2, L>(v, lane);
    }
  }
}

template <int V, int L>
__device__ __forceinline__ int32_t warp_transpose_sum(int32_t (&v)[L], int lane) {
  static_assert(V <= L, "reducing more values than the array holds");
  transpose_sum_round<V, 16, L>(v, lane);
  return v[0];
}

// MT tokens (1, 2, 4); XT = activation type for the fused quantiser, or
// DecNoFuse.  Column thread ct (0..255) of either team owns packed words
// ct, ct+256, ... (nwj = ceil(K/16 / 256) <= 8/MT of them); the transposed
// activation words for them sit in 16-byte shared slots, filled by the two
// teams together and read by both.  Each team takes half of every stage's
// rows (up to 16 / MT each), so only that row loop is unrolled.
//
// Synchronisation: the producer lane initialises the stage barriers, issues
// the first copies, waits for the preceding grid (the only thread that
// does) and releases named barrier 3; the compute warps wait there, pass
// barrier 1 twice (activation absmax, activation slots complete), and need
// no CTA-wide barrier inside the stage loop: each warp adds its row totals
// into the chunk's shared slots with atomics and bumps the chunk's counter;
// the warp that arrives last finishes the chunk (subtract xsum, rescale,
// store).
template <int MT, typename XT, typename OutT>
__global__ void __launch_bounds__(kDecThreads, 2) k_decode(const DecodeArgs a) {
  constexpr bool kFused = !std::is_same<XT, DecNoFuse>::value;
  constexpr int RT = 16 / MT;  // rows per team per stage (RT * MT = 16 sums)
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = a.K, P = K >> 2, NW = K >> 4;
  const int nwj = (NW + kDecColThreads - 1) / kDecColThreads;
  const int S = a.stages;
  const int stage_bytes = a.rows_per_stage * P;
  uint4* xslot = reinterpret_cast<uint4*>(smem);  // [nwj][MT][256 columns]
  // the M activation rows as given (bf16, or int8 x~), copied in one bulk copy
  constexpr int kXElem = kFused ? 2 : 1;
  uint8_t* xbuf = smem + nwj * MT * kDecColThreads * 16;
  const int xbytes = a.M * K * kXElem;
  uint8_t* stages = xbuf + ((MT * K * kXElem + 127) & ~127);
  DecTail& T = *reinterpret_cast<DecTail*>(stages + S * stage_bytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_begin = blockIdx.x * a.rows_per_cta;
  const int nrows = min(a.N, r_begin + a.rows_per_cta) - r_begin;
  const int rps = a.rows_per_stage;
  const int nchunks = nrows > 0 ? (nrows + rps - 1) / rps : 0;
  pdl_trigger();  // the next grid may launch; it waits for our completion before reading y

  if (warp == kDecComputeWarps) {
    // ------------------------------------------------ producer warp
    auto issue = [&](int c) {
      const int s = c % S;
      const int rows = min(rps, nrows - c * rps);
      const uint32_t bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(P);
      mbar_arrive_expect_tx(&T.full[s], bytes);
      bulk_load_1d(stages + s * stage_bytes, a.packed + static_cast<int64_t>(r_begin + c * rps) * P,
                   bytes, &T.full[s]);
    };
    const int first = min(S, nchunks);
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(&T.full[s], 1);
        mbar_init(&T.empty[s], kDecComputeWarps);
      }
      mbar_init(&T.xfull, 1);
      T.abort_flag = 0;
      mbar_init_fence();
      if (a.weights_static)
        for (int c = 0; c < first; ++c) issue(c);
      pdl_wait();  // the preceding grid is complete and its writes are visible
      mbar_arrive_expect_tx(&T.xfull, static_cast<uint32_t>(xbytes));
      bulk_load_1d(xbuf, a.x, static_cast<uint32_t>(xbytes), &T.xfull);
      T.gamma = *a.gamma;
      if (!a.weights_static)
        for (int c = 0; c < first; ++c) issue(c);
    }
    __syncwarp();
    named_arrive(3, kDecThreads);  // barriers initialised, inputs readable
    if (lane == 0) {
      for (int c = S; c < nchunks; ++c) {
        const int s = c % S;
        if (!mbar_wait(&T.empty[s], static_cast<uint32_t>(c / S - 1) & 1u, &T.abort_flag)) break;
        issue(c);
      }
    }
    return;
  }

  // ------------------------------------------------ compute warps
  const int tid = threadIdx.x;
  const int team = tid / kDecColThreads;
  const int ct = tid - team * kDecColThreads;
  for (int i = tid; i < nchunks * 32; i += kDecComputeThreads) (&T.red[0][0])[i] = 0;
  for (int i = tid; i < nchunks; i += kDecComputeThreads) T.cnt[i] = 0;
  if (tid < 8) T.s_xsum[tid] = 0;
  named_sync(3, kDecThreads);  // wait for the producer: inputs of earlier kernels are visible
  const float gamma = T.gamma;
  const bool x_ok =
      __all_sync(0xFFFFFFFFu, mbar_wait(&T.xfull, 0, &T.abort_flag));  // activations in xbuf
  if constexpr (kFused) {
    static_assert(sizeof(XT) == 2, "the fused decode quantiser takes bf16 activations");
    // Word slots j are split between the teams: team t takes j = t, t+2, ...
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float amax = 0.0f;
#pragma unroll 1
      for (int j = team; j < nwj; j += kDecTeams) {
        const int w = ct + j * kDecColThreads;
        if (m < a.M && w < NW) {
          float f[16];
          load16_bf16_smem(xbuf + (m * K + 16 * w) * 2, f);
#pragma unroll
          for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) T.s_max[warp][m] = amax;
    }
    named_sync(1, kDecComputeThreads);  // also orders the zeroing above
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float e = T.s_max[0][m];
#pragma unroll
      for (int i = 1; i < kDecComputeWarps; ++i) e = fmaxf(e, T.s_max[i][m]);
      const float eta = fmaxf(e, 1e-5f);
      const float rcp = __frcp_rn(eta);
      int32_t psum = 0;
#pragma unroll 1
      for (int j = team; j < nwj; j += kDecTeams) {
        const int w = ct + j * kDecColThreads;
        uint32_t q0 = 0, q1 = 0, q2 = 0, q3 = 0;
        if (m < a.M && w < NW) {
          float f[16];
          load16_bf16_smem(xbuf + (m * K + 16 * w) * 2, f);
          int32_t q[16];
          quantise16(f, eta, rcp, q);
#pragma unroll
          for (int i = 0; i < 16; ++i) psum += q[i];
          q0 = pack4_i8(q[0], q[1], q[2], q[3]);
          q1 = pack4_i8(q[4], q[5], q[6], q[7]);
          q2 = pack4_i8(q[8], q[9], q[10], q[11]);
          q3 = pack4_i8(q[12], q[13], q[14], q[15]);
          if (a.xq_out && blockIdx.x == 0)
            *reinterpret_cast<uint4*>(a.xq_out + static_cast<int64_t>(m) * K + 16 * w) =
                make_uint4(q0, q1, q2, q3);
        }
        uint4 t;
        transpose4x4_bytes(q0, q1, q2, q3, t.x, t.y, t.z, t.w);
        xslot[(j * MT + m) * kDecColThreads + ct] = t;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xFFFFFFFFu, psum, o);
      if (lane == 0) atomicAdd(&T.s_xsum[m], psum);
      if (tid == 0) {
        T.s_scale[m] = token_scale(eta, gamma);
        if (blockIdx.x == 0 && m < a.M && a.eta_out) a.eta_out[m] = eta;
      }
    }
  } else {
#pragma unroll 1
    for (int j = team; j < nwj; j += kDecTeams)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int w = ct + j * kDecColThreads;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < a.M && w < NW) v = *reinterpret_cast<const uint4*>(xbuf + m * K + 16 * w);
        uint4 t;
        transpose4x4_bytes(v.x, v.y, v.z, v.w, t.x, t.y, t.z, t.w);
        xslot[(j * MT + m) * kDecColThreads + ct] = t;
      }
    if (tid < MT) {
      T.s_scale[tid] = (tid < a.M) ? token_scale(a.eta[tid], gamma) : 0.0f;
      T.s_xsum[tid] = (tid < a.M) ? a.xsum[tid] : 0;
    }
  }
  named_sync(1, kDecComputeThreads);  // activation slots of both teams are complete

  for (int c = 0; c < (x_ok ? nchunks : 0); ++c) {
    const int s = c % S;
    const bool ok =
        __all_sync(0xFFFFFFFFu, mbar_wait(&T.full[s], static_cast<uint32_t>(c / S) & 1u, &T.abort_flag));
    if (!ok) break;
    const uint8_t* st = stages + s * stage_bytes;
    const int rows = min(rps, nrows - c * rps);
    const int half = (rows + 1) >> 1;        // team 0: rows [0, half), team 1: [half, rows)
    const int row0 = team * half;
    const int trows = min(half, rows - row0);  // this team's rows (may be 0)
    int32_t acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0;
    if (trows > 0) {
#pragma unroll 1
      for (int j = 0; j < nwj; ++j) {
        uint32_t xw[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4 v = xslot[(j * MT + m) * kDecColThreads + ct];
          xw[m][0] = v.x; xw[m][1] = v.y; xw[m][2] = v.z; xw[m][3] = v.w;
        }
        // words this thread does not own read word NW-1 against zero activations
        const uint8_t* col = st + row0 * P + 4 * min(ct + j * kDecColThreads, NW - 1);
        // Rows in warp-uniform blocks of 4; inside a block the code is
        // branch-free so the shared loads can be issued early (rows past the
        // team's last read that last row again; their sums are discarded).
#pragma unroll
        for (int r0 = 0; r0 < RT; r0 += 4) {
          if (r0 < trows) {
#pragma unroll
            for (int r = r0; r < r0 + 4 && r < RT; ++r) {
              const uint32_t pw = *reinterpret_cast<const uint32_t*>(col + min(r, trows - 1) * P);
              const uint32_t c0 = pw & 0x03030303u, c1 = (pw >> 2) & 0x03030303u;
              const uint32_t c2 = (pw >> 4) & 0x03030303u, c3 = (pw >> 6) & 0x03030303u;
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                int32_t t = acc[r * MT + m];
                t = __dp4a(static_cast<int>(c0), static_cast<int>(xw[m][0]), t);
                t = __dp4a(static_cast<int>(c1), static_cast<int>(xw[m][1]), t);
                t = __dp4a(static_cast<int>(c2), static_cast<int>(xw[m][2]), t);
                t = __dp4a(static_cast<int>(c3), static_cast<int>(xw[m][3]), t);
                acc[r * MT + m] = t;
              }
            }
          }
        }
      }
    }
    // The stage is fully read into registers: hand it back to the producer.
    __syncwarp();
    if (lane == 0) mbar_arrive(&T.empty[s]);
    // Warp totals: the lane with index l << (5 - log2 V) holds the sum of value
    // l = (team row l / MT, token l % MT); fewer rounds for fewer rows.
    // Only values of this team's real rows are added (the clamped duplicate
    // rows past them would land in the other team's slots).
    if (trows > 0) {
      const int base = row0 * MT, nval = trows * MT;
      if (nval > 8) {
        const int32_t v = warp_transpose_sum<16>(acc, lane);
        if ((lane & 1) == 0 && (lane >> 1) < nval) atomicAdd(&T.red[c][base + (lane >> 1)], v);
      } else if (nval > 4) {
        const int32_t v = warp_transpose_sum<8>(acc, lane);
        if ((lane & 3) == 0 && (lane >> 2) < nval) atomicAdd(&T.red[c][base + (lane >> 2)], v);
      } else {
        const int32_t v = warp_transpose_sum<4>(acc, lane);
        if ((lane & 7) == 0 && (lane >> 3) < nval) atomicAdd(&T.red[c][base + (lane >> 3)], v);
      }
    }
    __threadfence_block();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = (atomicAdd(&T.cnt[c], 1) == kDecComputeWarps - 1);
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (last) {
      __threadfence_block();
      const int r = lane / MT, m = lane - r * MT;
      if (r < rows && m < a.M) {
        const int32_t tot = *reinterpret_cast<volatile int32_t*>(&T.red[c][lane]);
        const int32_t xs = *reinterpret_cast<volatile int32_t*>(&T.s_xsum[m]);
        const float sc = *reinterpret_cast<volatile float*>(&T.s_scale[m]);
        if constexpr (kFused) {
          if (c == 0 && r == 0 && blockIdx.x == 0 && a.xsum_out) a.xsum_out[m] = xs;
        }
        const int32_t yi = tot - xs;
        const int64_t o = static_cast<int64_t>(m) * a.N + r_begin + c * rps + r;
        store_out<OutT>(a.y, o, rescale(yi, sc));
        if (a.y_int) a.y_int[o] = yi;
      }
    }
  }
}

}  // namespace bl

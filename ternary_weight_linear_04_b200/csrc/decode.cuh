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
// bytes), and for the layer sizes of a decoder a single launch is short
// enough that its latency chain matters as much as bandwidth:
//   * CTA b owns a contiguous range of output rows, cut into blocks of RB
//     rows.  One producer warp moves the range into a ring of shared-memory
//     stages with cp.async.bulk (whole blocks per stage, tens of KB in flight
//     per SM, no register cost).  When the caller declares the weights
//     static, the first stages and gamma are requested before
//     griddepcontrol.wait, so under programmatic dependent launch the weight
//     stream overlaps the previous kernel and only the activations wait.
//   * The 16 compute warps form teams of G warps; a team owns whole row
//     blocks (blocks b = team, team + teams, ...), and its 32*G lanes split
//     the packed row into 32-bit words (lane t: words t, t + 32G, ...; a word
//     = 16 codes = 16 activations).  G and RB are chosen on the host per
//     (K, N, M) so that padding words and padding rows stay small; with G = 1
//     a warp finishes its rows alone, with no cross-warp step.
//   * The activations are quantised once per CTA into shared slots, 16 bytes
//     per (token, word), transposed 4x4 so byte lane b of slot word j holds
//     activation 4b + j of the group.
//   * Decode is SIMD within a register: a packed word holds codes
//     c = t + 1 in {0,1,2}, code k of the word in bits 2k..2k+1, so byte b
//     holds codes 4b..4b+3.  w & 0x03030303 and (w >> 4) & 0x03030303 line
//     up codes 4b and 4b+2 of every byte (factor 1); w & 0x0C0C0C0C and
//     (w >> 4) & 0x0C0C0C0C codes 4b+1 and 4b+3 shifted left by 2 (factor
//     4), so one dp4a per plane against the matching activation word adds
//     sum x~ * c for four of them and the two factor classes go to two
//     accumulators (acc1 + acc4 / 4 at the end, exact).  sum x~ * t =
//     sum x~ * c - sum x~, so xsum is subtracted once per output.
//   * A transposed warp reduction (values halved per shuffle round) leaves
//     one row total per lane group; with G > 1 the team's warps add theirs
//     with shared atomics and the last to arrive stores the block.
//   * Only the producer lane waits for the preceding grid; every other
//     thread waits on it through a named barrier.  The same lane then lets
//     the next grid launch (griddepcontrol.launch_dependents), early enough
//     for that grid's weight stream to overlap this kernel's work.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kDecComputeWarps = 16;
constexpr int kDecComputeThreads = 32 * kDecComputeWarps;
constexpr int kDecThreads = kDecComputeThreads + 32;  // + producer warp
constexpr int kDecMaxStages = 8;
constexpr int kDecMaxBlocks = 64;  // row blocks per CTA when warps share a block (reduction slots)
constexpr int kDecMaxMT = 4;
constexpr int kDecMaxSeg = 4;  // matrices sharing one activation input in one launch

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

// x~ given (not fused): the int8 activations themselves.
struct DecNoFuse {};

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
  int blocks_per_chunk;  // row blocks per ring stage
  int stages;            // <= kDecMaxStages
  int weights_static;
  int team_warps;        // G: warps sharing one row block (they split K)
  int teams;             // teams * G <= 16 warps accumulate
  int nwj;               // words per lane: 32 * G * nwj >= K / 16
  int x_staged;          // the activations are bulk-copied into shared memory
  int8_t* xq_out;        // fused, optional: CTA 0 writes x~, eta, xsum
  float* eta_out;
  int32_t* xsum_out;
  // Several matrices sharing these activations (nseg >= 1): CTAs
  // [seg_cta0[s], seg_cta0[s+1]) work on segment s, whose packed weights,
  // gamma, output and row count replace packed / gamma / y / N above.
  int nseg;              // 0 = the single matrix above
  int seg_cta0[kDecMaxSeg + 1];
  const uint8_t* seg_packed[kDecMaxSeg];
  const float* seg_gamma[kDecMaxSeg];
  void* seg_y[kDecMaxSeg];
  int seg_N[kDecMaxSeg];
};

// Shared memory after the stages: barriers, flags, per-token values and the
// per-block reduction slots.
struct DecTail {
  uint64_t full[kDecMaxStages];
  uint64_t empty[kDecMaxStages];
  uint64_t xfull;  // the activation rows are in xbuf
  int abort_flag;
  float gamma;
  uint32_t s_max[kDecComputeWarps][kDecMaxMT];  // per-warp max |x| (fp32 bits)
  float s_scale[kDecMaxMT];
  int32_t s_xsum[kDecMaxMT];
  int32_t red[kDecMaxBlocks][16];
  int32_t cnt[kDecMaxBlocks];
};

// Sum of V values (V = 1, 2, 4, 8 or 16; the first V entries of v) across
// the 32 lanes, transposed: each of log2(V) rounds keeps half of the values
// (the lower or upper half, by one lane bit, starting from bit 4) and adds
// the partner's copy; the remaining rounds are a plain butterfly.
// Afterwards lane l holds the warp total of value l >> (5 - log2 V).
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

constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

// MT tokens (1, 2, 4); RB rows per block (RB * MT <= 16); XT = activation
// type for the fused quantiser (bf16), or DecNoFuse when x~ is given.
//
// Shared memory: [x~ slots: MT x 32*G*nwj x 16 B][activations, if staged]
// [ring: stages x blocks_per_chunk x RB x K/4 B][DecTail].
//
// Synchronisation: the producer lane initialises the barriers, issues the
// first copies (and reads gamma) when the weights are static, waits for the
// preceding grid (the only thread that does), copies the activations and
// releases named barrier 3; the compute warps wait there, pass barrier 1
// twice (activation absmax; activation slots complete), then run the block
// loop with no CTA-wide barrier: a warp releases a stage after its blocks in
// it are done, and with G > 1 the last warp of a team to add into a block's
// slots stores that block.
template <int MT, int RB, typename XT, typename OutT>
__global__ void __launch_bounds__(kDecThreads, 2) k_decode(const DecodeArgs a) {
  constexpr bool kFused = !std::is_same<XT, DecNoFuse>::value;
  constexpr int V = RB * MT;            // values per lane per block
  constexpr bool kTwoAcc = V <= 8;      // two accumulators (5 ALU / word) fit the registers
  static_assert(V >= 1 && V <= 16 && (V & (V - 1)) == 0, "RB * MT must be 1, 2, 4, 8 or 16");
  static_assert(MT <= kDecMaxMT, "at most 4 tokens");
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = a.K, P = K >> 2, NW = K >> 4;
  const int G = a.team_warps;
  const int NWP = 32 * G * a.nwj;       // word slots per token (>= NW)
  constexpr int kXElem = kFused ? 2 : 1;
  uint8_t* xt = smem;                   // [MT][NWP] x 16 B
  uint8_t* xbuf = smem + MT * NWP * 16;
  const int xbytes = a.M * K * kXElem;
  uint8_t* stages = xbuf + (a.x_staged ? ((xbytes + 127) & ~127) : 0);
  const int rows_per_chunk = a.blocks_per_chunk * RB;
  const int stage_bytes = rows_per_chunk * P;
  const int S = a.stages;
  DecTail& T = *reinterpret_cast<DecTail*>(stages + S * stage_bytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's matrix (one of several sharing the activations, or the only one)
  int cta = blockIdx.x, seg = 0;
  if (a.nseg > 0) {
    while (seg + 1 < a.nseg && cta >= a.seg_cta0[seg + 1]) ++seg;
    cta -= a.seg_cta0[seg];
  }
  const uint8_t* const packed = a.nseg > 0 ? a.seg_packed[seg] : a.packed;
  const float* const gamma_p = a.nseg > 0 ? a.seg_gamma[seg] : a.gamma;
  void* const y_out = a.nseg > 0 ? a.seg_y[seg] : a.y;
  const int N = a.nseg > 0 ? a.seg_N[seg] : a.N;
  const int r_begin = cta * a.rows_per_cta;
  const int nrows = max(0, min(N - r_begin, a.rows_per_cta));
  const int nblocks = (nrows + RB - 1) / RB;
  const int nchunks = (nrows + rows_per_chunk - 1) / rows_per_chunk;
  const int acc_warps = a.teams * G;

  if (warp == kDecComputeWarps) {
    // ------------------------------------------------ producer warp
    auto issue = [&](int c) {
      const int s = c % S;
      const int rows = min(rows_per_chunk, nrows - c * rows_per_chunk);
      const uint32_t bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(P);
      mbar_arrive_expect_tx(&T.full[s], bytes);
      bulk_load_1d(stages + s * stage_bytes,
                   packed + static_cast<int64_t>(r_begin + c * rows_per_chunk) * P, bytes,
                   &T.full[s]);
    };
    const int first = min(S, nchunks);
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(&T.full[s], 1);
        mbar_init(&T.empty[s], acc_warps);
      }
      mbar_init(&T.xfull, 1);
      T.abort_flag = 0;
      mbar_init_fence();
      if (a.weights_static) {
        for (int c = 0; c < first; ++c) issue(c);
        T.gamma = *gamma_p;
      }
      pdl_wait();  // the preceding grid is complete and its writes are visible
      // Only now let the next grid launch: every SM then holds exactly this
      // kernel's CTAs, so the next grid's CTAs spread one per SM.  Launched
      // earlier, some of them land on SMs the preceding grid has not yet
      // left and pair up with another CTA of their own grid there, and that
      // SM's pair finishes last.
      pdl_trigger();
      if (a.x_staged) {
        mbar_arrive_expect_tx(&T.xfull, static_cast<uint32_t>(xbytes));
        bulk_load_1d(xbuf, a.x, static_cast<uint32_t>(xbytes), &T.xfull);
      }
      if (!a.weights_static) {
        for (int c = 0; c < first; ++c) issue(c);
        T.gamma = *gamma_p;
      }
    }
    __syncwarp();
    named_arrive(3, kDecThreads);  // barriers initialised, gamma in place, inputs readable
    if (lane == 0) {
      int issued = first;
      for (int c = S; c < nchunks; ++c) {
        const int s = c % S;
        if (!mbar_wait(&T.empty[s], static_cast<uint32_t>(c / S - 1) & 1u, &T.abort_flag)) break;
        issue(c);
        issued = c + 1;
      }
      // Before this warp exits, the copies it issued have landed (bounded
      // waits): after an abort nothing may still be writing into shared
      // memory when the CTA ends.  In the normal flow they have already
      // been consumed, or land shortly, and the waits return at once.
      for (int c = issued > S ? issued - S : 0; c < issued; ++c)
        mbar_drain(&T.full[c % S], static_cast<uint32_t>(c / S) & 1u);
      if (a.x_staged) mbar_drain(&T.xfull, 0);
    }
    return;
  }

  // ------------------------------------------------ compute warps
  const int tid = threadIdx.x;
  if (G > 1) {
    for (int i = tid; i < nblocks * 16; i += kDecComputeThreads) (&T.red[0][0])[i] = 0;
    for (int i = tid; i < nblocks; i += kDecComputeThreads) T.cnt[i] = 0;
  }
  if (tid < kDecMaxMT) T.s_xsum[tid] = 0;
  named_sync(3, kDecThreads);  // wait for the producer: inputs of earlier kernels are visible
  const float gamma = T.gamma;
  bool x_ok = true;
  if (a.x_staged) x_ok = __all_sync(0xFFFFFFFFu, mbar_wait(&T.xfull, 0, &T.abort_flag));
  const uint8_t* xsrc = a.x_staged ? xbuf : static_cast<const uint8_t*>(a.x);
  uint4* xslot = reinterpret_cast<uint4*>(xt);

  if constexpr (kFused) {
    static_assert(sizeof(XT) == 2, "the fused decode quantiser takes bf16 activations");
    // Pass 1: per-token max |x|, 8 activations per thread and step.  |x| of
    // a bf16 is its bit pattern with the sign cleared, and for non-negative
    // values the bf16 order is the order of those patterns, so the maximum
    // is taken on bf16x2 pairs.
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      uint32_t amax = 0;
      if (m < a.M) {
        for (int o = tid; o < 2 * NW; o += kDecComputeThreads) {
          const uint4 u = *reinterpret_cast<const uint4*>(xsrc + (static_cast<int64_t>(m) * K + 8 * o) * 2);
          const uint32_t wd[4] = {u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu, u.z & 0x7FFF7FFFu,
                                  u.w & 0x7FFF7FFFu};
          __nv_bfloat162 h[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) h[i] = *reinterpret_cast<const __nv_bfloat162*>(&wd[i]);
          const __nv_bfloat162 t = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
          const uint32_t tb = *reinterpret_cast<const uint32_t*>(&t);
          amax = max(amax, max(tb << 16, tb & 0xFFFF0000u));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) T.s_max[warp][m] = amax;
    }
    named_sync(1, kDecComputeThreads);  // also orders the zeroing above
    // Pass 2: quantise 4 activations (one int8 word in natural order) per
    // thread and step, and scatter its bytes into the transposed slot of
    // its group of 16 (byte j of quad b -> slot word j, byte b); padding
    // words get zeros.
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      uint32_t e = 0;
#pragma unroll
      for (int i = 0; i < kDecComputeWarps; ++i) e = max(e, T.s_max[i][m]);
      const float eta = fmaxf(__uint_as_float(e), 1e-5f);
      const float rr = rcp_approx(eta);
      const float qs = __fmul_rn(127.0f, rr);
      const float heta = __fmul_rn(0.5f, eta);
      const bool eta_bf16 = is_bf16_value(eta);
      int32_t psum = 0;
      for (int qd = tid; qd < 4 * NWP; qd += kDecComputeThreads) {
        const int w = qd >> 2;
        uint32_t word = 0;
        if (m < a.M && w < NW) {
          const uint2 u = *reinterpret_cast<const uint2*>(xsrc + (static_cast<int64_t>(m) * K + 4 * qd) * 2);
          const float f[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                              __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u)};
          uint32_t b[4];
          if (eta_bf16) {
            code_bits_bf16_n<4>(f, b, eta, heta, qs, rr);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) b[i] = quantise_exact_bits(f[i], eta);
          }
          word = pack_lowbytes(b[0], b[1], b[2], b[3]);
          psum = __dp4a(static_cast<int>(word), 0x01010101, psum);
          if (a.xq_out && blockIdx.x == 0)
            *reinterpret_cast<uint32_t*>(a.xq_out + static_cast<int64_t>(m) * K + 4 * qd) = word;
        }
        uint8_t* sl = xt + (static_cast<int64_t>(m) * NWP + w) * 16 + (qd & 3);
        sl[0] = static_cast<uint8_t>(word);
        sl[4] = static_cast<uint8_t>(word >> 8);
        sl[8] = static_cast<uint8_t>(word >> 16);
        sl[12] = static_cast<uint8_t>(word >> 24);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xFFFFFFFFu, psum, o);
      if (lane == 0 && psum != 0) atomicAdd(&T.s_xsum[m], psum);
      if (tid == 0) {
        T.s_scale[m] = token_scale(eta, gamma);
        if (blockIdx.x == 0 && m < a.M && a.eta_out) a.eta_out[m] = eta;
      }
    }
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      for (int w = tid; w < NWP; w += kDecComputeThreads) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < a.M && w < NW)
          v = *reinterpret_cast<const uint4*>(xsrc + static_cast<int64_t>(m) * K + 16 * w);
        uint4 t;
        transpose4x4_bytes(v.x, v.y, v.z, v.w, t.x, t.y, t.z, t.w);
        xslot[m * NWP + w] = t;
      }
    if (tid < MT) {
      T.s_scale[tid] = (tid < a.M) ? token_scale(a.eta[tid], gamma) : 0.0f;
      T.s_xsum[tid] = (tid < a.M) ? a.xsum[tid] : 0;
    }
  }
  named_sync(1, kDecComputeThreads);  // activation slots, scales and sums are complete
  if (warp >= acc_warps) return;

  const int team = warp / G, g = warp - team * G;
  const int tt = g * 32 + lane;          // this lane's first word
  const int wstep = 32 * G;
  constexpr int kGroup = 32 / V;         // lanes holding each reduced value
  for (int c = 0; c < (x_ok ? nchunks : 0); ++c) {
    const int s = c % S;
    const bool ok =
        __all_sync(0xFFFFFFFFu, mbar_wait(&T.full[s], static_cast<uint32_t>(c / S) & 1u, &T.abort_flag));
    if (!ok) break;
    const uint8_t* st = stages + s * stage_bytes;
    const int b0 = c * a.blocks_per_chunk;
    const int b_end = min(nblocks, b0 + a.blocks_per_chunk);
    for (int b = b0 + (team - b0 % a.teams + a.teams) % a.teams; b < b_end; b += a.teams) {
      const int row0 = b * RB;                     // first row of the block in this CTA
      const int brows = min(RB, nrows - row0);     // real rows (the rest repeat the last one)
      const uint8_t* blk = st + (row0 - c * rows_per_chunk) * P;
      int32_t acc1[V], acc4[kTwoAcc ? V : 1];
#pragma unroll
      for (int i = 0; i < V; ++i) acc1[i] = 0;
#pragma unroll
      for (int i = 0; i < (kTwoAcc ? V : 1); ++i) acc4[i] = 0;
#pragma unroll 2
      for (int j = 0; j < a.nwj; ++j) {
        const int w = tt + j * wstep;
        uint32_t xw[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4 v = xslot[m * NWP + w];
          xw[m][0] = v.x; xw[m][1] = v.y; xw[m][2] = v.z; xw[m][3] = v.w;
        }
        // padding words read word NW-1 against zero activations
        const uint8_t* col = blk + 4 * min(w, NW - 1);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const uint32_t pw = *reinterpret_cast<const uint32_t*>(col + min(r, brows - 1) * P);
          if constexpr (kTwoAcc) {
            const uint32_t h = pw >> 4;
            const int p0 = static_cast<int>(pw & 0x03030303u), p1 = static_cast<int>(pw & 0x0C0C0C0Cu);
            const int p2 = static_cast<int>(h & 0x03030303u), p3 = static_cast<int>(h & 0x0C0C0C0Cu);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              acc1[r * MT + m] = __dp4a(p0, static_cast<int>(xw[m][0]), acc1[r * MT + m]);
              acc4[r * MT + m] = __dp4a(p1, static_cast<int>(xw[m][1]), acc4[r * MT + m]);
              acc1[r * MT + m] = __dp4a(p2, static_cast<int>(xw[m][2]), acc1[r * MT + m]);
              acc4[r * MT + m] = __dp4a(p3, static_cast<int>(xw[m][3]), acc4[r * MT + m]);
            }
          } else {
            const int p0 = static_cast<int>(pw & 0x03030303u);
            const int p1 = static_cast<int>((pw >> 2) & 0x03030303u);
            const int p2 = static_cast<int>((pw >> 4) & 0x03030303u);
            const int p3 = static_cast<int>((pw >> 6) & 0x03030303u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              int32_t t = acc1[r * MT + m];
              t = __dp4a(p0, static_cast<int>(xw[m][0]), t);
              t = __dp4a(p1, static_cast<int>(xw[m][1]), t);
              t = __dp4a(p2, static_cast<int>(xw[m][2]), t);
              t = __dp4a(p3, static_cast<int>(xw[m][3]), t);
              acc1[r * MT + m] = t;
            }
          }
        }
      }
      if constexpr (kTwoAcc) {
#pragma unroll
        for (int i = 0; i < V; ++i) acc1[i] += acc4[i] >> 2;  // acc4 is a multiple of 4
      }
      const int32_t tot = warp_transpose_sum<V>(acc1, lane);
      const int vi = lane >> ilog2(kGroup);     // value held: row vi / MT, token vi % MT
      const bool holder = (lane & (kGroup - 1)) == 0;
      auto finish = [&](int v, int32_t total) {
        const int r = v / MT, m = v - r * MT;
        if (r < brows && m < a.M) {
          const int32_t yi = total - T.s_xsum[m];
          const int64_t o = static_cast<int64_t>(m) * N + r_begin + row0 + r;
          store_out<OutT>(y_out, o, rescale(yi, T.s_scale[m]));
          if (a.y_int) a.y_int[o] = yi;
          if constexpr (kFused) {
            if (blockIdx.x == 0 && b == 0 && r == 0 && a.xsum_out) a.xsum_out[m] = T.s_xsum[m];
          }
        }
      };
      if (G == 1) {
        if (holder) finish(vi, tot);
      } else {
        if (holder) atomicAdd(&T.red[b][vi], tot);
        __threadfence_block();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = (atomicAdd(&T.cnt[b], 1) == G - 1);
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (last) {
          __threadfence_block();
          if (lane < V) finish(lane, *reinterpret_cast<volatile int32_t*>(&T.red[b][lane]));
        }
      }
    }
    // this warp's blocks of the stage are done: hand it back to the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(&T.empty[s]);
  }
}

}  // namespace bl

// rmsnorm_rows.cuh -- RMSNorm (no affine, eps 1e-6) fused with the
// per-token absmax int8 quantiser for bf16 rows, streamed through shared
// memory, with the sum of squares found in fp64 and proved.
//
// [Production] "2. Absmax Dynamic Activation Quantization": the readings
// and the results are those of k_rmsnorm_quant (rmsnorm.cuh): mean(x^2) =
// RN32(RN64(exact sum of x^2) / K), r = RN32(1 / RN32(sqrt(mean + 1e-6))),
// x_norm = RN32(x * r), then the fp32 absmax quantiser on x_norm.
//
// Layout: a few persistent CTAs per SM; CTA b takes rows b, b + gridDim.x,
// ... through a ring of S row buffers in its shared memory.  Thread 0 fills
// a buffer with one bulk copy per row (cp.async.bulk, completion counted in
// bytes on the buffer's mbarrier) and keeps the next S - 1 rows in flight
// while the CTA works on the current one from shared memory, so the three
// passes over a row (max |x|, sum of squares, quantise) read shared memory,
// not L1 or L2, and each SM keeps (CTAs per SM) x (S - 1) rows of HBM reads
// outstanding.  A buffer is refilled once the row's last block reduction
// has passed (every thread has read it by then).
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "quant.cuh"
#include "rmsnorm.cuh"

namespace bl {

constexpr int kRowsThreads = 256;
constexpr int kRowsMaxStages = 4;

// The 8 fp32 codes of quantise_fast for one vector of bf16 x times the
// RMSNorm scale r (x_norm = RN32(x * r)), packed in order; the near-tie test
// is one vote over the 8 values, so only a vector holding a near tie takes
// the IEEE quotient, for the values that need it.
__device__ __forceinline__ uint2 codes8_norm(const uint4 v, float r, float eta, float qs) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float xn[8];
  uint32_t b[8];
  bool near = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t h = (i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16);
    xn[i] = __fmul_rn(__uint_as_float(h), r);
    const float c = __fmul_rn(xn[i], qs);
    const float t = __fadd_rn(c, kRneMagic);
    const float d = __fsub_rn(c, __fsub_rn(t, kRneMagic));
    b[i] = __float_as_uint(t);
    near |= fabsf(d) > kTieGuard;
  }
  if (__builtin_expect(near, 0)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float c = __fmul_rn(xn[i], qs);
      const float t = __fadd_rn(c, kRneMagic);
      if (fabsf(__fsub_rn(c, __fsub_rn(t, kRneMagic))) > kTieGuard) b[i] = quantise_exact_bits(xn[i], eta);
    }
  }
  return make_uint2(pack_lowbytes(b[0], b[1], b[2], b[3]), pack_lowbytes(b[4], b[5], b[6], b[7]));
}

// ms = RN32(RN64(S) / K) for an fp64 S (the division in fp64).
__device__ __forceinline__ float mean_square_f32(double S, double Kd) {
  return __double2float_rn(__ddiv_rn(S, Kd));
}

// RMSNorm + quantiser for rows with 16-byte vectors (K a multiple of 8, x
// 16-byte and xq 8-byte aligned), stages * 2K bytes of dynamic shared
// memory.  Same readings and results as k_rmsnorm_quant; the sum of
// squares S is found in fp64 and proved rather than summed exactly:
//   * every x^2 of a bf16 x has at most 16 significant bits, so the square
//     of its fp64 widening (widen_bf16_mag, pack.cuh) is exact, and one
//     DFMA adds it with a single rounding; zeros and subnormals widen to
//     values below 2^-126, whose squares (below 2^-252) stand for 0 or the
//     true square;
//   * S^ = the fp64 sum (per thread, then a warp butterfly, then thread 0
//     over the warps): a sum of non-negative terms over a tree of height h
//     is within gamma_h = h u / (1 - h u) (u = 2^-53) of the exact sum of
//     its terms, so |S^ - S| <= B = 1.003 h u S^ + K 2^-252;
//   * everything after depends on S only through ms = RN32(RN64(S) / K),
//     monotone in S: if S^ - B and S^ + B give the same ms, that is the
//     exact ms.  Otherwise (S within about h 2^-53 of a rounding boundary of
//     ms: rare by chance, but rows can be built for it) the CTA sums the
//     row's squares exactly as k_rmsnorm_quant does and takes ms from that.
__global__ void __launch_bounds__(kRowsThreads) k_rmsnorm_rows(const __nv_bfloat16* __restrict__ x,
                                                                    int64_t M, int64_t K, int stages,
                                                                    int8_t* __restrict__ xq,
                                                                    float* __restrict__ eta_out,
                                                                    int32_t* __restrict__ xsum_out) {
  constexpr int NT = kRowsThreads;
  constexpr int NWARP = NT / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bar[kRowsMaxStages];
  __shared__ unsigned long long sb[kBuckets];  // exact pass: terms below the register window
  __shared__ unsigned long long red_lo[NWARP], red_hi[NWARP];
  __shared__ double red_d[NWARP];
  __shared__ float redf[NWARP];
  __shared__ int32_t redi[NWARP];
  __shared__ int s_abort, s_exact, s_tail;
  __shared__ float s_ms;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
  const int nv = static_cast<int>(K >> 3);
  const int64_t G = gridDim.x;
  const double Kd = static_cast<double>(K);
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&bar[s], 1);
    mbar_init_fence();
    s_abort = 0;
  }
  __syncthreads();
  pdl_wait();
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      const int64_t r = blockIdx.x + s * G;
      if (r < M) {
        mbar_arrive_expect_tx(&bar[s], row_bytes);
        bulk_load_1d(smem + static_cast<size_t>(s) * row_bytes, x + r * K, row_bytes, &bar[s]);
      }
    }
    pdl_trigger();
  }
  // Height of the fp64 summation tree: the DFMAs of one thread, five
  // butterfly levels, NWARP - 1 additions over the warps.
  const int h = 8 * ((nv + NT - 1) / NT) + 5 + (NWARP - 1);
  int64_t i = 0;
  for (;; ++i) {
    const int64_t r = blockIdx.x + i * G;
    if (r >= M) break;
    const int s = static_cast<int>(i % stages);
    const uint32_t parity = static_cast<uint32_t>(i / stages) & 1u;
    const uint4* buf = reinterpret_cast<const uint4*>(smem + static_cast<size_t>(s) * row_bytes);
    // Thread 0 waits for the row (bounded); the barrier hands it to the
    // other threads (and makes every thread leave together if the wait ran
    // out) without 255 threads polling the mbarrier.  The phase stays
    // complete until this buffer is refilled: one try_wait per thread then
    // observes it, which makes the copied row visible to that thread.
    const bool ok = tid != 0 || mbar_wait(&bar[s], parity, &s_abort);
    if (__syncthreads_or(!ok)) break;
    (void)mbar_try_wait(&bar[s], parity);

    // Pass 0: max |x|.  Pass 1: the fp64 sum of squares.
    __nv_bfloat162 mx = __float2bfloat162_rn(0.0f);
    double sq = 0.0;
    for (int v = tid; v < nv; v += NT) {
      const uint4 xv = buf[v];
      mx = absmax8_bf16(mx, xv);
      const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double a = widen_bf16_mag(w[j]), b = widen_bf16_mag(w[j] >> 16);
        sq = __fma_rn(a, a, sq);
        sq = __fma_rn(b, b, sq);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq = __dadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, o));
    if (lane == 0) red_d[warp] = sq;
    const float amax = block_max_nt<NT>(fmaxf(__low2float(mx), __high2float(mx)), redf);  // its barriers publish red_d
    if (tid == 0) {
      double S = red_d[0];
      for (int w = 1; w < NWARP; ++w) S = __dadd_rn(S, red_d[w]);
      const double g = 1.003 * static_cast<double>(h) * 0x1p-53;
      const double B = __dadd_ru(__dmul_ru(g, S), __dmul_ru(Kd, 0x1p-252));
      const float lo = mean_square_f32(fmax(__dsub_rd(S, B), 0.0), Kd);
      const float hi = mean_square_f32(__dadd_ru(S, B), Kd);
      s_exact = lo != hi;
      s_ms = lo;
      s_tail = 0;
    }
    __syncthreads();
    if (s_exact) {  // block-uniform
      // The exact sum, as in k_rmsnorm_quant: terms within kSqWindow
      // exponents of the row's largest as 128-bit integers, the rest (and
      // subnormals) into per-exponent buckets.
      for (int b = tid; b < kBuckets; b += NT) sb[b] = 0;
      __syncthreads();
      const int emax = max(1, static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu));
      const int ebase = max(1, emax - kSqWindow);
      unsigned __int128 acc = 0;
      auto add_term = [&](uint32_t hb) {
        uint32_t b, m2;
        sq_term(hb, b, m2);
        const bool in_win = static_cast<int>(b) >= ebase;
        // m2 != 0: a finite value, so b <= emax and the shift stays below 82
        if (in_win && m2 != 0) acc += static_cast<unsigned __int128>(m2) << (2 * (static_cast<int>(b) - ebase));
        if (__any_sync(0xFFFFFFFFu, !in_win && m2 != 0)) {
          s_tail = 1;
          bucket_add_warp_bm(sb, b, in_win ? 0u : m2);
        }
      };
      for (int t = 0; t < (nv + NT - 1) / NT; ++t) {  // the same trips in every lane
        const int v = tid + NT * t;
        const uint4 xv = v < nv ? buf[v] : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          add_term(w[j] & 0xFFFFu);
          add_term(w[j] >> 16);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += shfl_xor_u128(acc, o);
      if (lane == 0) {
        red_lo[warp] = static_cast<unsigned long long>(acc);
        red_hi[warp] = static_cast<unsigned long long>(acc >> 64);
      }
      __syncthreads();  // also completes the bucket adds
      if (tid == 0) {
        unsigned __int128 tot = 0;
        for (int w = 0; w < NWARP; ++w) tot += (static_cast<unsigned __int128>(red_hi[w]) << 64) | red_lo[w];
        const double S = s_tail ? sumsq_rn64(tot, ebase, sb, 1, ebase - 1) : u128_rn64(tot, 2 * ebase - 268);
        s_ms = mean_square_f32(S, Kd);
      }
      __syncthreads();
    }
    const float rn = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(s_ms, 1e-6f)));
    const float eta = fmaxf(__fmul_rn(amax, rn), 1e-5f);
    const float qs = quant_scale(eta);

    // Pass 2: quantise x_norm = RN32(x * r).
    uint2* qrow = reinterpret_cast<uint2*>(xq + r * K);
    int32_t sum = 0;
    for (int v = tid; v < nv; v += NT) {
      const uint2 q = codes8_norm(buf[v], rn, eta, qs);
      qrow[v] = q;
      sum = __dp4a(static_cast<int>(q.x), 0x01010101, sum);
      sum = __dp4a(static_cast<int>(q.y), 0x01010101, sum);
    }
    sum = block_sum_nt<NT>(sum, redi);  // past its barriers every thread is done with buf
    if (tid == 0) {
      eta_out[r] = eta;
      xsum_out[r] = sum;
      const int64_t rn2 = r + stages * G;
      if (rn2 < M) {
        mbar_arrive_expect_tx(&bar[s], row_bytes);
        bulk_load_1d(smem + static_cast<size_t>(s) * row_bytes, x + rn2 * K, row_bytes, &bar[s]);
      }
    }
  }
  if (tid == 0) {
    for (int64_t j = i; j < i + stages; ++j)
      if (blockIdx.x + j * G < M) mbar_drain(&bar[j % stages], static_cast<uint32_t>(j / stages) & 1u);
  }
}

}  // namespace bl

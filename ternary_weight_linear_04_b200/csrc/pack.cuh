// pack.cuh -- load-time kernels: absmean gamma and 2-bit ternary packing.
//
// [Production] "1. Absmean Weight Quantization": gamma = mean |W| over the
// whole matrix (WeightQuantizerSTE clamps it at 1e-5), W~ = Clip(Round(W /
// gamma), -1, +1).  [Production] "Production Deployment Standards"
// guideline 1 and [No-Multiply] "Kernel Implementation: The Lookup Table
// Approach": codes 00 = -1, 01 = 0, 10 = +1, four per byte, element j in
// bits 2j..2j+1.
//
// gamma must be bit-identical wherever it is computed, because the ternary
// threshold sits exactly at |W| = gamma/2.  A floating-point reduction in
// any fixed order is not reproducible across devices, so the sum of |W| is
// taken exactly: |W| = m * 2^(b-150) with m < 2^24 an integer and b the
// (clamped) biased exponent, and the m are summed in 64-bit integer buckets,
// one per b.  A single thread then forms the exact total as a 384-bit
// integer, rounds it once to fp64 (nearest even), divides by N*K in fp64 and
// rounds once to fp32.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kBuckets = 256;

__global__ void k_zero_u64(unsigned long long* p, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0;
}

// sb[b] += m for one (bucket b, integer m < 2^24) per lane.  All 32 lanes
// must call it together (lanes with nothing to add pass m = 0).  Lanes that
// share a bucket are summed with one warp reduction and a single shared
// atomic, one distinct bucket per loop trip.
__device__ __forceinline__ void bucket_add_warp_bm(unsigned long long* sb, uint32_t b, uint32_t m) {
  const int lane = threadIdx.x & 31;
  unsigned todo = 0xFFFFFFFFu;
  while (todo) {
    const int leader = __ffs(todo) - 1;
    const uint32_t lb = __shfl_sync(0xFFFFFFFFu, b, leader);
    const bool mine = (b == lb);
    const unsigned grp = __ballot_sync(0xFFFFFFFFu, mine);
    const uint32_t s = __reduce_add_sync(0xFFFFFFFFu, mine ? m : 0u);  // < 32 * 2^24
    if (lane == leader && s) atomicAdd(&sb[lb], static_cast<unsigned long long>(s));
    todo &= ~grp;
  }
}

// Adds one fp32 bit pattern per lane: bucket = biased exponent, m = integer
// mantissa (|W| = m * 2^(b-150)).
__device__ __forceinline__ void bucket_add_warp(unsigned long long* sb, uint32_t u) {
  const uint32_t e = (u >> 23) & 0xFFu;
  const uint32_t frac = u & 0x7FFFFFu;
  const uint32_t b = e ? e : 1u;                  // subnormals share bucket 1
  const uint32_t m = e ? (frac | 0x800000u) : frac;
  bucket_add_warp_bm(sb, b, m);
}

// buckets[b] += sum of the integer mantissas m of all |W| with bucket b.
// With `skip` set (the fp64 sum already decided gamma) the CTAs return at
// once.
__global__ void __launch_bounds__(256) k_absmean_buckets(const float* __restrict__ W, int64_t count,
                                                          unsigned long long* buckets,
                                                          const int* __restrict__ skip) {
  if (skip && *skip) return;
  __shared__ unsigned long long sb[kBuckets];
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) sb[i] = 0;
  __syncthreads();

  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const bool vec = ((reinterpret_cast<uintptr_t>(W) & 15u) == 0);
  const int64_t nvec = vec ? count / 4 : 0;
  // Vector part: every lane of a warp runs the same number of trips.
  const int64_t trips = (nvec + nthreads - 1) / nthreads;
  const uint4* W4 = reinterpret_cast<const uint4*>(W);
  for (int64_t t = 0; t < trips; ++t) {
    const int64_t i = tid + t * nthreads;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (i < nvec) v = ld_nc_na_v4(W4 + i);
    bucket_add_warp(sb, v.x);
    bucket_add_warp(sb, v.y);
    bucket_add_warp(sb, v.z);
    bucket_add_warp(sb, v.w);
  }
  // Scalar tail (or everything, when W is not 16-byte aligned).
  const int64_t rest = count - nvec * 4;
  const int64_t trips_s = (rest + nthreads - 1) / nthreads;
  const uint32_t* Wu = reinterpret_cast<const uint32_t*>(W) + nvec * 4;
  for (int64_t t = 0; t < trips_s; ++t) {
    const int64_t i = tid + t * nthreads;
    const uint32_t u = (i < rest) ? Wu[i] : 0u;
    bucket_add_warp(sb, u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x)
    if (sb[i]) atomicAdd(&buckets[i], sb[i]);
}

// One thread: exact total of the buckets, rounded to fp64, then gamma.
__global__ void k_gamma_finalize(const unsigned long long* __restrict__ buckets, int64_t count,
                                 float* gamma_out, const int* __restrict__ skip) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (skip && *skip) return;  // gamma was decided by the fp64 sum
  // Fixed point with its unit at 2^-149: bucket b contributes m * 2^(b-1).
  constexpr int kLimbs = 12;  // 384 bits: max position 253 + 64 < 384
  uint32_t L[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) L[i] = 0;
  for (int b = 1; b < kBuckets - 1; ++b) {
    const unsigned long long v = buckets[b];
    if (!v) continue;
    const int pos = b - 1;
    const int li = pos >> 5, sh = pos & 31;
    const unsigned __int128 w = static_cast<unsigned __int128>(v) << sh;  // < 2^95
    uint64_t carry = 0;
    for (int i = 0; i < 3 || carry; ++i) {
      if (li + i >= kLimbs) break;
      const uint64_t part = (i < 3) ? static_cast<uint64_t>(static_cast<uint32_t>(w >> (32 * i))) : 0u;
      const uint64_t s = static_cast<uint64_t>(L[li + i]) + part + carry;
      L[li + i] = static_cast<uint32_t>(s);
      carry = s >> 32;
    }
  }
  int top = -1;
  for (int i = kLimbs - 1; i >= 0; --i) {
    if (L[i]) { top = 32 * i + 31 - __clz(L[i]); break; }
  }
  double S = 0.0;
  if (top >= 0) {
    // Gather bits [lo, top] (at most 53) into an integer mantissa.
    const int lo = top > 52 ? top - 52 : 0;
    unsigned long long mant = 0;
    for (int bit = top; bit >= lo; --bit) mant = (mant << 1) | ((L[bit >> 5] >> (bit & 31)) & 1u);
    if (lo > 0) {
      const uint32_t guard = (L[(lo - 1) >> 5] >> ((lo - 1) & 31)) & 1u;
      bool sticky = false;
      for (int bit = lo - 2; bit >= 0 && !sticky; --bit) sticky = (L[bit >> 5] >> (bit & 31)) & 1u;
      if (guard && (sticky || (mant & 1ull))) mant += 1;  // ties to even; 2^53 stays exact
    }
    S = scalbn(static_cast<double>(mant), lo - 149);
  }
  const double g = S / static_cast<double>(count);  // IEEE fp64 division
  float gf = __double2float_rn(g);
  if (gf < 1e-5f) gf = 1e-5f;
  *gamma_out = gf;
}

// ---------------------------------------------------------------- fp64 sum
// The single-matrix pack first sums |W| in fp64 and proves gamma from that
// sum; the exact buckets above run only when the proof fails.
//   * |W| of an fp32 W has 24 significant bits, exact in fp64; it is widened
//     from its bit pattern (exponent field + 896, the fraction moved down 3
//     bits), which for zeros and subnormals gives a wrong value below
//     2^-126;
//   * the fp64 sum Ŝ is formed over a tree of height h (each thread's adds,
//     a warp butterfly, the 8 warps of a CTA, one atomic add per CTA in any
//     order); for non-negative terms it is within h u / (1 - h u)
//     (u = 2^-53) of the exact sum of its terms, so
//     |Ŝ - S| <= B = 1.003 h u Ŝ + count 2^-126;
//   * gamma = max(RN32(RN64(S) / count), 1e-5) is monotone in S: if Ŝ - B
//     and Ŝ + B (rounded outward) give the same gamma, it is the exact one.
//     Otherwise (S within about h 2^-53 of a rounding boundary of gamma)
//     the buckets run.

// (The widening helpers and the ternary threshold below are host callable:
// a host test checks them on every fp32 / bf16 magnitude and against IEEE
// division.)
__host__ __device__ __forceinline__ double widen_f32_mag(uint32_t u) {
  const uint32_t a = u & 0x7FFFFFFFu;
  return f64_from_words((a >> 3) + 0x38000000u, a << 29);
}

// The fp64 value of a bf16 magnitude (the low 15 bits of h), built the same
// way: exponent field + 896 (1023 - 127), significand bits moved up.  Exact
// for normal values; zeros and subnormals (exponent field 0) come out as a
// wrong value below 2^-126.
__host__ __device__ __forceinline__ double widen_bf16_mag(uint32_t h) {
  return f64_from_words(((h & 0x7FFFu) << 13) + 0x38000000u, 0u);
}

// *acc += sum |W| in fp64 (grid-stride, 16-byte loads when W allows).
__global__ void __launch_bounds__(256) k_absmean_f64(const float* __restrict__ W, int64_t count,
                                                      double* acc) {
  __shared__ double red[8];
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const bool vec = ((reinterpret_cast<uintptr_t>(W) & 15u) == 0);
  const int64_t nvec = vec ? count / 4 : 0;
  const uint4* W4 = reinterpret_cast<const uint4*>(W);
  // Four independent chains (one per vector lane), so the fp64 adds do not
  // serialise the loop: each chain adds at most count / threads + 1 terms,
  // two more adds join them.
  double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll 4
  for (int64_t i = tid; i < nvec; i += nthreads) {
    const uint4 v = ld_nc_na_v4(W4 + i);
    s0 = __dadd_rn(s0, widen_f32_mag(v.x));
    s1 = __dadd_rn(s1, widen_f32_mag(v.y));
    s2 = __dadd_rn(s2, widen_f32_mag(v.z));
    s3 = __dadd_rn(s3, widen_f32_mag(v.w));
  }
  const uint32_t* Wu = reinterpret_cast<const uint32_t*>(W);
  for (int64_t i = nvec * 4 + tid; i < count; i += nthreads) s0 = __dadd_rn(s0, widen_f32_mag(Wu[i]));
  double s = __dadd_rn(__dadd_rn(s0, s1), __dadd_rn(s2, s3));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = red[0];
    for (int w = 1; w < 8; ++w) t = __dadd_rn(t, red[w]);
    atomicAdd(acc, t);
  }
}

// One thread: gamma from the fp64 sum when the bound decides it (then
// *decided = 1 and *gamma_out is written), else *decided = 0.  h is the
// height of k_absmean_f64's summation tree.
__global__ void k_gamma_decide(const double* __restrict__ acc, int64_t count, int64_t h,
                               float* gamma_out, int* decided) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const double S = *acc;
  const double cnt = static_cast<double>(count);
  const double g = 1.003 * static_cast<double>(h) * 0x1p-53;
  const double B = __dadd_ru(__dmul_ru(g, S), __dmul_ru(cnt, 0x1p-126));
  const float lo = fmaxf(__double2float_rn(__ddiv_rn(fmax(__dsub_rd(S, B), 0.0), cnt)), 1e-5f);
  const float hi = fmaxf(__double2float_rn(__ddiv_rn(__dadd_ru(S, B), cnt)), 1e-5f);
  if (lo == hi) {
    *gamma_out = lo;
    *decided = 1;
  } else {
    *decided = 0;
  }
}

// t = Clip(RNE(RN32(w / gamma)), -1, 1) is +1 exactly when RN32(w / gamma)
// exceeds 0.5 (0.5 itself rounds to the even 0, and anything at or above 1.5
// clips back to 1), -1 exactly when it is below -0.5, else 0.  RN32(q) > 0.5
// exactly when q > 0.5 + 2^-25, the midpoint between 0.5 and the next fp32
// (which rounds to the even 0.5), and RN32 is odd, so with
// T = gamma * (0.5 + 2^-25) -- exact in fp64: 24 x 25 significant bits --
// t = +1 iff w > T and -1 iff w < -T.  For an fp32 w, w > T iff w > RD32(T).
// One comparison per weight replaces the IEEE division.
__host__ __device__ __forceinline__ float ternary_threshold(float gamma) {
  return f32_rd(static_cast<double>(gamma) * (0.5 + 0x1p-25));  // the product is exact
}

__host__ __device__ __forceinline__ uint32_t ternary_code(float w, float thr) {
  return (w > thr) ? 2u : ((w < -thr) ? 0u : 1u);
}

// One packed byte per thread and step: four weights -> four 2-bit codes.
// With K % 4 == 0 (and W 16-byte aligned) packed byte i holds weights
// 4i .. 4i+3 of the flat matrix: one 16-byte load, no row arithmetic.
// Otherwise the row n = i / P and the column are formed per byte.
__global__ void __launch_bounds__(256) k_ternarise_pack2(const float* __restrict__ W, int64_t N,
                                                          int64_t K, const float* __restrict__ gamma_p,
                                                          uint8_t* __restrict__ packed) {
  const int64_t P = (K + 3) / 4;
  const int64_t total = N * P;
  const float thr = ternary_threshold(*gamma_p);
  const bool vec = ((K & 3) == 0) && ((reinterpret_cast<uintptr_t>(W) & 15u) == 0);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  if (vec) {
    const float4* W4 = reinterpret_cast<const float4*>(W);
#pragma unroll 4
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += stride) {
      const float4 v = __ldg(W4 + idx);
      packed[idx] = static_cast<uint8_t>(ternary_code(v.x, thr) | (ternary_code(v.y, thr) << 2) |
                                         (ternary_code(v.z, thr) << 4) | (ternary_code(v.w, thr) << 6));
    }
    return;
  }
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += stride) {
    const int64_t n = idx / P;
    const int64_t b = idx - n * P;
    const int64_t k0 = 4 * b;
    float w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = (k0 + j < K) ? __ldg(W + n * K + k0 + j) : 0.0f;
    uint32_t byte = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t code = (k0 + j < K) ? ternary_code(w[j], thr) : 1u;
      byte |= code << (2 * j);
    }
    packed[idx] = static_cast<uint8_t>(byte);
  }
}

// Base-3 packing of the same trits ("compact ternary packing", [Additive]
// "Energy, Memory Bandwidth, and Serving Economics"; the layout is this
// library's): byte g of a row = sum_j (t_{5g+j} + 1) * 3^j, j = 0..4, trits
// past K are 0, rows of S = 16 * ceil(ceil(K/5) / 16) bytes (padding bytes
// hold five zero trits, 121).  Same ternarisation test as k_ternarise_pack2.
__global__ void __launch_bounds__(256) k_ternarise_pack3(const float* __restrict__ W, int64_t N,
                                                          int64_t K, int64_t S,
                                                          const float* __restrict__ gamma_p,
                                                          uint8_t* __restrict__ packed3) {
  const int64_t total = N * S;
  const float thr = ternary_threshold(*gamma_p);
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / S;
    const int64_t k0 = 5 * (idx - n * S);
    uint32_t byte = 0, pw = 1;
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const uint32_t digit = (k0 + j < K) ? ternary_code(__ldg(W + n * K + k0 + j), thr) : 1u;
      byte += digit * pw;
      pw *= 3u;
    }
    packed3[idx] = static_cast<uint8_t>(byte);
  }
}

}  // namespace bl

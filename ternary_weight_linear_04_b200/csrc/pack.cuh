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
__global__ void __launch_bounds__(256) k_absmean_buckets(const float* __restrict__ W, int64_t count,
                                                          unsigned long long* buckets) {
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
                                 float* gamma_out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
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

// One thread per packed byte: four weights -> four 2-bit codes.
// t = Clip(RNE(RN32(w / gamma)), -1, 1) is +1 exactly when the quotient
// exceeds 0.5 (0.5 itself rounds to the even 0, and anything at or above
// 1.5 clips back to 1), -1 exactly when it is below -0.5, else 0.
__global__ void __launch_bounds__(256) k_ternarise_pack2(const float* __restrict__ W, int64_t N,
                                                          int64_t K, const float* __restrict__ gamma_p,
                                                          uint8_t* __restrict__ packed) {
  const int64_t P = (K + 3) / 4;
  const int64_t total = N * P;
  const float gamma = *gamma_p;
  const bool vec = ((K & 3) == 0) && ((reinterpret_cast<uintptr_t>(W) & 15u) == 0);
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / P;
    const int64_t b = idx - n * P;
    const int64_t k0 = 4 * b;
    float w[4];
    if (vec) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(W + n * K + k0));
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = (k0 + j < K) ? __ldg(W + n * K + k0 + j) : 0.0f;
    }
    uint32_t byte = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t code = 1u;
      if (k0 + j < K) {
        const float q = __fdiv_rn(w[j], gamma);
        code = (q > 0.5f) ? 2u : ((q < -0.5f) ? 0u : 1u);
      }
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
  const float gamma = *gamma_p;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / S;
    const int64_t k0 = 5 * (idx - n * S);
    uint32_t byte = 0, pw = 1;
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      uint32_t digit = 1u;
      if (k0 + j < K) {
        const float q = __fdiv_rn(__ldg(W + n * K + k0 + j), gamma);
        digit = (q > 0.5f) ? 2u : ((q < -0.5f) ? 0u : 1u);
      }
      byte += digit * pw;
      pw *= 3u;
    }
    packed3[idx] = static_cast<uint8_t>(byte);
  }
}

}  // namespace bl

// rmsnorm.cuh -- RMSNorm (no affine, eps 1e-6) fused with the per-token
// absmax int8 quantiser, bf16 activations.
//
// [Production] "2. Absmax Dynamic Activation Quantization" normalises the
// activations with RMSNorm without affine parameters before quantising them,
// and BitLinear158.forward writes it as norm = rsqrt(mean(x^2) + 1e-6),
// x_norm = x * norm.  Readings (every step reproducible bit for bit):
//   * mean(x^2) = RN32(RN64(exact sum of x^2) / K), the division in fp64.
//     The sum is exact whatever the order: a bf16 x is m * 2^(e-134) with an
//     integer m < 2^8 and e its biased exponent (1 for subnormals), so
//     x^2 = m^2 * 2^(2e-268).  With e_max the row's largest exponent and
//     e_base = max(1, e_max - 40), every term with e >= e_base is the integer
//     m^2 * 4^(e - e_base) < 2^96 in units of 2^(2 e_base - 268), summed in a
//     128-bit register per thread and then across the block (K <= 2^24 keeps
//     the total below 2^120).  Terms further down (values below 2^-40 of the
//     row's largest, rare) go to 64-bit shared buckets, one per e.  One
//     thread rounds the exact total once to fp64;
//   * rsqrt(v) = RN32(1 / RN32(sqrt(v))): an IEEE fp32 square root, then an
//     IEEE fp32 division; x_norm = RN32(x * r);
//   * eta = max(max |x_norm|, 1e-5) = max(RN32(max |x| * r), 1e-5) (rounding
//     is monotone), then the fp32 quantiser of quant.cuh on x_norm.
// One 256-thread CTA per token row: pass 0 takes max |x|, pass 1 sums the
// squares, one thread forms the scales, pass 2 quantises (the row is read
// from memory once; the later passes hit L1).
#pragma once

#include "common.cuh"
#include "pack.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kSqLimbs = 20;   // 640 bits; the total stays below 2^563
constexpr int kSqWindow = 40;  // exponents summed in registers below the row's largest

__host__ __device__ inline int clz32(uint32_t v) {
#ifdef __CUDA_ARCH__
  return __clz(v);
#else
  return __builtin_clz(v);
#endif
}

// The nonnegative integer in L[0..n) (32-bit limbs, least significant first)
// times 2^unit_exp, rounded once to fp64, nearest even.
__host__ __device__ inline double limbs_rn64(const uint32_t* L, int n, int unit_exp) {
  int hi = n - 1;
  while (hi >= 0 && L[hi] == 0) --hi;
  if (hi < 0) return 0.0;
  const int top = 32 * hi + 31 - clz32(L[hi]);
  const int lo = top > 52 ? top - 52 : 0;  // lowest of the 53 kept bits
  const int w = lo >> 5;
  unsigned __int128 t = 0;
  for (int i = 2; i >= 0; --i) t = (t << 32) | (w + i < n ? L[w + i] : 0u);
  uint64_t mant = static_cast<uint64_t>(t >> (lo & 31));  // bits above top are zero
  if (lo > 0) {
    const int g = lo - 1;  // guard bit; sticky = any bit below it
    const uint32_t guard = (L[g >> 5] >> (g & 31)) & 1u;
    bool sticky = (L[g >> 5] & ((1u << (g & 31)) - 1u)) != 0;
    for (int i = (g >> 5) - 1; i >= 0 && !sticky; --i) sticky = L[i] != 0;
    if (guard && (sticky || (mant & 1u))) mant += 1;  // 2^53 stays exact
  }
  return scalbn(static_cast<double>(mant), lo + unit_exp);
}

// L += v * 2^pos (v < 2^120, pos >= 0, the sum fitting in n limbs).
__host__ __device__ inline void limbs_add(uint32_t* L, int n, unsigned __int128 v, int pos) {
  const int li = pos >> 5, sh = pos & 31;
  uint32_t part[5];
  const unsigned __int128 lo = v << sh;                             // bits 0..127 of v * 2^sh
  const uint32_t top = sh ? static_cast<uint32_t>(v >> (128 - sh)) : 0u;  // bits 128.. (v < 2^120)
  for (int i = 0; i < 4; ++i) part[i] = static_cast<uint32_t>(lo >> (32 * i));
  part[4] = top;
  uint64_t carry = 0;
  for (int i = 0; li + i < n && (i < 5 || carry); ++i) {
    const uint64_t s = static_cast<uint64_t>(L[li + i]) + (i < 5 ? part[i] : 0u) + carry;
    L[li + i] = static_cast<uint32_t>(s);
    carry = s >> 32;
  }
}

// RN64 of win * 2^(2 wb - 268) + sum_b sb[b] * 2^(2b-268) over b in
// [bmin, bmax] (win < 2^120, sb[b] < 2^48, 1 <= wb, b <= 254).
__host__ __device__ inline double sumsq_rn64(unsigned __int128 win, int wb,
                                             const unsigned long long* sb, int bmin, int bmax) {
  uint32_t L[kSqLimbs];
  for (int i = 0; i < kSqLimbs; ++i) L[i] = 0;
  limbs_add(L, kSqLimbs, win, 2 * wb - 2);  // unit 2^-266
  for (int b = bmin; b <= bmax; ++b)
    if (sb[b]) limbs_add(L, kSqLimbs, sb[b], 2 * b - 2);
  return limbs_rn64(L, kSqLimbs, -266);
}

// RN64 of win * 2^exp2 (win < 2^128).
__host__ __device__ inline double u128_rn64(unsigned __int128 win, int exp2) {
  uint32_t L[4];
  for (int i = 0; i < 4; ++i) L[i] = static_cast<uint32_t>(win >> (32 * i));
  return limbs_rn64(L, 4, exp2);
}

// Bucket and m^2 of one bf16 bit pattern (inf and NaN add nothing).
__device__ __forceinline__ void sq_term(uint32_t h, uint32_t& b, uint32_t& m2) {
  const uint32_t e = (h >> 7) & 0xFFu;
  const uint32_t m = e ? ((h & 0x7Fu) | 0x80u) : (h & 0x7Fu);
  b = e ? e : 1u;
  m2 = e == 0xFFu ? 0u : m * m;
}

__device__ __forceinline__ unsigned __int128 shfl_xor_u128(unsigned __int128 v, int o) {
  const unsigned long long lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<unsigned long long>(v), o);
  const unsigned long long hi =
      __shfl_xor_sync(0xFFFFFFFFu, static_cast<unsigned long long>(v >> 64), o);
  return (static_cast<unsigned __int128>(hi) << 64) | lo;
}

__global__ void __launch_bounds__(256) k_rmsnorm_quant(const __nv_bfloat16* __restrict__ x,
                                                        int64_t M, int64_t K, int vec,
                                                        int8_t* __restrict__ xq,
                                                        float* __restrict__ eta_out,
                                                        int32_t* __restrict__ xsum_out) {
  __shared__ unsigned long long sb[kBuckets];  // terms below the register window
  __shared__ unsigned long long red_lo[8], red_hi[8];
  __shared__ float redf[8];
  __shared__ int32_t redi[8];
  __shared__ int s_tail;
  __shared__ float s_r, s_eta;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t K8 = vec ? K / 8 : 0;
  const uint4* row4 = nullptr;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const __nv_bfloat16* row = x + m * K;
    const uint16_t* rowh = reinterpret_cast<const uint16_t*>(row);
    row4 = reinterpret_cast<const uint4*>(row);
    sb[tid] = 0;  // 256 threads, 256 buckets
    if (tid == 0) s_tail = 0;
    // Pass 0: max |x| as a bf16 magnitude pattern (order-preserving).
    uint32_t hmax = 0;
    if (vec) {
      for (int64_t i = tid; i < K8; i += 256) {
        const uint4 v = __ldg(row4 + i);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          hmax = max(hmax, max(wd[j] & 0x7FFFu, (wd[j] >> 16) & 0x7FFFu));
      }
    } else {
      for (int64_t k = tid; k < K; k += 256) hmax = max(hmax, rowh[k] & 0x7FFFu);
    }
    // Its barriers also order the bucket clearing before pass 1.
    const float amax = block_max_256(__uint_as_float(hmax << 16), redf);
    const int emax = max(1, static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu));
    const int ebase = max(1, emax - kSqWindow);
    // Pass 1: every lane of a warp runs the same trips (the rare bucket add
    // is a warp-wide operation).
    unsigned __int128 acc = 0;
    auto add_term = [&](uint32_t h) {
      uint32_t b, m2;
      sq_term(h, b, m2);
      const bool in_win = static_cast<int>(b) >= ebase;
      if (in_win) acc += static_cast<unsigned __int128>(m2) << (2 * (static_cast<int>(b) - ebase));
      if (__any_sync(0xFFFFFFFFu, !in_win && m2 != 0)) {
        s_tail = 1;
        bucket_add_warp_bm(sb, b, in_win ? 0u : m2);
      }
    };
    if (vec) {
      for (int64_t t = 0; t < (K8 + 255) / 256; ++t) {
        const int64_t i = tid + 256 * t;
        const uint4 v = i < K8 ? __ldg(row4 + i) : make_uint4(0, 0, 0, 0);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          add_term(wd[j] & 0xFFFFu);
          add_term(wd[j] >> 16);
        }
      }
    } else {
      for (int64_t t = 0; t < (K + 255) / 256; ++t) {
        const int64_t k = tid + 256 * t;
        add_term(k < K ? rowh[k] : 0u);
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
      for (int w = 0; w < 8; ++w)
        tot += (static_cast<unsigned __int128>(red_hi[w]) << 64) | red_lo[w];
      const double S = s_tail ? sumsq_rn64(tot, ebase, sb, 1, ebase - 1)
                              : u128_rn64(tot, 2 * ebase - 268);
      const float ms = __double2float_rn(S / static_cast<double>(K));  // IEEE fp64 division
      const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, 1e-6f)));
      s_r = r;
      s_eta = fmaxf(__fmul_rn(amax, r), 1e-5f);
    }
    __syncthreads();
    const float r = s_r, eta = s_eta;
    const float qs = quant_scale(eta);
    int8_t* qrow = xq + m * K;
    int32_t sum = 0;
    if (vec) {
      for (int64_t i = tid; i < K8; i += 256) {
        const uint4 v = __ldg(row4 + i);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
        uint32_t c[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float f = __uint_as_float((wd[j >> 1] >> (16 * (j & 1))) << 16);
          const int32_t q = quantise_fast(__fmul_rn(f, r), eta, qs);
          sum += q;
          c[j] = static_cast<uint32_t>(q);
        }
        reinterpret_cast<uint2*>(qrow)[i] =
            make_uint2(pack_lowbytes(c[0], c[1], c[2], c[3]), pack_lowbytes(c[4], c[5], c[6], c[7]));
      }
    } else {
      for (int64_t k = tid; k < K; k += 256) {
        const float f = __uint_as_float(static_cast<uint32_t>(rowh[k]) << 16);
        const int32_t q = quantise_fast(__fmul_rn(f, r), eta, qs);
        qrow[k] = static_cast<int8_t>(q);
        sum += q;
      }
    }
    sum = block_sum_256(sum, redi);
    if (tid == 0) {
      eta_out[m] = eta;
      xsum_out[m] = sum;
    }
    __syncthreads();  // before the next row clears the buckets
  }
}

}  // namespace bl

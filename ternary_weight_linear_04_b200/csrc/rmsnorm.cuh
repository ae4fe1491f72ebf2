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
//     x^2 = m^2 * 2^(2e-268); the m^2 are added in 64-bit integer buckets,
//     one per e, and one thread forms the total as a 640-bit integer and
//     rounds it once to fp64;
//   * rsqrt(v) = RN32(1 / RN32(sqrt(v))): an IEEE fp32 square root, then an
//     IEEE fp32 division; x_norm = RN32(x * r);
//   * eta = max(max |x_norm|, 1e-5) = max(RN32(max |x| * r), 1e-5) (rounding
//     is monotone), then the fp32 quantiser of quant.cuh on x_norm.
// One 256-thread CTA per token row: pass 1 adds the m^2 into shared buckets
// and takes max |x|; one thread forms the scales; pass 2 quantises.
#pragma once

#include "common.cuh"
#include "pack.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kSqLimbs = 20;  // 640 bits; the total stays below 2^563

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

// RN64 of sum_b sb[b] * 2^(2b-268) over b in [bmin, bmax] (sb[b] < 2^48).
__host__ __device__ inline double sumsq_rn64(const unsigned long long* sb, int bmin, int bmax) {
  uint32_t L[kSqLimbs];
  for (int i = 0; i < kSqLimbs; ++i) L[i] = 0;
  for (int b = bmin; b <= bmax; ++b) {
    const unsigned long long v = sb[b];
    if (!v) continue;
    const int pos = 2 * b - 2;  // unit 2^-266
    const int li = pos >> 5;
    const unsigned __int128 wv = static_cast<unsigned __int128>(v) << (pos & 31);  // < 2^79
    uint64_t carry = 0;
    for (int i = 0; li + i < kSqLimbs && (i < 3 || carry); ++i) {
      const uint64_t part = i < 3 ? static_cast<uint32_t>(wv >> (32 * i)) : 0u;
      const uint64_t s = static_cast<uint64_t>(L[li + i]) + part + carry;
      L[li + i] = static_cast<uint32_t>(s);
      carry = s >> 32;
    }
  }
  return limbs_rn64(L, kSqLimbs, -266);
}

// Bucket and m^2 of one bf16 bit pattern (inf and NaN add nothing).
__device__ __forceinline__ void sq_term(uint32_t h, uint32_t& b, uint32_t& m2) {
  const uint32_t e = (h >> 7) & 0xFFu;
  const uint32_t m = e ? ((h & 0x7Fu) | 0x80u) : (h & 0x7Fu);
  b = e ? e : 1u;
  m2 = e == 0xFFu ? 0u : m * m;
}

__global__ void __launch_bounds__(256) k_rmsnorm_quant(const __nv_bfloat16* __restrict__ x,
                                                        int64_t M, int64_t K, int vec,
                                                        int8_t* __restrict__ xq,
                                                        float* __restrict__ eta_out,
                                                        int32_t* __restrict__ xsum_out) {
  __shared__ unsigned long long sb[kBuckets];
  __shared__ float redf[8];
  __shared__ int32_t redi[8];
  __shared__ float s_r, s_eta;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x;
  const int64_t K8 = vec ? K / 8 : 0;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const __nv_bfloat16* row = x + m * K;
    const uint16_t* rowh = reinterpret_cast<const uint16_t*>(row);
    for (int i = tid; i < kBuckets; i += 256) sb[i] = 0;
    __syncthreads();
    // Pass 1: every lane of a warp runs the same trips (the bucket add is a
    // warp-wide operation).
    uint32_t hmax = 0;  // max |x| as a bf16 magnitude pattern (order-preserving)
    if (vec) {
      const uint4* row4 = reinterpret_cast<const uint4*>(row);
      for (int64_t t = 0; t < (K8 + 255) / 256; ++t) {
        const int64_t i = tid + 256 * t;
        const uint4 v = i < K8 ? __ldg(row4 + i) : make_uint4(0, 0, 0, 0);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t h = (wd[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
          uint32_t b, m2;
          sq_term(h, b, m2);
          hmax = max(hmax, h & 0x7FFFu);
          bucket_add_warp_bm(sb, b, m2);
        }
      }
    } else {
      for (int64_t t = 0; t < (K + 255) / 256; ++t) {
        const int64_t k = tid + 256 * t;
        const uint32_t h = k < K ? rowh[k] : 0u;
        uint32_t b, m2;
        sq_term(h, b, m2);
        hmax = max(hmax, h & 0x7FFFu);
        bucket_add_warp_bm(sb, b, m2);
      }
    }
    // Its barriers also make every bucket add visible.
    const float amax = block_max_256(__uint_as_float(hmax << 16), redf);
    if (tid < 32) {
      uint32_t lmin = kBuckets, lmax = 0;
      for (int b = tid; b < kBuckets; b += 32)
        if (sb[b]) { lmin = min(lmin, static_cast<uint32_t>(b)); lmax = max(lmax, static_cast<uint32_t>(b)); }
      lmin = __reduce_min_sync(0xFFFFFFFFu, lmin);
      lmax = __reduce_max_sync(0xFFFFFFFFu, lmax);
      if (tid == 0) {
        const double S = sumsq_rn64(sb, static_cast<int>(lmin), static_cast<int>(lmax));
        const float ms = __double2float_rn(S / static_cast<double>(K));  // IEEE fp64 division
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, 1e-6f)));
        s_r = r;
        s_eta = fmaxf(__fmul_rn(amax, r), 1e-5f);
      }
    }
    __syncthreads();
    const float r = s_r, eta = s_eta;
    const float qs = quant_scale(eta);
    int8_t* qrow = xq + m * K;
    int32_t sum = 0;
    if (vec) {
      const uint4* row4 = reinterpret_cast<const uint4*>(row);
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

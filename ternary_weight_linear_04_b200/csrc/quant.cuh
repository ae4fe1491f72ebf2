// quant.cuh -- per-token absmax int8 quantisation of activations.
//
// [Production] "2. Absmax Dynamic Activation Quantization" and its
// ActivationQuantizerSTE: eta = per-token max |x| clamped at 1e-5, then
// x~ = Round(x * 127 / eta) with the product and the quotient each rounded
// once in fp32, in that order, and round half to even.  The clip to
// [-127, 127] never binds (the largest |x| maps to exactly 127) but is kept.
// The row sum of x~ is emitted too: the accumulate kernels that feed 2-bit
// codes c = t + 1 straight into integer dot products subtract it back out
// (sum x~ * t = sum x~ * c - sum x~).
#pragma once

#include <cstring>
#include <type_traits>

#include "common.cuh"

namespace bl {

template <typename T>
__device__ __forceinline__ float load_as_f32(const T* p);
template <>
__device__ __forceinline__ float load_as_f32<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_as_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// x~ = clip(RNE(RN32(RN32(x * 127) / eta)), -127, 127), computed exactly but
// without a division per element.  Only the integer RNE(q) is needed, and it
// only depends on which side of the nearest half-integer q falls.  With
// s = RN32(127 * RN32(1/eta)), the product c = RN32(x * s) differs from
// 127x/eta by a relative error of at most 3 roundings, and q = RN32(a/eta)
// (a = RN32(127x)) by at most 2, so |c - q| <= 127 * 5 * 2^-24 < 3.8e-5
// (|x| <= eta).  If c is farther than 2^-14 (6.1e-5) from its nearest
// half-integer, q lies strictly on the same side and RNE(q) = RNE(c);
// otherwise the IEEE quotient itself is formed.  |c| < 127.5, so the clip
// never binds on the fast path.
//
// RNE(c) comes from the fp32 adder, not the conversion unit: for |c| < 2^22,
// t = RN32(c + 1.5 * 2^23) lies on the integer grid of [2^23, 2^24), so t's
// low mantissa bits hold RNE(c) in two's complement (its low byte is the
// int8 code) and t - 1.5 * 2^23 is RNE(c) exactly; c - RNE(c) is exact too
// (the operands are within a factor of two, or RNE(c) = 0).
constexpr float kRneMagic = 12582912.0f;        // 1.5 * 2^23
constexpr uint32_t kRneMagicBits = 0x4B400000u;  // its bit pattern
constexpr float kTieGuard = 0.49993896484375f;   // 0.5 - 2^-14

// The exact quotient, out of line so the common path stays a few instructions
// and the divide is a real (rarely taken) branch rather than predicated code.
__device__ __noinline__ float quotient_exact(float a, float eta) { return __fdiv_rn(a, eta); }

// Scale for the fast path: RN32(127 * RN32(1 / eta)).
__device__ __forceinline__ float quant_scale(float eta) {
  return __fmul_rn(127.0f, __frcp_rn(eta));
}

// The exact code of one value, as the bit pattern of RNE(q) + 1.5 * 2^23.
__device__ __forceinline__ uint32_t quantise_exact_bits(float x, float eta) {
  const float q = quotient_exact(__fmul_rn(x, 127.0f), eta);
  return __float_as_uint(__fadd_rn(fminf(fmaxf(rintf(q), -127.0f), 127.0f), kRneMagic));
}

__device__ __forceinline__ int32_t quantise_fast(float x, float eta, float s) {
  const float c = __fmul_rn(x, s);
  float t = __fadd_rn(c, kRneMagic);
  const float d = __fsub_rn(c, __fsub_rn(t, kRneMagic));
  uint32_t bits = __float_as_uint(t);
  if (fabsf(d) > kTieGuard) bits = quantise_exact_bits(x, eta);
  return static_cast<int32_t>(bits - kRneMagicBits);
}

// bf16 activations, exactly, with no division and no branch.  When x and
// eta are both bf16 values (eta >= 1e-5 is then one of the |x|):
//   * a = 127x is exact in fp32 (8 x 7 significant bits);
//   * for every half-integer h, a/eta is either exactly h or farther from h
//     than 1/(2 * 255 * 2^9), far more than half an fp32 ulp of h (below
//     2^-18): with x = mx 2^ex, eta = me 2^ee (8-bit integers mx, me),
//     a/eta - h is an integer over 2 me 2^max(0, ee-ex), and exponent gaps of
//     10 or more leave |a/eta| < 0.25, away from every h.  So RN32 keeps
//     a/eta on its side of every h, and RNE(RN32(a/eta)) = RNE(a/eta) with
//     ties (a/eta = h exactly) to even;
//   * the fast candidate n0 = RNE(RN32(x * s)) is within 0.5 + 3.8e-5 of
//     a/eta (see above), and e = a - n0 * eta is exact in fp32: n0 * eta has
//     at most 15 significant bits, and the difference spans at most 24 bits
//     (for x far below eta, n0 is 0 or +-1).  One fma forms it.
// So RNE(a/eta) = n0 + 1 if e > eta/2, n0 - 1 if e < -eta/2, and on
// |e| = eta/2 exactly (a tie) the even one of n0 and n0 + sign(e).  The
// result is returned as the bit pattern of RNE + 1.5 * 2^23 (low byte = the
// int8 code); |a/eta| <= 127, so it stays within [-127, 127].
// heta = 0.5 * eta (exact).
__device__ __forceinline__ uint32_t code_bits_bf16(float x, float eta, float heta, float s) {
  const float t = __fadd_rn(__fmul_rn(x, s), kRneMagic);
  const float n0 = __fsub_rn(t, kRneMagic);
  const float e = __fmaf_rn(x, 127.0f, -__fmul_rn(n0, eta));
  uint32_t bits = __float_as_uint(t);
  bits += (e > heta) ? 1u : 0u;
  bits -= (e < -heta) ? 1u : 0u;
  if (fabsf(e) == heta && (bits & 1u)) bits += (e > 0.0f) ? 1u : 0xFFFFFFFFu;
  return bits;
}

// Round-to-nearest fp32 steps callable from host and device, each one IEEE
// operation (no contraction): the device uses the _rn intrinsics, the host
// its own IEEE arithmetic (a host build of this header must not contract,
// e.g. gcc -ffp-contract=off), so the exhaustive host checks of the rules
// below run the same arithmetic as the kernels.
__host__ __device__ __forceinline__ float f32_mul(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}
__host__ __device__ __forceinline__ float f32_sub(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fsub_rn(a, b);
#else
  return a - b;
#endif
}
__host__ __device__ __forceinline__ float f32_fma(float a, float b, float c) {
#ifdef __CUDA_ARCH__
  return __fmaf_rn(a, b, c);
#else
  return fmaf(a, b, c);
#endif
}
__host__ __device__ __forceinline__ uint32_t f32_bits(float v) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(v);
#else
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
#endif
}

// The bf16 quantiser rule of the kernels: x~ = RNE(RN32(RN32(x*127)/eta))
// exactly, with no division, from an approximate reciprocal.  x and eta are
// bf16 values (eta >= 1e-5), heta = eta/2, r approximates 1/eta within
// 2^-21 relative (rcp.approx has 1 ulp) and s = RN32(127 r).  With
// q = 127x/eta (|q| <= 127; 127x and the quotient's RN32 keep q's side of
// every half-integer, see code_bits_bf16):
//   * t = RN32(x s + M), M = 1.5 * 2^23: t - M = n0 is an integer with
//     |n0 - q| < 1 (x s is within 127 (2^-21 + 2^-24) < 7e-5 of q);
//   * e = 127x - n0 eta, exact (one fma; see code_bits_bf16);
//   * RN32(e r + t) rounds M + n0 + e/eta + err, |err| <= |e/eta| 2^-21 <
//     2.5e-7, to an integer, and q = n0 + e/eta.  q is either exactly a half-integer or at least
//     1/(2 * 255 * 2^9) > 3.8e-6 away from every half-integer (the
//     denominator argument of code_bits_bf16; exponent gaps of 10 or more
//     leave |q| < 0.25), so the fp32 adder's rounding to an integer is
//     RNE(q) for every q that is not a tie;
//   * a tie is exactly |e| = eta/2; then the even one of n0 and n0 + sign(e)
//     is taken (t's last significand bit is n0's parity).
// Returns the bit pattern of RNE(q) + M (its low byte is the int8 code).
__host__ __device__ __forceinline__ uint32_t code_bits_bf16_r(float x, float eta, float heta, float s,
                                                              float r) {
  const float t = f32_fma(x, s, kRneMagic);
  const float n0 = f32_sub(t, kRneMagic);
  const float e = f32_fma(-n0, eta, f32_mul(x, 127.0f));
  uint32_t b = f32_bits(f32_fma(e, r, t));
  if (fabsf(e) == heta) {
    const uint32_t tb = f32_bits(t);
    b = (tb & 1u) ? tb + (e > 0.0f ? 1u : 0xFFFFFFFFu) : tb;
  }
  return b;
}

// 1/eta to within 1 ulp (the hardware reciprocal approximation), for the
// candidate and correction of code_bits_bf16_r.
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// Whether v is a bf16 value (its low 16 bits are zero).
__device__ __forceinline__ bool is_bf16_value(float v) {
  return (__float_as_uint(v) & 0xFFFFu) == 0;
}

// One bf16 activation (widened exactly to fp32).  When eta is the 1e-5
// floor rather than a bf16 value (every |x| of the row below 1e-5), the
// argument above does not hold and the code takes the IEEE quotient
// (a uniform branch: eta is shared by the row).
// s = RN32(127 r), r = rcp_approx(eta) (see code_bits_bf16_r).
__device__ __forceinline__ int32_t quantise_bf16(float x, float eta, float heta, float s, float r,
                                                 bool eta_bf16) {
  const uint32_t bits = eta_bf16 ? code_bits_bf16_r(x, eta, heta, s, r) : quantise_exact_bits(x, eta);
  return static_cast<int32_t>(bits - kRneMagicBits);
}

// Low bytes of four words, in order, packed into one word.
__device__ __forceinline__ uint32_t pack_lowbytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Block-wide reductions over NT threads (NT a multiple of 32, at most 1024;
// red holds NT / 32 values).
template <int NT>
__device__ __forceinline__ float block_max_nt(float v, float* red) {
  static_assert(NT % 32 == 0 && NT <= 1024, "whole warps, at most 32");
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < NT / 32) ? red[l] : 0.0f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

template <int NT>
__device__ __forceinline__ int32_t block_sum_nt(int32_t v, int32_t* red) {
  static_assert(NT % 32 == 0 && NT <= 1024, "whole warps, at most 32");
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < NT / 32) ? red[l] : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float block_max_256(float v, float* red) { return block_max_nt<256>(v, red); }
__device__ __forceinline__ int32_t block_sum_256(int32_t v, int32_t* red) {
  return block_sum_nt<256>(v, red);
}

// 8 activations per 16-byte load for bf16, 4 for fp32.
template <typename T>
struct QVec;
template <>
struct QVec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static void store(int8_t* p, const int32_t (&q)[8]) {
    uint2 o;
    o.x = (q[0] & 0xFF) | ((q[1] & 0xFF) << 8) | ((q[2] & 0xFF) << 16) | (static_cast<uint32_t>(q[3]) << 24);
    o.y = (q[4] & 0xFF) | ((q[5] & 0xFF) << 8) | ((q[6] & 0xFF) << 16) | (static_cast<uint32_t>(q[7]) << 24);
    *reinterpret_cast<uint2*>(p) = o;
  }
};
template <>
struct QVec<float> {
  static constexpr int kN = 4;
  __device__ static void load(const float* p, float (&f)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  __device__ static void store(int8_t* p, const int32_t (&q)[4]) {
    *reinterpret_cast<uint32_t*>(p) =
        (q[0] & 0xFF) | ((q[1] & 0xFF) << 8) | ((q[2] & 0xFF) << 16) | (static_cast<uint32_t>(q[3]) << 24);
  }
};

// One NT-thread CTA per token row (NT = 256 for many rows; 1024 for a few
// rows, where the launch is latency: then the 16 values per thread kept in
// registers cover rows up to 16384 bf16 values, and nothing is read twice).
// `vec` = the row can be read with 16-byte loads (K a multiple of the
// vector width, x 16-byte aligned) and xq written with 8/4-byte stores.  The
// first kCache vectors of each thread stay in registers between the absmax
// pass and the quantise pass (all of the row for K up to NT * 8 * kCache
// bf16 values), so the row is read from memory once; longer rows read the
// rest again.
template <typename T, int NT>
__global__ void __launch_bounds__(NT) k_quant_act(const T* __restrict__ x, int64_t M, int64_t K,
                                                   int vec, int8_t* __restrict__ xq,
                                                   float* __restrict__ eta_out,
                                                   int32_t* __restrict__ xsum_out) {
  __shared__ float redf[NT / 32];
  __shared__ int32_t redi[NT / 32];
  constexpr int V = QVec<T>::kN;
  constexpr int kCache = 16 / V;  // 16 values per thread kept in registers
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const T* row = x + m * K;
    int8_t* qrow = xq + m * K;
    float amax = 0.0f;
    float cache[kCache][V];
    if (vec) {
#pragma unroll
      for (int c = 0; c < kCache; ++c) {
        const int64_t k = (static_cast<int64_t>(threadIdx.x) + NT * c) * V;
        if (k < K) {
          QVec<T>::load(row + k, cache[c]);
#pragma unroll
          for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(cache[c][i]));
        }
      }
      for (int64_t k = (static_cast<int64_t>(threadIdx.x) + NT * kCache) * V; k < K; k += NT * V) {
        float f[V];
        QVec<T>::load(row + k, f);
#pragma unroll
        for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(f[i]));
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += NT) amax = fmaxf(amax, fabsf(load_as_f32(row + k)));
    }
    amax = block_max_nt<NT>(amax, redf);
    const float eta = fmaxf(amax, 1e-5f);
    const float qs = kBf16 ? 0.0f : quant_scale(eta);
    const float rr = kBf16 ? rcp_approx(eta) : 0.0f;
    const float rs = __fmul_rn(127.0f, rr);
    const float heta = __fmul_rn(0.5f, eta);
    const bool eta_bf16 = is_bf16_value(eta);
    int32_t sum = 0;
    auto quant_store = [&](int64_t k, const float (&f)[V]) {
      int32_t q[V];
#pragma unroll
      for (int i = 0; i < V; ++i) {
        q[i] = kBf16 ? quantise_bf16(f[i], eta, heta, rs, rr, eta_bf16) : quantise_fast(f[i], eta, qs);
        sum += q[i];
      }
      QVec<T>::store(qrow + k, q);
    };
    if (vec) {
#pragma unroll
      for (int c = 0; c < kCache; ++c) {
        const int64_t k = (static_cast<int64_t>(threadIdx.x) + NT * c) * V;
        if (k < K) quant_store(k, cache[c]);
      }
      for (int64_t k = (static_cast<int64_t>(threadIdx.x) + NT * kCache) * V; k < K; k += NT * V) {
        float f[V];
        QVec<T>::load(row + k, f);
        quant_store(k, f);
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += NT) {
        const float xv = load_as_f32(row + k);
        const int32_t q = kBf16 ? quantise_bf16(xv, eta, heta, rs, rr, eta_bf16) : quantise_fast(xv, eta, qs);
        sum += q;
        qrow[k] = static_cast<int8_t>(q);
      }
    }
    sum = block_sum_nt<NT>(sum, redi);
    if (threadIdx.x == 0) {
      eta_out[m] = eta;
      xsum_out[m] = sum;
    }
  }
}

// The absmax of eight bf16 values (one 16-byte vector) folded into a pair
// of running maxima: the bf16x2 max of the magnitudes, exact (a selection;
// a NaN operand yields the other, as fmaxf does).
__device__ __forceinline__ __nv_bfloat162 absmax8_bf16(__nv_bfloat162 m, const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h;
    const uint32_t a = w[i] & 0x7FFF7FFFu;  // clear both sign bits
    memcpy(&h, &a, 4);
    m = __hmax2(m, h);
  }
  return m;
}

// code_bits_bf16_r for N bf16 values at once (a bf16 eta): the candidate
// and correction run for all N, and the tie test |e| = eta/2 is one vote
// over the N, so only a group holding an exact tie (rare) takes the branch
// that applies the tie rule.  Same bits as code_bits_bf16_r value by value.
// (Host and device: the host check of the rule runs this same code.)
template <int N>
__host__ __device__ __forceinline__ void code_bits_bf16_n(const float (&f)[N], uint32_t (&b)[N],
                                                          float eta, float heta, float s, float r) {
  bool tie = false;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float t = f32_fma(f[i], s, kRneMagic);
    const float n0 = f32_sub(t, kRneMagic);
    const float e = f32_fma(-n0, eta, f32_mul(f[i], 127.0f));
    b[i] = f32_bits(f32_fma(e, r, t));
    tie |= fabsf(e) == heta;
  }
  if (__builtin_expect(tie, 0)) {
#pragma unroll
    for (int i = 0; i < N; ++i) b[i] = code_bits_bf16_r(f[i], eta, heta, s, r);
  }
}

// The codes of eight bf16 values (one 16-byte vector), packed in order
// (byte i of the result = code of value i), for a bf16 eta; the tie vote
// runs over groups of G values (8, or 4 where registers are scarce).
template <int G = 8>
__device__ __forceinline__ uint2 codes8_bf16(const uint4 v, float eta, float heta, float s, float r) {
  static_assert(G == 4 || G == 8, "groups of 4 or 8 values");
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t b[8];
#pragma unroll
  for (int g = 0; g < 8 / G; ++g) {
    float f[G];
    uint32_t bg[G];
#pragma unroll
    for (int i = 0; i < G / 2; ++i) {
      f[2 * i] = __uint_as_float(w[g * G / 2 + i] << 16);
      f[2 * i + 1] = __uint_as_float(w[g * G / 2 + i] & 0xFFFF0000u);
    }
    code_bits_bf16_n<G>(f, bg, eta, heta, s, r);
#pragma unroll
    for (int i = 0; i < G; ++i) b[g * G + i] = bg[i];
  }
  return make_uint2(pack_lowbytes(b[0], b[1], b[2], b[3]), pack_lowbytes(b[4], b[5], b[6], b[7]));
}

// The same eight codes by the IEEE quotient, for a row whose eta is the
// 1e-5 floor (not a bf16 value).
__device__ __forceinline__ uint2 codes8_exact(const uint4 v, float eta) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    b[2 * i] = quantise_exact_bits(__uint_as_float(w[i] << 16), eta);
    b[2 * i + 1] = quantise_exact_bits(__uint_as_float(w[i] & 0xFFFF0000u), eta);
  }
  return make_uint2(pack_lowbytes(b[0], b[1], b[2], b[3]), pack_lowbytes(b[4], b[5], b[6], b[7]));
}

// bf16 rows read with 16-byte loads (K a multiple of 8, x 16-byte and xq
// 8-byte aligned): one NT-thread CTA per token row (grid-stride over rows).
// Each thread keeps its first CV vectors of the row as packed bf16 pairs
// between the absmax pass and the quantise pass (the whole row for K up to
// NT * 8 * CV; longer rows read the rest again), so the per-value work is
// the bf16x2 max, one unpack and the five fp32 operations of the code, and
// the row sum is one dp4a per four codes, added into xsum by one atomic per
// warp (two block barriers fewer per row).  Same results as k_quant_act.
template <int NT, int CV>
__global__ void __launch_bounds__(NT) k_quant_bf16(const __nv_bfloat16* __restrict__ x, int64_t M,
                                                    int64_t K, int8_t* __restrict__ xq,
                                                    float* __restrict__ eta_out,
                                                    int32_t* __restrict__ xsum_out) {
  __shared__ float redf[NT / 32];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t nv = K >> 3;  // 16-byte vectors per row
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
    uint2* qrow = reinterpret_cast<uint2*>(xq + m * K);
    uint4 cache[CV];
    __nv_bfloat162 mx = __float2bfloat162_rn(0.0f);
#pragma unroll
    for (int c = 0; c < CV; ++c) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(NT) * c;
      cache[c] = v < nv ? __ldg(row + v) : make_uint4(0, 0, 0, 0);
      mx = absmax8_bf16(mx, cache[c]);
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(NT) * CV; v < nv; v += NT)
      mx = absmax8_bf16(mx, __ldg(row + v));
    if (threadIdx.x == 0) xsum_out[m] = 0;  // ordered before the warps' adds by the barriers below
    const float amax = block_max_nt<NT>(fmaxf(__low2float(mx), __high2float(mx)), redf);
    const float eta = fmaxf(amax, 1e-5f);
    if (threadIdx.x == 0) eta_out[m] = eta;
    const float r = rcp_approx(eta);
    const float s = __fmul_rn(127.0f, r);
    const float heta = __fmul_rn(0.5f, eta);
    const bool eta_bf16 = is_bf16_value(eta);
    int32_t sum = 0;
    auto emit = [&](int64_t v, const uint4 xv) {
      const uint2 q = eta_bf16 ? codes8_bf16(xv, eta, heta, s, r) : codes8_exact(xv, eta);
      qrow[v] = q;
      sum = __dp4a(static_cast<int>(q.x), 0x01010101, sum);
      sum = __dp4a(static_cast<int>(q.y), 0x01010101, sum);
    };
#pragma unroll
    for (int c = 0; c < CV; ++c) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(NT) * c;
      if (v < nv) emit(v, cache[c]);
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(NT) * CV; v < nv; v += NT) emit(v, __ldg(row + v));
    // The row sum without a block reduction: each warp adds its part with
    // one atomic (integers, so the order of the adds does not matter).
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if ((threadIdx.x & 31) == 0) atomicAdd(xsum_out + m, sum);
  }
}

}  // namespace bl

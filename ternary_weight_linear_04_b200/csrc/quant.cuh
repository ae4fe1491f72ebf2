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
// rcp = RN32(1/eta) the product q' = RN32(a * rcp) is within 2^-23 * |a/eta|
// <= 1.6e-5 of a/eta, and q = RN32(a/eta) within 3.9e-6 of it (|a/eta| <=
// 127), so |q - q'| < 2e-5.  If q' is farther than 2^-14 (6.1e-5) from its
// nearest half-integer, q lies strictly on the same side and RNE(q) =
// RNE(q'); otherwise the IEEE quotient itself is formed.
// The exact quotient, out of line so the common path stays a few instructions
// and the divide is a real (rarely taken) branch rather than predicated code.
__device__ __noinline__ float quotient_exact(float a, float eta) { return __fdiv_rn(a, eta); }

__device__ __forceinline__ int32_t quantise_fast(float x, float eta, float rcp) {
  const float a = __fmul_rn(x, 127.0f);
  float q = __fmul_rn(a, rcp);
  const float fr = q - floorf(q);
  if (fabsf(fr - 0.5f) < 6.103515625e-05f) q = quotient_exact(a, eta);
  const float r = fminf(fmaxf(rintf(q), -127.0f), 127.0f);  // rintf: nearest, ties to even
  return static_cast<int32_t>(r);
}

// The same for 16 values at once, with no branch in the common path: all 16
// candidates are formed first, and only if some lane of the warp has a value
// near a tie does the warp take the (rare) exact fix-up loop.
__device__ __forceinline__ void quantise16(const float (&f)[16], float eta, float rcp,
                                           int32_t (&q)[16]) {
  float a[16];
  uint32_t near = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    a[i] = __fmul_rn(f[i], 127.0f);
    const float c = __fmul_rn(a[i], rcp);
    const float fr = c - floorf(c);
    near |= (fabsf(fr - 0.5f) < 6.103515625e-05f ? 1u : 0u) << i;
    q[i] = static_cast<int32_t>(fminf(fmaxf(rintf(c), -127.0f), 127.0f));
  }
  if (__any_sync(__activemask(), near != 0)) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((near >> i) & 1u) {
        const float c = quotient_exact(a[i], eta);
        q[i] = static_cast<int32_t>(fminf(fmaxf(rintf(c), -127.0f), 127.0f));
      }
    }
  }
}

// Block-wide reductions over 256 threads.
__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < 8) ? red[l] : 0.0f;
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return __shfl_sync(0xFFFFFFFFu, v, 0);
}

__device__ __forceinline__ int32_t block_sum_256(int32_t v, int32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < 8) ? red[l] : 0;
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return __shfl_sync(0xFFFFFFFFu, v, 0);
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

// One 256-thread CTA per token row.  `vec` = the row can be read with
// 16-byte loads (K a multiple of the vector width, x 16-byte aligned) and
// xq written with 8/4-byte stores.
template <typename T>
__global__ void __launch_bounds__(256) k_quant_act(const T* __restrict__ x, int64_t M, int64_t K,
                                                    int vec, int8_t* __restrict__ xq,
                                                    float* __restrict__ eta_out,
                                                    int32_t* __restrict__ xsum_out) {
  __shared__ float redf[8];
  __shared__ int32_t redi[8];
  constexpr int V = QVec<T>::kN;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const T* row = x + m * K;
    int8_t* qrow = xq + m * K;
    float amax = 0.0f;
    if (vec) {
      for (int64_t k = static_cast<int64_t>(threadIdx.x) * V; k < K; k += 256 * V) {
        float f[V];
        QVec<T>::load(row + k, f);
#pragma unroll
        for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(f[i]));
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += 256) amax = fmaxf(amax, fabsf(load_as_f32(row + k)));
    }
    amax = block_max_256(amax, redf);
    const float eta = fmaxf(amax, 1e-5f);
    const float rcp = __frcp_rn(eta);
    int32_t sum = 0;
    if (vec) {
      for (int64_t k = static_cast<int64_t>(threadIdx.x) * V; k < K; k += 256 * V) {
        float f[V];
        QVec<T>::load(row + k, f);
        int32_t q[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
          q[i] = quantise_fast(f[i], eta, rcp);
          sum += q[i];
        }
        QVec<T>::store(qrow + k, q);
      }
    } else {
      for (int64_t k = threadIdx.x; k < K; k += 256) {
        const int32_t q = quantise_fast(load_as_f32(row + k), eta, rcp);
        sum += q;
        qrow[k] = static_cast<int8_t>(q);
      }
    }
    sum = block_sum_256(sum, redi);
    if (threadIdx.x == 0) {
      eta_out[m] = eta;
      xsum_out[m] = sum;
    }
  }
}

}  // namespace bl

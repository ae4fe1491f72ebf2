// gemv.cuh -- decode-time accumulate kernels (small M), CUDA cores.
//
// [Production] "The MatMul-Free Breakthrough" and [Additive] "3. Additive
// Integer Accumulation": y_int[m,n] = sum_{W~=+1} x~ - sum_{W~=-1} x~, with
// zero weights skipped; then the rescale of [Production] pipeline step 5.
//
// At small M the layer is a stream over the packed weights (N*K/4 bytes),
// so the fast kernel is built around HBM: 16-byte non-caching loads of the
// packed rows, several rows per warp in flight, and decode in registers.
// Decode is SIMD-within-a-register: a packed 32-bit word holds 16 codes
// c = t + 1 in {0,1,2}; (word >> 2j) & 0x03030303 lines up the j-th code of
// each of its four bytes, and one dp4a against the matching four int8
// activations adds sum x~ * c for them.  sum x~ * t = sum x~ * c - sum x~,
// so the row sum of x~ (xsum, from the quantiser) is subtracted once at the
// end.  The activations are staged in shared memory with each group of 16
// transposed 4x4 so the bytes dp4a needs are one aligned word.
#pragma once

#include "common.cuh"

namespace bl {

template <typename OutT>
__device__ __forceinline__ void store_out(void* y, int64_t idx, float v);
template <>
__device__ __forceinline__ void store_out<float>(void* y, int64_t idx, float v) {
  static_cast<float*>(y)[idx] = v;
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(void* y, int64_t idx, float v) {
  static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
}

// Fast path.  Needs K % 64 == 0 and 16-byte aligned xq and packed.
// MT tokens (compile time, 1..8), R rows per warp task (1, 2 or 4).
// Dynamic shared memory: MT*K bytes of transposed activations.
template <int MT, int R, typename OutT>
__global__ void __launch_bounds__(256) k_gemv_swar(const int8_t* __restrict__ xq,
                                                    const float* __restrict__ eta,
                                                    const int32_t* __restrict__ xsum, int M,
                                                    int K, const uint8_t* __restrict__ packed,
                                                    const float* __restrict__ gamma_p, int N,
                                                    void* __restrict__ y,
                                                    int32_t* __restrict__ y_int) {
  extern __shared__ __align__(16) uint8_t sx[];
  __shared__ float s_scale[MT];
  __shared__ int32_t s_xsum[MT];

  const int tid = threadIdx.x;
  const int groups = K >> 4;  // 16-activation groups per token
  // Stage x~ (M rows, zero rows beyond M) transposed within each group.
  for (int u = tid; u < MT * groups; u += blockDim.x) {
    const int m = u / groups;
    const int g = u - m * groups;
    uint4 a = make_uint4(0, 0, 0, 0);
    if (m < M) a = __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K) + g);
    uint4 t;
    transpose4x4_bytes(a.x, a.y, a.z, a.w, t.x, t.y, t.z, t.w);
    reinterpret_cast<uint4*>(sx + static_cast<int64_t>(m) * K)[g] = t;
  }
  if (tid < MT) {
    const float gamma = *gamma_p;
    s_scale[tid] = (tid < M) ? token_scale(eta[tid], gamma) : 0.0f;
    s_xsum[tid] = (tid < M) ? xsum[tid] : 0;
  }
  __syncthreads();

  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int P = K >> 2;       // packed bytes per row
  const int C = K >> 6;       // 16-byte packed chunks per row
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int r0 = (blockIdx.x * (blockDim.x >> 5) + warp) * R; r0 < N; r0 += warps_total * R) {
    int32_t acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0;

    for (int c = lane; c < C; c += 32) {
      uint4 p[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        p[r] = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);  // zeros
        if (r0 + r < N)
          p[r] = ld_nc_na_v4(packed + static_cast<int64_t>(r0 + r) * P + 16 * c);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4* xs = reinterpret_cast<const uint4*>(sx + static_cast<int64_t>(m) * K + 64 * c);
        const uint4 x0 = xs[0], x1 = xs[1], x2 = xs[2], x3 = xs[3];
        const uint32_t xw[4][4] = {{x0.x, x0.y, x0.z, x0.w},
                                   {x1.x, x1.y, x1.z, x1.w},
                                   {x2.x, x2.y, x2.z, x2.w},
                                   {x3.x, x3.y, x3.z, x3.w}};
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t pw[4] = {p[r].x, p[r].y, p[r].z, p[r].w};
          int32_t a = acc[r][m];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t codes = (pw[q] >> (2 * j)) & 0x03030303u;
              a = __dp4a(static_cast<int>(codes), static_cast<int>(xw[q][j]), a);
            }
          }
          acc[r][m] = a;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int32_t v = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        acc[r][m] = v;
      }
    // Lane (r*MT + m) writes output (m, r0 + r).
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (lane == ((r * MT + m) & 31) && m < M && r0 + r < N) {
          const int32_t yi = acc[r][m] - s_xsum[m];
          const int64_t o = static_cast<int64_t>(m) * N + r0 + r;
          store_out<OutT>(y, o, rescale(yi, s_scale[m]));
          if (y_int) y_int[o] = yi;
        }
      }
  }
}

// Generic path: any K >= 1, any alignment.  One warp per output row n and
// up to 8 tokens per block row (blockIdx.y); each packed byte is decoded
// code by code with the literal add / subtract / skip.
template <typename OutT>
__global__ void __launch_bounds__(256) k_gemv_generic(const int8_t* __restrict__ xq,
                                                       const float* __restrict__ eta, int64_t M,
                                                       int64_t K,
                                                       const uint8_t* __restrict__ packed,
                                                       const float* __restrict__ gamma_p,
                                                       int64_t N, void* __restrict__ y,
                                                       int32_t* __restrict__ y_int) {
  constexpr int MT = 8;
  const int lane = threadIdx.x & 31;
  const int64_t P = (K + 3) / 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * MT;
  const float gamma = *gamma_p;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N;
       n += warps_total) {
    int32_t acc[MT];
#pragma unroll
    for (int i = 0; i < MT; ++i) acc[i] = 0;
    for (int64_t b = lane; b < P; b += 32) {
      const uint32_t byte = packed[n * P + b];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t k = 4 * b + j;
        if (k >= K) break;
        const uint32_t code = (byte >> (2 * j)) & 3u;
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          if (m0 + i < M) {
            const int32_t xv = xq[(m0 + i) * K + k];
            if (code == 2u) acc[i] += xv;
            else if (code == 0u) acc[i] -= xv;
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      int32_t v = acc[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      if (lane == i && m0 + i < M) {
        const float s = token_scale(eta[m0 + i], gamma);
        const int64_t o = (m0 + i) * N + n;
        store_out<OutT>(y, o, rescale(v, s));
        if (y_int) y_int[o] = v;
      }
    }
  }
}

}  // namespace bl

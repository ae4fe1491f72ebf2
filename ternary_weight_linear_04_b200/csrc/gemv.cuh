// gemv.cuh -- generic accumulate kernel: any K >= 1, any alignment.
//
// [Production] "The MatMul-Free Breakthrough" and [Additive] "3. Additive
// Integer Accumulation": y_int[m,n] = sum_{W~=+1} x~ - sum_{W~=-1} x~, zero
// weights skipped, decoded code by code from the packed bytes exactly as
// [No-Multiply] "Kernel Implementation: The Lookup Table Approach" reads
// them; then the rescale of [Production] pipeline step 5.  Used for ragged
// K or unaligned buffers, where the fast kernels' layout needs are not met.
#pragma once

#include "common.cuh"

namespace bl {

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
  asm volatile("griddepcontrol.wait;" ::: "memory");
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

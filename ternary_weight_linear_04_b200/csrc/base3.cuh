// base3.cuh -- few-token accumulate kernel on base-3 packed weights.
//
// The same layer as decode.cuh ([Production] "The MatMul-Free Breakthrough":
// y_int = sum_{W~=+1} x~ - sum_{W~=-1} x~; pipeline step 5 rescale) on the
// compact ternary packing ([Additive] "Energy, Memory Bandwidth, and Serving
// Economics": five trits per byte, 1.6 bits per weight), the measured
// alternative to the 2-bit codes: 20 % fewer weight bytes, a costlier decode.
//
// A byte is decoded through a 243-entry table in shared memory: entry b
// holds the five base-3 digits of b (digit = t + 1 in {0, 1, 2}) as bytes,
// four in .x and the fifth in .y, so two dp4a against the matching five
// activations (kept as an 8-byte slot per group of five) add sum x~ * c for
// the group; sum x~ * t = sum x~ * c - sum x~ (padding trits are 0, digit 1,
// against zero activations).  Each warp takes 4 rows at a time; its lanes
// stride over the rows in 16-byte chunks (80 trits) read straight from
// global memory, 64 bytes in flight per lane; a transposed warp reduction
// gives each (row, token) total to one lane, which rescales and stores.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace bl {

constexpr int kG3Warps = 8;
constexpr int kG3Rows = 4;

// Arguments of one k_gemv3 launch (MT tokens starting at xq).
struct G3Launch {
  const int8_t* xq;
  const float* eta;
  const int32_t* xsum;
  int M, K, S;
  const uint8_t* packed3;
  const float* gamma;
  int N;
  void* y;
  int32_t* y_int;
};

__device__ __forceinline__ uint4 ld_nc_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// MT tokens (1, 2, 4) of x~ starting at xq (row stride K); rows of packed3
// have stride S (a multiple of 16).
template <int MT, typename OutT>
__global__ void __launch_bounds__(32 * kG3Warps) k_gemv3(
    const int8_t* __restrict__ xq, const float* __restrict__ eta, const int32_t* __restrict__ xsum,
    int M, int K, int S, const uint8_t* __restrict__ packed3, const float* __restrict__ gamma_p,
    int N, void* __restrict__ y, int32_t* __restrict__ y_int) {
  constexpr int V = kG3Rows * MT;
  extern __shared__ __align__(128) uint8_t smem[];
  uint2* lut = reinterpret_cast<uint2*>(smem);             // 256 entries
  uint2* xs = reinterpret_cast<uint2*>(smem + 256 * 8);    // [MT][S] activation slots
  float* s_scale = reinterpret_cast<float*>(xs + MT * S);
  int32_t* s_xsum = reinterpret_cast<int32_t*>(s_scale + MT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // digits of every byte value (entries 243..255 never occur; zeros)
  for (int b = tid; b < 256; b += blockDim.x) {
    uint32_t d[5], v = static_cast<uint32_t>(b);
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      d[j] = v % 3u;
      v /= 3u;
    }
    lut[b] = b < 243 ? make_uint2(d[0] | (d[1] << 8) | (d[2] << 16) | (d[3] << 24), d[4])
                     : make_uint2(0u, 0u);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int i = tid; i < MT * S; i += blockDim.x) {
    const int m = i / S, g = i - m * S;
    uint32_t lo = 0, hi = 0;
    if (m < M) {
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        const int k = 5 * g + j;
        const uint32_t v = k < K ? static_cast<uint8_t>(xq[static_cast<int64_t>(m) * K + k]) : 0u;
        if (j < 4) lo |= v << (8 * j);
        else hi = v;
      }
    }
    xs[i] = make_uint2(lo, hi);
  }
  if (tid < MT) {
    const float gamma = *gamma_p;
    s_scale[tid] = tid < M ? token_scale(eta[tid], gamma) : 0.0f;
    s_xsum[tid] = tid < M ? xsum[tid] : 0;
  }
  __syncthreads();

  const int nchunk = S / 16;
  for (int r0 = (blockIdx.x * kG3Warps + warp) * kG3Rows; r0 < N;
       r0 += gridDim.x * kG3Warps * kG3Rows) {
    int32_t acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0;
    const uint8_t* rows[kG3Rows];
#pragma unroll
    for (int r = 0; r < kG3Rows; ++r) rows[r] = packed3 + static_cast<int64_t>(min(r0 + r, N - 1)) * S;
    for (int c = lane; c < nchunk; c += 32) {
      uint4 pw[kG3Rows];
#pragma unroll
      for (int r = 0; r < kG3Rows; ++r) pw[r] = ld_nc_v4(rows[r] + 16 * c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {        // 32-bit word of the chunk
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {   // byte of the word
          const int g = 16 * c + 4 * q + bb;
          uint2 xv[MT];
#pragma unroll
          for (int m = 0; m < MT; ++m) xv[m] = xs[m * S + g];
#pragma unroll
          for (int r = 0; r < kG3Rows; ++r) {
            const uint32_t wq = q == 0 ? pw[r].x : (q == 1 ? pw[r].y : (q == 2 ? pw[r].z : pw[r].w));
            const uint2 l = lut[(wq >> (8 * bb)) & 0xFFu];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              acc[r * MT + m] = __dp4a(static_cast<int>(l.x), static_cast<int>(xv[m].x), acc[r * MT + m]);
              acc[r * MT + m] = __dp4a(static_cast<int>(l.y), static_cast<int>(xv[m].y), acc[r * MT + m]);
            }
          }
        }
      }
    }
    const int32_t tot = warp_transpose_sum<V>(acc, lane);
    constexpr int kGroup = 32 / V;
    if ((lane & (kGroup - 1)) == 0) {
      const int vi = lane >> ilog2(kGroup);
      const int r = vi / MT, m = vi - r * MT;
      const int n = r0 + r;
      if (n < N && m < M) {
        const int32_t yi = tot - s_xsum[m];
        const int64_t o = static_cast<int64_t>(m) * N + n;
        store_out<OutT>(y, o, rescale(yi, s_scale[m]));
        if (y_int) y_int[o] = yi;
      }
    }
  }
}

}  // namespace bl

// decode.cuh -- decode-time accumulate kernel (M <= 4 tokens), CUDA cores,
// packed weights streamed into shared memory by bulk copies (TMA engine).
//
// [Production] "The MatMul-Free Breakthrough" and [Additive] "3. Additive
// Integer Accumulation": y_int[m,n] = sum_{W~=+1} x~ - sum_{W~=-1} x~ (zeros
// skipped); [Production] pipeline step 5: y = y_int * (eta*gamma)/127.
// Optionally fused with the quantiser of [Production] "2. Absmax Dynamic
// Activation Quantization" (each CTA quantises the few activation rows it
// needs itself, so decode is one kernel per layer).
//
// At a few tokens the layer is a stream over the packed weights (N*K/4
// bytes), so the kernel is organised around HBM:
//   * CTA b owns a contiguous block of rows; one producer warp moves it into
//     a ring of shared-memory stages with cp.async.bulk (one copy per stage,
//     many KB in flight per SM, no register cost);
//   * when the caller declares the weights static, the first stages are
//     requested before griddepcontrol.wait, so under programmatic dependent
//     launch the weight stream overlaps the previous kernel's tail;
//   * 8 compute warps decode four rows at a time: a packed 32-bit word holds
//     16 codes c = t + 1 in {0,1,2}; (word >> 2j) & 0x03030303 lines up the
//     j-th code of each byte and one dp4a adds sum x~ * c for four of them;
//     sum x~ * t = sum x~ * c - sum x~, so xsum is subtracted once at the end;
//   * activations live in shared memory transposed 4x4 within each group of
//     16 (so dp4a's four bytes are one word) and stored plane by plane, so a
//     warp's 16-byte reads are consecutive (no bank conflicts).
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kDecStageBytes = 16384;
constexpr int kDecStages = 4;
constexpr int kDecComputeWarps = 8;
constexpr int kDecThreads = 32 * (kDecComputeWarps + 1);

__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch: wait for the preceding grid (and its memory)
// / allow the next grid to launch.  No-ops when launched without the
// attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Shared offset of activation group g (16 values) of one token, in bytes,
// in the plane layout: plane q = g % 4 holds groups 4cc + q at cc * 16.
__device__ __forceinline__ int dec_group_off(int g, int C) { return ((g & 3) * C + (g >> 2)) * 16; }

template <typename XT>
struct DecLoad16;
template <>
struct DecLoad16<__nv_bfloat16> {
  __device__ static void load(const __nv_bfloat16* p, float (&f)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    const uint4 a = __ldg(q), b = __ldg(q + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct DecLoad16<float> {
  __device__ static void load(const float* p, float (&f)[16]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(q + i);
      f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
    }
  }
};

// Reduction across the 256 compute threads (named barrier 1).
__device__ __forceinline__ float dec_block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  named_sync(1, 32 * kDecComputeWarps);
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kDecComputeWarps; ++i) r = fmaxf(r, red[i]);
  named_sync(1, 32 * kDecComputeWarps);
  return r;
}

__device__ __forceinline__ int32_t dec_block_sum(int32_t v, int32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  named_sync(1, 32 * kDecComputeWarps);
  int32_t r = 0;
#pragma unroll
  for (int i = 0; i < kDecComputeWarps; ++i) r += red[i];
  named_sync(1, 32 * kDecComputeWarps);
  return r;
}

__device__ __forceinline__ uint32_t pack4_i8(int32_t a, int32_t b, int32_t c, int32_t d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | (static_cast<uint32_t>(d) << 24);
}

struct DecodeArgs {
  const void* x;         // activations (FUSED) or x~ (int8), M x K
  const float* eta;      // !FUSED: per-token scales
  const int32_t* xsum;   // !FUSED: per-token sums of x~
  int M, K, N;
  const uint8_t* packed;
  const float* gamma;
  void* y;
  int32_t* y_int;        // optional
  int rows_per_cta;
  int weights_static;
  int8_t* xq_out;        // FUSED, optional: CTA 0 writes x~, eta, xsum
  float* eta_out;
  int32_t* xsum_out;
};

template <int MT>
struct DecSmem {
  static size_t bytes(int K) {
    const size_t xs = (static_cast<size_t>(MT) * K + 127) & ~static_cast<size_t>(127);
    return xs + static_cast<size_t>(kDecStages) * kDecStageBytes + 2 * 8 * kDecStages + 16 +
           8 * MT + 4 * 2 * kDecComputeWarps + 64;
  }
};

// CTAs resident per SM: two for one or two tokens (room for the next kernel's
// CTAs to start streaming under programmatic dependent launch), one above.
template <int MT>
struct DecOcc {
  static constexpr int kCtasPerSm = MT <= 2 ? 2 : 1;
};

template <int MT, bool FUSED, typename XT, typename OutT>
__global__ void __launch_bounds__(kDecThreads, DecOcc<MT>::kCtasPerSm) k_decode(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = a.K, C = K >> 6, P = K >> 2;
  uint8_t* sx = smem;
  uint8_t* stages = smem + ((static_cast<size_t>(MT) * K + 127) & ~static_cast<size_t>(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kDecStages * kDecStageBytes);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDecStages);
  float* s_scale = reinterpret_cast<float*>(empty + kDecStages) + 4;
  int32_t* s_xsum = reinterpret_cast<int32_t*>(s_scale + MT);
  float* s_redf = reinterpret_cast<float*>(s_xsum + MT);
  int32_t* s_redi = reinterpret_cast<int32_t*>(s_redf + kDecComputeWarps);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_begin = blockIdx.x * a.rows_per_cta;
  const int r_end = min(a.N, r_begin + a.rows_per_cta);
  const int nrows = r_end - r_begin;
  const int rps = min(nrows, kDecStageBytes / P);  // whole rows per stage
  const int nchunks = nrows > 0 ? (nrows + rps - 1) / rps : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kDecComputeWarps);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  pdl_trigger();  // the next grid may launch; it waits for our completion before reading y

  if (warp == kDecComputeWarps) {
    // ------------------------------------------------ producer warp
    if (lane == 0) {
      auto issue = [&](int c) {
        const int s = c % kDecStages;
        const int rows = min(rps, nrows - c * rps);
        const uint32_t bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(P);
        mbar_arrive_expect_tx(full + s, bytes);
        bulk_load_1d(stages + s * kDecStageBytes,
                     a.packed + static_cast<int64_t>(r_begin + c * rps) * P, bytes, full + s);
      };
      const int first = min(kDecStages, nchunks);
      if (a.weights_static)
        for (int c = 0; c < first; ++c) issue(c);
      pdl_wait();
      if (!a.weights_static)
        for (int c = 0; c < first; ++c) issue(c);
      for (int c = kDecStages; c < nchunks; ++c) {
        const int s = c % kDecStages;
        if (!mbar_wait(empty + s, static_cast<uint32_t>(c / kDecStages - 1) & 1u, abort_flag)) break;
        issue(c);
      }
    }
    return;  // the compute warps synchronise among themselves only (barrier 1)
  }

  // ------------------------------------------------ compute warps (256 threads)
  pdl_wait();
  const int tid = threadIdx.x;
  const int groups = K >> 4;
  const float gamma = *a.gamma;
  if constexpr (FUSED) {
    const XT* x = static_cast<const XT*>(a.x);
    for (int m = 0; m < MT; ++m) {
      if (m >= a.M) {  // unused token slot: zeros
        for (int g = tid; g < groups; g += 32 * kDecComputeWarps)
          *reinterpret_cast<uint4*>(sx + m * K + dec_group_off(g, C)) = make_uint4(0, 0, 0, 0);
        if (tid == 0) { s_scale[m] = 0.0f; s_xsum[m] = 0; }
        continue;
      }
      const XT* row = x + static_cast<int64_t>(m) * K;
      float amax = 0.0f;
      for (int g = tid; g < groups; g += 32 * kDecComputeWarps) {
        float f[16];
        DecLoad16<XT>::load(row + 16 * g, f);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
      }
      amax = dec_block_max(amax, s_redf);
      const float eta = fmaxf(amax, 1e-5f);
      const float rcp = __frcp_rn(eta);
      int32_t sum = 0;
      for (int g = tid; g < groups; g += 32 * kDecComputeWarps) {
        float f[16];
        DecLoad16<XT>::load(row + 16 * g, f);
        int32_t q[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          q[i] = quantise_fast(f[i], eta, rcp);
          sum += q[i];
        }
        const uint32_t w0 = pack4_i8(q[0], q[1], q[2], q[3]);
        const uint32_t w1 = pack4_i8(q[4], q[5], q[6], q[7]);
        const uint32_t w2 = pack4_i8(q[8], q[9], q[10], q[11]);
        const uint32_t w3 = pack4_i8(q[12], q[13], q[14], q[15]);
        if (a.xq_out && blockIdx.x == 0)
          *reinterpret_cast<uint4*>(a.xq_out + static_cast<int64_t>(m) * K + 16 * g) =
              make_uint4(w0, w1, w2, w3);
        uint4 t;
        transpose4x4_bytes(w0, w1, w2, w3, t.x, t.y, t.z, t.w);
        *reinterpret_cast<uint4*>(sx + m * K + dec_group_off(g, C)) = t;
      }
      sum = dec_block_sum(sum, s_redi);
      if (tid == 0) {
        s_scale[m] = token_scale(eta, gamma);
        s_xsum[m] = sum;
        if (blockIdx.x == 0) {
          if (a.eta_out) a.eta_out[m] = eta;
          if (a.xsum_out) a.xsum_out[m] = sum;
        }
      }
    }
  } else {
    const int8_t* xq = static_cast<const int8_t*>(a.x);
    for (int u = tid; u < MT * groups; u += 32 * kDecComputeWarps) {
      const int m = u / groups;
      const int g = u - m * groups;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m < a.M) v = __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K) + g);
      uint4 t;
      transpose4x4_bytes(v.x, v.y, v.z, v.w, t.x, t.y, t.z, t.w);
      *reinterpret_cast<uint4*>(sx + m * K + dec_group_off(g, C)) = t;
    }
    if (tid < MT) {
      s_scale[tid] = (tid < a.M) ? token_scale(a.eta[tid], gamma) : 0.0f;
      s_xsum[tid] = (tid < a.M) ? a.xsum[tid] : 0;
    }
  }
  named_sync(1, 32 * kDecComputeWarps);

  for (int c = 0; c < nchunks; ++c) {
    const int s = c % kDecStages;
    const bool ok =
        __all_sync(0xFFFFFFFFu, mbar_wait(full + s, static_cast<uint32_t>(c / kDecStages) & 1u, abort_flag));
    if (!ok) break;
    const uint8_t* st = stages + s * kDecStageBytes;
    const int rows = min(rps, nrows - c * rps);
    for (int rr = warp * 4; rr < rows; rr += 4 * kDecComputeWarps) {
      int32_t acc[4][MT];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[i][m] = 0;
      for (int cc = lane; cc < C; cc += 32) {
        uint4 p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          p[i] = (rr + i < rows) ? *reinterpret_cast<const uint4*>(st + (rr + i) * P + 16 * cc)
                                 : make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          uint32_t xw[4][4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = *reinterpret_cast<const uint4*>(sx + m * K + (q * C + cc) * 16);
            xw[q][0] = v.x; xw[q][1] = v.y; xw[q][2] = v.z; xw[q][3] = v.w;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t pw[4] = {p[i].x, p[i].y, p[i].z, p[i].w};
            int32_t t = acc[i][m];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int j = 0; j < 4; ++j)
                t = __dp4a(static_cast<int>((pw[q] >> (2 * j)) & 0x03030303u),
                           static_cast<int>(xw[q][j]), t);
            acc[i][m] = t;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int32_t v = acc[i][m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
          acc[i][m] = v;
        }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int n = r_begin + c * rps + rr + i;
          if (lane == i * MT + m && rr + i < rows && m < a.M) {
            const int32_t yi = acc[i][m] - s_xsum[m];
            const int64_t o = static_cast<int64_t>(m) * a.N + n;
            store_out<OutT>(a.y, o, rescale(yi, s_scale[m]));
            if (a.y_int) a.y_int[o] = yi;
          }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + s);
  }
}

}  // namespace bl

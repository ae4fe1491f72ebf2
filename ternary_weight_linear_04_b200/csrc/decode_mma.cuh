// decode_mma.cuh -- the accumulate for a few tokens (9 to 16) with each CTA's
// weights in registers and the products on the warp-level tensor-core MMA
// (mma.sync m16n8k32, s8 x s8 -> s32).
//
// [Production] "The MatMul-Free Breakthrough" (y_int = the sum of x~ where
// W~ = +1 minus the sum where W~ = -1, here as sum c * x~ - sum x~ with the
// codes c = W~ + 1) and pipeline step 5 (y = y_int * (eta * gamma) / 127),
// for a decode batch whose x~, eta and xsum are given.  The integer sums are
// exact whatever the order, so the result is the oracle's bit for bit.
//
// Why this instruction: at 9..16 tokens each weight feeds few products.
// dp4a does 4 of them per lane and instruction (256 per cycle per SM);
// mma.sync m16n8k32 does 4096 per warp instruction and issues about one per
// two cycles per SM (measured: 2048 int8 products per cycle per SM), without
// the tensor-memory and mbarrier hand-offs that a tcgen05 pipeline needs per
// tile, which at these sizes cost more than the products.
//
// Layout (one CTA of 16 warps per SM, the rows of the one-token geometry):
//   * the CTA's rows (at most 64) form RBK blocks of 16; warp w takes block
//     w % RBK and K part w / RBK of KP = 16 / RBK parts, NS steps of 64 K;
//   * lane (g, q) = (lane / 4, lane % 4) holds, per step, the 32-bit packed
//     words 4s + q of rows g and g + 8 of its block (16 codes each), loaded
//     before griddepcontrol.wait when the weights are static;
//   * A operand: plane j = (w >> 2j) & 0x03030303 of a word holds codes
//     j, 4+j, 8+j, 12+j in its bytes.  MMA 1 of a step takes planes 0 and 1,
//     MMA 2 planes 2 and 3, so the K order inside a step is a permutation the
//     B operand repeats: the transposed slots (byte b of slot word j =
//     activation 16 w + 4 b + j) give lane (g, q) its B registers for token g
//     of a tile and word 4s + q with one 16-byte load (words j = 0, 1 for MMA
//     1, 2, 3 for MMA 2);
//   * tokens in tiles of 8 (the MMA's N); the token stride of the slots is
//     padded to 4 mod 8 slots, so the 16-byte loads of a quarter-warp (two
//     tokens, four words) hit eight different bank groups;
//   * the KP partial 16 x 8 tiles of a block go through shared memory, laid
//     out [K part][token][CTA row] with the token stride padded to 4 mod 32
//     words: the fragment stores of a warp fall in 32 different banks and
//     the reads, consecutive rows of one token per warp, in consecutive
//     banks; after one barrier each thread adds the parts of one (row,
//     token), subtracts xsum, rescales and stores.
// Every CTA stages the whole of x~ (M x K bytes, from L2): at 16 tokens and
// K = 8640 that is 138 KB per CTA, 20 MB of L2 reads per launch, three
// times the weight bytes, which is why the kernel stops at 16 tokens (32
// token slots measured slower than the tensor-core kernel, whose split K
// reads only its share of x~).
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace bl {

constexpr int kMmaThreads = 512;
constexpr int kMmaMaxTokens = 16;

struct MmaDecodeArgs {
  const int8_t* xq;        // M x K
  const float* eta;        // M
  const int32_t* xsum;     // M
  int M, K, N;
  const uint8_t* packed;
  const float* gamma;
  void* y;                 // M x N, fp32 or bf16 (y_bf16)
  int y_bf16;
  int32_t* y_int;          // optional
  int rows_per_cta;        // <= 16 * RBK
  int weights_static;
};

// Slots per token, padded to 4 mod 8 (see above).
__host__ __device__ constexpr int mma_slot_stride(int nw) { return ((nw + 3) / 8) * 8 + 4; }

// Words per token of the partial tiles: the CTA's 16 RBK rows, plus 4.
__host__ __device__ constexpr int mma_part_stride(int rbk) { return 16 * rbk + 4; }

// Shared memory: NT8 * 8 tokens x stride slots of 16 bytes, then the partial
// tiles: KP = 16 / RBK parts x NT8 * 8 tokens x mma_part_stride(RBK) int32.
__host__ __device__ constexpr size_t mma_decode_smem(int nt8, int rbk, int K) {
  return static_cast<size_t>(nt8) * 8 * mma_slot_stride(K / 16) * 16 +
         static_cast<size_t>(16 / rbk) * nt8 * 8 * mma_part_stride(rbk) * 4;
}

__device__ __forceinline__ void mma_s8_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ld_nc_na_b32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// NT8 tiles of 8 tokens (M <= 8 NT8; up to 8 tokens the register kernel of
// decode_reg.cuh is the faster), RBK row blocks of 16 (rows per CTA <=
// 16 RBK), NS steps of 64 K per warp (K <= 64 NS * 16 / RBK).
template <int NT8, int RBK, int NS>
__global__ void __launch_bounds__(kMmaThreads, 1) k_decode_mma(const MmaDecodeArgs a) {
  static_assert(NT8 == 2 || NT8 == 4, "16 or 32 token slots");
  static_assert(RBK == 1 || RBK == 2 || RBK == 4, "1, 2 or 4 row blocks");
  constexpr int KP = 16 / RBK;
  constexpr int T = NT8 * 8;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float s_scale[T];
  __shared__ int32_t s_xsum[T];
  const int K = a.K, NW = K >> 4, P = K >> 2, M = a.M;
  const int stride = mma_slot_stride(NW);
  uint4* xslot = reinterpret_cast<uint4*>(smem);
  int32_t* part = reinterpret_cast<int32_t*>(smem + static_cast<size_t>(T) * stride * 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int rb = warp % RBK, kp = warp / RBK;
  const int r_begin = blockIdx.x * a.rows_per_cta;
  const int nrows = max(0, min(a.N - r_begin, a.rows_per_cta));
  const int w0 = kp * NS * 4;  // this warp's first packed word along K

  // Rows g and g + 8 of this warp's block (rows past the CTA's repeat its
  // last one; words past K/16 are zero codes against zero slots).
  uint32_t wa[NS], wb[NS];
  auto load_weights = [&]() {
    const int ra = min(16 * rb + g, max(nrows - 1, 0));
    const int rbw = min(16 * rb + g + 8, max(nrows - 1, 0));
    const uint8_t* pa = a.packed + static_cast<int64_t>(r_begin + ra) * P;
    const uint8_t* pb = a.packed + static_cast<int64_t>(r_begin + rbw) * P;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int wi = w0 + 4 * s + q;
      const bool in = nrows > 0 && wi < NW;
      wa[s] = in ? ld_nc_na_b32(pa + 4 * wi) : 0u;
      wb[s] = in ? ld_nc_na_b32(pb + 4 * wi) : 0u;
    }
  };
  float gamma = 0.0f;
  if (a.weights_static) {
    load_weights();
    gamma = __ldg(a.gamma);
  }
  pdl_wait();  // the previous kernel is complete and its writes are visible
  if (tid == 0) pdl_trigger();
  if (!a.weights_static) {
    load_weights();
    gamma = __ldg(a.gamma);
  }

  // x~ slots, transposed (byte b of slot word j = activation 16 w + 4 b + j),
  // token t at slots t * stride ..; tokens past M and words past K/16 zero.
  // Every 16-byte copy of the real rows is in flight at once (cp.async,
  // L2-resident rows), then each thread transposes the slots it copied.
  const int real = M * stride;
  for (int qd = tid; qd < T * stride; qd += kMmaThreads) {
    const int t = qd / stride, w = qd - t * stride;
    if (t < M && w < NW)
      cp_async_16(xslot + qd, reinterpret_cast<const uint4*>(a.xq + static_cast<int64_t>(t) * K) + w);
    else
      xslot[qd] = make_uint4(0, 0, 0, 0);
  }
  cp_async_wait_all();
  for (int qd = tid; qd < real; qd += kMmaThreads) {
    const uint4 v = xslot[qd];
    uint4 o;
    transpose4x4_bytes(v.x, v.y, v.z, v.w, o.x, o.y, o.z, o.w);
    xslot[qd] = o;
  }
  if (tid < T) {
    s_scale[tid] = tid < M ? token_scale(a.eta[tid], gamma) : 0.0f;
    s_xsum[tid] = tid < M ? a.xsum[tid] : 0;
  }
  __syncthreads();

  int c[NT8][4];
#pragma unroll
  for (int n = 0; n < NT8; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const uint32_t ua = wa[s], ub = wb[s];
    const uint32_t a0 = ua & 0x03030303u, b0p = ub & 0x03030303u;
    const uint32_t a1 = (ua >> 2) & 0x03030303u, b1p = (ub >> 2) & 0x03030303u;
    const uint32_t a2 = (ua >> 4) & 0x03030303u, b2p = (ub >> 4) & 0x03030303u;
    const uint32_t a3 = (ua >> 6) & 0x03030303u, b3p = (ub >> 6) & 0x03030303u;
    const int w = w0 + 4 * s + q;  // slot of lane (g, q) in this step
#pragma unroll
    for (int n = 0; n < NT8; ++n) {
      const uint4 xv = xslot[(8 * n + g) * stride + w];
      // fragment rows: registers 0, 2 = row g, 1, 3 = row g + 8; K slots
      // 4q..4q+3 (registers 0, 1) and 16+4q.. (registers 2, 3)
      mma_s8_16832(c[n], a0, b0p, a1, b1p, xv.x, xv.y);
      mma_s8_16832(c[n], a2, b2p, a3, b3p, xv.z, xv.w);
    }
  }
  // C fragment: c0, c1 = row g, tokens 2q, 2q+1; c2, c3 = row g + 8.
  // part[kp][token T][CTA row, stride PS]
  constexpr int PS = mma_part_stride(RBK);
  int32_t* pp = part + static_cast<size_t>(kp) * T * PS + 16 * rb + g;
#pragma unroll
  for (int n = 0; n < NT8; ++n) {
    const int t0 = 8 * n + 2 * q;
    pp[t0 * PS] = c[n][0];
    pp[(t0 + 1) * PS] = c[n][1];
    pp[t0 * PS + 8] = c[n][2];
    pp[(t0 + 1) * PS + 8] = c[n][3];
  }
  __syncthreads();
  // One (row, token) per thread and round: rows fastest, so the stores of a
  // token's outputs are contiguous.
  for (int e = tid; e < 16 * RBK * T; e += kMmaThreads) {
    const int t = e / (16 * RBK), row = e - t * (16 * RBK);
    if (row >= nrows || t >= M) continue;
    int32_t tot = 0;
#pragma unroll
    for (int k = 0; k < KP; ++k) tot += part[(static_cast<size_t>(k) * T + t) * PS + row];
    const int32_t yi = tot - s_xsum[t];
    const int64_t o = static_cast<int64_t>(t) * a.N + r_begin + row;
    const float yv = rescale(yi, s_scale[t]);
    if (a.y_bf16) store_out<__nv_bfloat16>(a.y, o, yv);
    else store_out<float>(a.y, o, yv);
    if (a.y_int) a.y_int[o] = yi;
  }
}

}  // namespace bl

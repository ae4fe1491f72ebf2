// decode_reg.cuh -- the one-token layer with each CTA's weights held in
// registers: quantise + accumulate + rescale in one kernel.
//
// [Production] "2. Absmax Dynamic Activation Quantization" (per-token absmax,
// x~ = RNE(x * 127 / eta)), "The MatMul-Free Breakthrough" (y_int = sum of x~
// where W~ = +1 minus the sum where W~ = -1) and pipeline step 5 (y = y_int *
// (eta * gamma) / 127), for one token at decoder layer sizes.
//
// One token is a stream over the packed weights, and a layer of a decoder is
// short enough that its dependency chain (wait for the previous layer, read
// and quantise x, accumulate, store) sets its time, not the bandwidth.  This
// kernel keeps that chain short:
//   * the CTA's rows are cut into blocks of RB rows, one block per warp (16
//     warps, at most 16 * RB rows per CTA); lane l of a warp holds the 32-bit
//     words l, l + 32, ... (NJ of them) of each of its RB rows in registers;
//   * with static weights those loads (and gamma) are issued before
//     griddepcontrol.wait, so they stream while the previous kernel runs;
//     there is no shared-memory ring, no bulk copy and no barrier on them;
//   * after the wait every thread reads its 16-byte chunks of x from global
//     memory, the block takes max |x| (one __syncthreads), and each thread
//     quantises its own chunks with the division-free exact rule of
//     code_bits_bf16_r into 16-byte slots (byte b of slot word j =
//     activation 4b + j of its group of 16), one more __syncthreads;
//   * the accumulate is SIMD within a register as in decode.cuh (planes
//     w & 0x03030303, w & 0x0C0C0C0C and the same on w >> 4 against the
//     matching slot words, sum x~ c - sum x~ = sum x~ t), then a transposed
//     warp reduction leaves each row total on one lane, which rescales and
//     stores it.
// 512 threads and at most 56 registers each (the launch bound names 576
// threads so that the compiler keeps to 56): the next layer's CTA must fit
// on the SM beside this one under programmatic dependent launch, and the
// register file is split over four sub-partitions of 16K registers, each
// holding a quarter of a CTA's warps.  The shared-memory decode kernel puts
// five of its 17 warps (56 registers) on one sub-partition, 8960
// registers; four warps of this kernel at 64 registers (8192) would not fit
// beside them, at 56 (7168) they do.  Measured on a 70B-class layer's seven
// projections chained under dependent launch: 104 us with the cap, 142 us at
// 64 registers (every switch between the two kernels then lost the overlap).
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "quant.cuh"

namespace bl {

constexpr int kRegThreads = 512;

struct RegDecodeArgs {
  const __nv_bfloat16* x;  // one token, K values
  int K, N;
  const uint8_t* packed;
  const float* gamma;
  void* y;                 // 1 x N, fp32 or bf16 (y_bf16)
  int y_bf16;
  int32_t* y_int;          // optional
  int rows_per_cta;        // <= 16 * RB
  int weights_static;
  int8_t* xq_out;          // optional: CTA 0 writes x~, eta, xsum
  float* eta_out;
  int32_t* xsum_out;
};

// The codes of one 16-byte chunk of bf16 activations when eta is the 1e-5
// floor (not a bf16 value): IEEE quotients.  Out of line: rare, and kept out
// of the registers of the common path.
__device__ __noinline__ uint2 quantise_chunk_exact(uint4 v, float eta) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  uint32_t q[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    q[2 * j] = quantise_exact_bits(__uint_as_float(u[j] << 16), eta);
    q[2 * j + 1] = quantise_exact_bits(__uint_as_float(u[j] & 0xFFFF0000u), eta);
  }
  return make_uint2(pack_lowbytes(q[0], q[1], q[2], q[3]), pack_lowbytes(q[4], q[5], q[6], q[7]));
}

__device__ __forceinline__ uint32_t ld_nc_na_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// NJ words per lane and row (K <= 512 NJ), RB rows per warp.  Shared
// memory: 32 NJ slots of 16 bytes.
template <int RB, int NJ>
__global__ void __launch_bounds__(kRegThreads + 64, 2) k_decode_reg(const RegDecodeArgs a) {
  static_assert(RB == 1 || RB == 2 || RB == 4, "RB rows per warp: 1, 2 or 4");
  constexpr int XC = (NJ + 7) / 8;  // 16-byte chunks of x per thread
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t s_max[16];
  __shared__ int32_t s_xs[16];
  __shared__ float s_scale;
  uint4* xslot = reinterpret_cast<uint4*>(smem);
  const int K = a.K, NW = K >> 4, P = K >> 2;
  constexpr int NWP = 32 * NJ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r_begin = blockIdx.x * a.rows_per_cta;
  const int nrows = max(0, min(a.N - r_begin, a.rows_per_cta));
  const int row0 = warp * RB;

  // This warp's rows (padding rows repeat the last one; padding words are
  // code 01, a zero weight, against zeroed activation slots).
  uint32_t wreg[RB][NJ];
  auto load_weights = [&]() {
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int row = min(row0 + r, max(nrows - 1, 0));
      const uint8_t* rp = a.packed + static_cast<int64_t>(r_begin + row) * P;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int wi = lane + 32 * j;
        wreg[r][j] = (nrows > 0 && wi < NW) ? ld_nc_na_u32(rp + 4 * wi) : 0x55555555u;
      }
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

  // x: 16-byte chunks tid + 512 i; max |x| per element (bit patterns of
  // non-negative bf16 values order like the values).  The chunks are read
  // again (from L1) to quantise them, which keeps registers for the weights.
  const int nch = K >> 3;
  const uint4* x4 = reinterpret_cast<const uint4*>(a.x);
  uint32_t amax = 0;
#pragma unroll
  for (int i = 0; i < XC; ++i) {
    const int c = tid + kRegThreads * i;
    const uint4 v = c < nch ? x4[c] : make_uint4(0, 0, 0, 0);
    const uint32_t w4[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
#pragma unroll
    for (int j = 0; j < 4; ++j) amax = max(amax, max(w4[j] << 16, w4[j] & 0xFFFF0000u));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) s_max[warp] = amax;
  for (int w = NW + tid; w < NWP; w += kRegThreads) xslot[w] = make_uint4(0, 0, 0, 0);
  __syncthreads();

  uint32_t e = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) e = max(e, s_max[i]);
  const float eta = fmaxf(__uint_as_float(e), 1e-5f);
  const float rr = rcp_approx(eta);
  const float qs = __fmul_rn(127.0f, rr);
  const float heta = __fmul_rn(0.5f, eta);
  const bool eta_bf16 = is_bf16_value(eta);  // else eta is the 1e-5 floor: exact quotients
  const bool write_xq = a.xq_out != nullptr && blockIdx.x == 0;
  int32_t psum = 0;
#pragma unroll
  for (int i = 0; i < XC; ++i) {
    const int c = tid + kRegThreads * i;
    if (c < nch) {
      const uint4 v = x4[c];
      uint32_t lo, hi;
      if (eta_bf16) {
        // value by value (the grouped tie vote of codes8_bf16 takes more
        // registers than this kernel's budget leaves, and measured slower)
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t q[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          q[2 * j] = code_bits_bf16_r(__uint_as_float(u[j] << 16), eta, heta, qs, rr);
          q[2 * j + 1] = code_bits_bf16_r(__uint_as_float(u[j] & 0xFFFF0000u), eta, heta, qs, rr);
        }
        lo = pack_lowbytes(q[0], q[1], q[2], q[3]);
        hi = pack_lowbytes(q[4], q[5], q[6], q[7]);
      } else {
        const uint2 lh = quantise_chunk_exact(v, eta);
        lo = lh.x;
        hi = lh.y;
      }
      psum = __dp4a(static_cast<int>(lo), 0x01010101, psum);
      psum = __dp4a(static_cast<int>(hi), 0x01010101, psum);
      if (write_xq) *reinterpret_cast<uint2*>(a.xq_out + 8 * c) = make_uint2(lo, hi);
      // chunk c is half h = c & 1 of slot c >> 1: its bytes j (lo) and j (hi)
      // go to slot word j, bytes 2h and 2h + 1
      uint8_t* sl = smem + (c >> 1) * 16 + 2 * (c & 1);
      *reinterpret_cast<uint16_t*>(sl + 0) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0040));
      *reinterpret_cast<uint16_t*>(sl + 4) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0051));
      *reinterpret_cast<uint16_t*>(sl + 8) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0062));
      *reinterpret_cast<uint16_t*>(sl + 12) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0073));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xFFFFFFFFu, psum, o);
  if (lane == 0) s_xs[warp] = psum;
  if (tid == 0) {
    s_scale = token_scale(eta, gamma);
    if (blockIdx.x == 0 && a.eta_out) a.eta_out[0] = eta;
  }
  __syncthreads();
  int32_t xsum = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) xsum += s_xs[i];
  if (tid == 0 && blockIdx.x == 0 && a.xsum_out) a.xsum_out[0] = xsum;
  if (row0 >= nrows) return;  // whole warps
  const float sc = s_scale;

  int32_t acc1[RB], acc4[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    acc1[r] = 0;
    acc4[r] = 0;
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const uint4 xv = xslot[lane + 32 * j];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const uint32_t pw = wreg[r][j];
      const uint32_t h = pw >> 4;
      acc1[r] = __dp4a(static_cast<int>(pw & 0x03030303u), static_cast<int>(xv.x), acc1[r]);
      acc4[r] = __dp4a(static_cast<int>(pw & 0x0C0C0C0Cu), static_cast<int>(xv.y), acc4[r]);
      acc1[r] = __dp4a(static_cast<int>(h & 0x03030303u), static_cast<int>(xv.z), acc1[r]);
      acc4[r] = __dp4a(static_cast<int>(h & 0x0C0C0C0Cu), static_cast<int>(xv.w), acc4[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < RB; ++r) acc1[r] += acc4[r] >> 2;  // acc4 is a multiple of 4
  const int32_t tot = warp_transpose_sum<RB>(acc1, lane);
  constexpr int kGroup = 32 / RB;
  const int vi = lane >> ilog2(kGroup);
  if ((lane & (kGroup - 1)) == 0 && row0 + vi < nrows) {
    const int32_t yi = tot - xsum;
    const int64_t o = r_begin + row0 + vi;
    const float yv = rescale(yi, sc);
    if (a.y_bf16) store_out<__nv_bfloat16>(a.y, o, yv);
    else store_out<float>(a.y, o, yv);
    if (a.y_int) a.y_int[o] = yi;
  }
}

// ---------------------------------------------------------------------------
// The same register-resident layout for 2 to 8 tokens whose x~, eta and
// xsum are given (the quantiser ran before, or the caller passes x~):
// [Production] "The MatMul-Free Breakthrough" and pipeline step 5 for a few
// decode tokens at once.
//   * weights as above: RB rows per warp, NJ words per lane and row, loaded
//     before griddepcontrol.wait when static;
//   * after the wait every thread stages its share of the MT x~ rows (all
//     16-byte loads issued together) into transposed slots, one set per
//     token; rows past M and words past K/16 are zeros;
//   * per word, the tokens go in pairs: two slot loads, then for each row the
//     four planes (w >> 2i) & 0x03030303 (code 4b + i in byte b, matching slot
//     word i) and 8 dp4a.  The planes are recomputed per pair rather than
//     kept, which holds the registers to weights + RB * MT accumulators + two
//     slots (at most 128, no spills at the instantiated shapes).  One CTA per
//     SM: in a decode layer the next launch is the quantiser's few CTAs,
//     which fit beside it, and this kernel's weights stream while they run;
//   * a transposed warp sum over the RB * MT values (up to 32, one per lane)
//     leaves each (row, token) total on one lane, which subtracts xsum,
//     rescales and stores it.
struct RegMultiArgs {
  const int8_t* xq;        // M x K (x~ given)
  const float* eta;        // M
  const int32_t* xsum;     // M
  const __nv_bfloat16* x;  // M x K (fused: quantised by every CTA)
  int8_t* xq_out;          // fused, optional: CTA 0 writes x~, eta, xsum
  float* eta_out;
  int32_t* xsum_out;
  int M, K, N;
  const uint8_t* packed;
  const float* gamma;
  void* y;                 // M x N, fp32 or bf16 (y_bf16)
  int y_bf16;
  int32_t* y_int;          // optional
  int rows_per_cta;        // <= 16 * RB
  int weights_static;
};

constexpr int kRegMultiMaxMT = 8;

// MT tokens (2, 4 or 8; M <= MT), RB rows per warp (RB * MT <= 32), NJ words
// per lane and row; FUSE: the CTA quantises the bf16 rows itself (used for
// two tokens: from three on the separate quantiser launch is cheaper).  Shared
// memory: MT * 32 NJ slots of 16 bytes.
template <int MT, int RB, int NJ, bool FUSE>
__global__ void __launch_bounds__(kRegThreads, 1) k_decode_regm(const RegMultiArgs a) {
  static_assert(MT == 2 || MT == 4 || MT == 8, "2, 4 or 8 tokens");
  static_assert(RB == 1 || RB == 2 || RB == 4, "RB rows per warp: 1, 2 or 4");
  constexpr int NWP = 32 * NJ;                           // slot words per token
  constexpr int XI = (MT * NWP + kRegThreads - 1) / kRegThreads;  // slots per thread
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float s_scale[MT];
  __shared__ int32_t s_xsum[MT];
  uint4* xslot = reinterpret_cast<uint4*>(smem);
  const int K = a.K, NW = K >> 4, P = K >> 2, M = a.M;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r_begin = blockIdx.x * a.rows_per_cta;
  const int nrows = max(0, min(a.N - r_begin, a.rows_per_cta));
  const int row0 = warp * RB;

  uint32_t wreg[RB][NJ];
  auto load_weights = [&]() {
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int row = min(row0 + r, max(nrows - 1, 0));
      const uint8_t* rp = a.packed + static_cast<int64_t>(r_begin + row) * P;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int wi = lane + 32 * j;
        wreg[r][j] = (nrows > 0 && wi < NW) ? ld_nc_na_u32(rp + 4 * wi) : 0x55555555u;
      }
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

  if constexpr (FUSE) {
    // The quantiser of [Production] "2. Absmax Dynamic Activation
    // Quantization" for every row, in every CTA: G = 16 / MT warps per
    // token; pass 1 takes max |x| (bit patterns of non-negative bf16 values
    // order like the values), pass 2 reads the chunks again (from L1),
    // quantises them with the division-free exact rule of code_bits_bf16_r
    // and scatters the codes into the transposed slots; padding words and
    // tokens stay zero.
    constexpr int G = 16 / MT;
    constexpr int XCF = (2 * NJ + G - 1) / G;  // 8-value chunks per thread and token (K <= 512 NJ)
    __shared__ uint32_t s_max[16];
    const int m = warp / G;                    // this warp's token
    const int gt = (warp - m * G) * 32 + lane;  // thread within the token's warps
    const int nch = K >> 3;
    const uint4* x4 = reinterpret_cast<const uint4*>(a.x + static_cast<int64_t>(m) * K);
    for (int i = tid; i < MT * NWP; i += kRegThreads) xslot[i] = make_uint4(0, 0, 0, 0);
    if (tid < MT) s_xsum[tid] = 0;
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < XCF; ++i) {
      const int c = gt + 32 * G * i;
      const uint4 v = (m < M && c < nch) ? x4[c] : make_uint4(0, 0, 0, 0);
      const uint32_t w4[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
#pragma unroll
      for (int k = 0; k < 4; ++k) amax = max(amax, max(w4[k] << 16, w4[k] & 0xFFFF0000u));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) s_max[warp] = amax;
    __syncthreads();  // also orders the zeroed slots before the scatter below
    uint32_t e = 0;
#pragma unroll
    for (int i = 0; i < G; ++i) e = max(e, s_max[m * G + i]);
    const float eta = fmaxf(__uint_as_float(e), 1e-5f);
    const float rr = rcp_approx(eta);
    const float qs = __fmul_rn(127.0f, rr);
    const float heta = __fmul_rn(0.5f, eta);
    const bool eta_bf16 = is_bf16_value(eta);  // else eta is the 1e-5 floor: exact quotients
    const bool write_xq = a.xq_out != nullptr && blockIdx.x == 0;
    int32_t psum = 0;
#pragma unroll
    for (int i = 0; i < XCF; ++i) {
      const int c = gt + 32 * G * i;
      if (m < M && c < nch) {
        const uint4 v = x4[c];
        uint32_t lo, hi;
        if (eta_bf16) {
          const uint2 q8 = codes8_bf16<4>(v, eta, heta, qs, rr);
          lo = q8.x;
          hi = q8.y;
        } else {
          const uint2 lh = quantise_chunk_exact(v, eta);
          lo = lh.x;
          hi = lh.y;
        }
        psum = __dp4a(static_cast<int>(lo), 0x01010101, psum);
        psum = __dp4a(static_cast<int>(hi), 0x01010101, psum);
        if (write_xq) *reinterpret_cast<uint2*>(a.xq_out + static_cast<int64_t>(m) * K + 8 * c) = make_uint2(lo, hi);
        // chunk c is half h = c & 1 of slot c >> 1 of token m: its bytes j
        // (lo) and j (hi) go to slot word j, bytes 2h and 2h + 1
        uint8_t* sl = smem + (static_cast<size_t>(m) * NWP + (c >> 1)) * 16 + 2 * (c & 1);
        *reinterpret_cast<uint16_t*>(sl + 0) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0040));
        *reinterpret_cast<uint16_t*>(sl + 4) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0051));
        *reinterpret_cast<uint16_t*>(sl + 8) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0062));
        *reinterpret_cast<uint16_t*>(sl + 12) = static_cast<uint16_t>(__byte_perm(lo, hi, 0x0073));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xFFFFFFFFu, psum, o);
    if (lane == 0 && m < M && psum != 0) atomicAdd(&s_xsum[m], psum);
    if (gt == 0 && m < M) {
      s_scale[m] = token_scale(eta, gamma);
      if (blockIdx.x == 0 && a.eta_out) a.eta_out[m] = eta;
    }
    __syncthreads();
    if (blockIdx.x == 0 && a.xsum_out && tid < M) a.xsum_out[tid] = s_xsum[tid];
  } else {
    // x~ slots: slot q = m * NWP + w holds the 16 activations of word w of
    // token m, transposed (byte b of slot word i = activation 16 w + 4 b + i).
    uint4 v[XI];
#pragma unroll
    for (int i = 0; i < XI; ++i) {
      const int q = tid + kRegThreads * i;
      const int m = q / NWP, w = q - m * NWP;
      v[i] = (q < MT * NWP && m < M && w < NW)
                 ? __ldg(reinterpret_cast<const uint4*>(a.xq + static_cast<int64_t>(m) * K) + w)
                 : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < XI; ++i) {
      const int q = tid + kRegThreads * i;
      if (q < MT * NWP) {
        uint4 t;
        transpose4x4_bytes(v[i].x, v[i].y, v[i].z, v[i].w, t.x, t.y, t.z, t.w);
        xslot[q] = t;
      }
    }
    if (tid < MT) {
      s_scale[tid] = tid < M ? token_scale(a.eta[tid], gamma) : 0.0f;
      s_xsum[tid] = tid < M ? a.xsum[tid] : 0;
    }
    __syncthreads();
  }

  if (row0 >= nrows) return;  // whole warps

  constexpr int V = RB * MT;
  int32_t acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
#pragma unroll
    for (int mp = 0; mp < MT; mp += 2) {
      const uint4 xa = xslot[mp * NWP + lane + 32 * j];
      const uint4 xb = xslot[(mp + 1) * NWP + lane + 32 * j];
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const uint32_t w = wreg[r][j];
        const int p0 = static_cast<int>(w & 0x03030303u);
        const int p1 = static_cast<int>((w >> 2) & 0x03030303u);
        const int p2 = static_cast<int>((w >> 4) & 0x03030303u);
        const int p3 = static_cast<int>((w >> 6) & 0x03030303u);
        int32_t ta = acc[r * MT + mp], tb = acc[r * MT + mp + 1];
        ta = __dp4a(p0, static_cast<int>(xa.x), ta);
        tb = __dp4a(p0, static_cast<int>(xb.x), tb);
        ta = __dp4a(p1, static_cast<int>(xa.y), ta);
        tb = __dp4a(p1, static_cast<int>(xb.y), tb);
        ta = __dp4a(p2, static_cast<int>(xa.z), ta);
        tb = __dp4a(p2, static_cast<int>(xb.z), tb);
        ta = __dp4a(p3, static_cast<int>(xa.w), ta);
        tb = __dp4a(p3, static_cast<int>(xb.w), tb);
        acc[r * MT + mp] = ta;
        acc[r * MT + mp + 1] = tb;
      }
    }
  }
  const int32_t tot = warp_transpose_sum<V>(acc, lane);
  constexpr int kGroup = 32 / V;
  const int vi = lane >> ilog2(kGroup);  // value held: row vi / MT, token vi % MT
  const int r = vi / MT, m = vi - r * MT;
  if ((lane & (kGroup - 1)) == 0 && row0 + r < nrows && m < M) {
    const int32_t yi = tot - s_xsum[m];
    const int64_t o = static_cast<int64_t>(m) * a.N + r_begin + row0 + r;
    const float yv = rescale(yi, s_scale[m]);
    if (a.y_bf16) store_out<__nv_bfloat16>(a.y, o, yv);
    else store_out<float>(a.y, o, yv);
    if (a.y_int) a.y_int[o] = yi;
  }
}

}  // namespace bl

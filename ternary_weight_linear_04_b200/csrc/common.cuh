// common.cuh -- shared device helpers for the BitLinear kernels (sm_100a).
//
// Inline PTX wrappers written from the public PTX ISA for mbarriers, bulk
// tensor copies (TMA) and the 5th-generation tensor core (tcgen05).  Every
// wait on a barrier is bounded: it polls %globaltimer and gives up after
// kWaitLimitNs, recording BL_ERR_TIMEOUT in the library's device error word,
// so a bug can never leave a GPU spinning forever.
#pragma once

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace bl {

// Device-side error word of the library (one per device): a kernel that
// gives up a wait stores a non-zero status here; bitlinear_device_error()
// reads and clears it.
__device__ int g_device_error;

#ifdef BL_TEST_HOOKS
// Fault-injection build used only by the timeout test: waits give up after
// 1 ms, and g_test_fault (set by bitlinear_test_set_fault) makes a kernel
// withhold one barrier arrival so that a wait runs out.
constexpr unsigned long long kWaitLimitNs = 1000000ull;  // 1 ms per wait
__device__ int g_test_fault;
#else
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait
#endif

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async proxy (TMA, tensor core).
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false (and records BL_ERR_TIMEOUT) if it does not complete within
// kWaitLimitNs, or immediately if *abort is already set.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      g_device_error = 5;  // BL_ERR_TIMEOUT
      *abort = 1;
      return false;
    }
  }
}

// After an abort: wait for a phase that an asynchronous copy or a tensor-core
// commit already issued by this CTA will complete, so that nothing is still
// writing into this CTA's shared memory (or reading its TMEM) when it exits.
// Ignores the abort flag; bounded by kWaitLimitNs like every other wait.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2D tiled bulk tensor load global -> shared (this CTA), completion counted
// in bytes on `bar`.  c0 is the innermost coordinate (in elements).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 16-byte asynchronous copy global -> shared through the load/store path
// (L2 only), and the wait for all of this thread's copies.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Generic-proxy writes to shared memory -> visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- clusters

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster arrives and waits (threads that
// have exited count as arrived).  Release/acquire: shared-memory writes
// before it, local or into another CTA's shared memory, are visible after.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// The address of this CTA's shared-memory location `p` in CTA `rank` of the
// cluster (same layout in every CTA).
__device__ __forceinline__ uint32_t cluster_map(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::i8, one CTA.
__device__ __forceinline__ void tc_mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::i8, one CTA.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this
// thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bit, 8 consecutive columns per thread.
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand in the 128-byte
// swizzle layout: rows of 128 bytes, 8-row atoms of 1024 bytes stacked with
// stride SBO = 1024 bytes; the 16-byte chunk index within a row is XORed
// with the row index within its atom.  Fields (PTX ISA, tcgen05 shared
// memory descriptor): start address >> 4 in bits 0-13, leading byte offset
// >> 4 in bits 16-29 (unused for swizzled K-major, set to 1), stride byte
// offset >> 4 in bits 32-45, version 1 in bits 46-47, base offset 0 (atoms
// 1024-byte aligned), swizzle mode 2 (128B) in bits 61-63.
__device__ __forceinline__ uint64_t make_sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor for tcgen05.mma kind::i8: s32 accumulate, A and B
// signed 8-bit, both K-major, shape M x N (M in {64,128}; N = 8 or a
// multiple of 16 in [16, 256]).  Bits: c_format 4-5 (2 = s32), a_format 7-9
// (1 = s8), b_format 10-12 (1 = s8), a/b major 15/16 (0 = K), N>>3 in 17-22,
// M>>4 in 24-28.
__host__ __device__ constexpr uint32_t make_idesc_i8(uint32_t M, uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// The same with A unsigned 8-bit (a_format 0) and B signed 8-bit.
__host__ __device__ constexpr uint32_t make_idesc_i8_u8s8(uint32_t M, uint32_t N) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ---------------------------------------------------------------- misc

__device__ __forceinline__ uint4 ld_nc_na_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 4x4 byte transpose of four words: out[j] byte i = in[i] byte j.
__device__ __forceinline__ void transpose4x4_bytes(uint32_t a0, uint32_t a1, uint32_t a2,
                                                   uint32_t a3, uint32_t& o0, uint32_t& o1,
                                                   uint32_t& o2, uint32_t& o3) {
  const uint32_t u0 = __byte_perm(a0, a1, 0x5140);  // a0.b0 a1.b0 a0.b1 a1.b1
  const uint32_t u1 = __byte_perm(a2, a3, 0x5140);  // a2.b0 a3.b0 a2.b1 a3.b1
  const uint32_t u2 = __byte_perm(a0, a1, 0x7362);  // a0.b2 a1.b2 a0.b3 a1.b3
  const uint32_t u3 = __byte_perm(a2, a3, 0x7362);  // a2.b2 a3.b2 a2.b3 a3.b3
  o0 = __byte_perm(u0, u1, 0x5410);
  o1 = __byte_perm(u0, u1, 0x7632);
  o2 = __byte_perm(u2, u3, 0x5410);
  o3 = __byte_perm(u2, u3, 0x7632);
}

// RN32(a / 127) without a divide: y = RN32(1/127), q0 = RN32(a y), the
// remainder a - 127 q0 is exact (one fma), and RN32(q0 + (a - 127 q0) y) is
// the correctly rounded quotient (P. Markstein, "IA-64 and Elementary
// Functions", 2000: a faithful quotient corrected with the exact remainder
// and the correctly rounded reciprocal).  Host callable; a host test checks
// it against IEEE division for every normal fp32 a >= 2^-119 (a / 127 normal).
__host__ __device__ __forceinline__ float div127_rn(float a) {
  constexpr float kInv127 = 1.0f / 127.0f;  // RN32(1/127), folded at compile time
#ifdef __CUDA_ARCH__
  const float q0 = __fmul_rn(a, kInv127);
  return __fmaf_rn(__fmaf_rn(-q0, 127.0f, a), kInv127, q0);
#else
  const float q0 = a * kInv127;
  return fmaf(fmaf(-q0, 127.0f, a), kInv127, q0);
#endif
}

// The fp64 value with high word hi and low word lo (host and device).
__host__ __device__ __forceinline__ double f64_from_words(uint32_t hi, uint32_t lo) {
#ifdef __CUDA_ARCH__
  return __hiloint2double(static_cast<int>(hi), static_cast<int>(lo));
#else
  const uint64_t u = (static_cast<uint64_t>(hi) << 32) | lo;
  double d;
  memcpy(&d, &u, 8);
  return d;
#endif
}

// RD32(x): the largest fp32 not above the fp64 x (host and device).
__host__ __device__ __forceinline__ float f32_rd(double x) {
#ifdef __CUDA_ARCH__
  return __double2float_rd(x);
#else
  float f = static_cast<float>(x);  // nearest
  if (static_cast<double>(f) > x) f = nextafterf(f, -INFINITY);
  return f;
#endif
}

// Rescale epilogue: s_m = RN32(RN32(eta_m * gamma) / 127) (computed once per
// token), y = RN32(RN32(float(y_int)) * s_m).  Each step is a single IEEE
// rounding (no contraction into an FMA).
__device__ __forceinline__ float token_scale(float eta, float gamma) {
  return div127_rn(__fmul_rn(eta, gamma));
}

__device__ __forceinline__ float rescale(int32_t y_int, float s) {
  return __fmul_rn(__int2float_rn(y_int), s);
}

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

}  // namespace bl

/*
 * bitlinear.h -- C ABI of the BitNet b1.58 BitLinear forward pass on one
 * NVIDIA B200 (sm_100a).
 *
 * The layer, as the pages define it (cited by title and section):
 *   [Production]  "BitNet b1.58 & 1-Bit LLMs in Production: Ternary
 *                 Quantization, MatMul-Free Kernels, and Edge AI Silicon
 *                 Deployment"
 *   [Additive]    "1-Bit Large Language Models and BitNet b1.58: How Ternary
 *                 Weights and Additive Kernels Eliminate Matrix
 *                 Multiplications"
 *   [No-Multiply] "BitNet b1.58: Ternary Weight LLMs That Eliminate Matrix
 *                 Multiplication"
 *
 *   gamma   = max(mean |W|, 1e-5)                 whole N x K matrix
 *   W~      = Clip(Round(W / gamma), -1, +1)      round half to even
 *   eta_m   = max(max_k |x[m,k]|, 1e-5)           per token m
 *   x~      = Clip(Round((x * 127) / eta_m), -127, 127)   int8
 *   y_int   = sum_{W~=+1} x~ - sum_{W~=-1} x~     int32, zeros skipped
 *   y       = y_int * ((eta_m * gamma) / 127)     fp32, or rounded to bf16
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller (for
 *     example torch tensors); the library allocates nothing and keeps no
 *     reference after the call returns.  Scratch space, where one is needed,
 *     is passed in by the caller.
 *   - Tensors are dense and row-major: W is N x K (out_features x
 *     in_features), x and x~ are M x K, y and y_int are M x N.
 *   - Every call is asynchronous on the CUDA stream `stream` (a cudaStream_t
 *     passed as void*; NULL = the legacy default stream) and never
 *     synchronises with the host.  gamma and eta stay on the device.
 *   - Arguments are checked before anything is launched.  A bad argument
 *     returns an error status and launches nothing; no call aborts or
 *     throws.  A CUDA launch error returns BL_ERR_CUDA.  Inputs must be
 *     finite; NaN or Inf inputs are outside the contract.
 *   - The results are bit-exact: packed bytes, x~, eta, xsum and y_int
 *     equal the CPU oracle's exactly, and y is the single fp32 rounding of
 *     float(y_int) * s_m with s_m = RN32(RN32(eta_m * gamma) / 127).
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BL_OK = 0,
    BL_ERR_INVALID_ARG = 1, /* null pointer, negative or zero size, unknown dtype */
    BL_ERR_UNSUPPORTED = 2, /* sizes beyond the stated limits, or no B200-class GPU */
    BL_ERR_ALIGNMENT = 3,   /* a pointer breaks the alignment stated for it */
    BL_ERR_CUDA = 4,        /* a CUDA runtime error at launch time */
    BL_ERR_TIMEOUT = 5      /* a kernel gave up a bounded wait (see bitlinear_device_error) */
} bl_status;

typedef enum {
    BL_F32 = 0,
    BL_BF16 = 1
} bl_dtype;

/* Which accumulate kernel bitlinear_forward_path runs. */
typedef enum {
    BL_PATH_AUTO = 0,    /* chosen from M, K and alignment (what bitlinear_forward does) */
    BL_PATH_GEMV = 1,    /* CUDA-core decode kernel, packed weights streamed from HBM */
    BL_PATH_TCGEN05 = 2, /* tensor-core kernel: tcgen05 kind::i8, accumulators in TMEM */
    BL_PATH_GENERIC = 3  /* any K, any alignment; plain add/sub/skip per code */
} bl_path;

/* Human-readable text for a status code (static storage, never NULL). */
const char* bitlinear_status_str(bl_status status);

/* Bytes of the packed ternary matrix: N * ceil(K/4).  0 if N or K < 1. */
size_t bitlinear_packed_bytes(int64_t N, int64_t K);

/* Bytes of scratch bitlinear_pack_weights needs (2064: 256 exponent buckets
 * of 64-bit integers, an fp64 sum and a flag).  The caller allocates it,
 * 8-byte aligned. */
size_t bitlinear_pack_workspace_bytes(void);

/*
 * Load-time half of the layer: absmean ternarisation and 2-bit packing.
 * [Production] "1. Absmean Weight Quantization" (gamma, Round then Clip) and
 * WeightQuantizerSTE (clamp at 1e-5); codes from [Production] "Production
 * Deployment Standards" guideline 1 and [No-Multiply] "Kernel
 * Implementation: The Lookup Table Approach".
 *
 *   W         in   fp32, N x K row-major (leading dimension K).
 *   N, K      in   out_features >= 1, in_features >= 1, N*K <= 2^40.
 *   packed    out  uint8, N x P with P = ceil(K/4) (bitlinear_packed_bytes):
 *                  byte n*P + k/4 holds code (W~[n,k] + 1) in bits
 *                  2*(k%4)..2*(k%4)+1, i.e. 00 = -1, 01 = 0, 10 = +1.
 *                  Codes past K in the last byte of a row are 01.
 *   gamma     out  one fp32 on the device: max(RN32(RN64(S) / (N*K)),
 *                  1e-5) with S the exact sum of |W| (order-independent,
 *                  so every GPU and the CPU oracle agree to the bit).  It
 *                  is taken from an fp64 sum of |W| when an error bound
 *                  proves that sum gives this value, else from exact
 *                  integer sums per exponent; the result is the same.
 *   workspace in   bitlinear_pack_workspace_bytes() bytes of device scratch;
 *                  overwritten; must not be shared by calls that may
 *                  overlap on the GPU.
 * Errors: BL_ERR_INVALID_ARG for null pointers or N, K < 1;
 * BL_ERR_UNSUPPORTED for N*K > 2^40; BL_ERR_ALIGNMENT if workspace is not
 * 8-byte or W not 4-byte aligned.
 */
bl_status bitlinear_pack_weights(const float* W, int64_t N, int64_t K,
                                 uint8_t* packed, float* gamma,
                                 void* workspace, void* stream);

/*
 * The three steps of bitlinear_pack_weights as separate calls, for a weight
 * matrix split by rows over several GPUs (each holding rows [n0, n1)).
 * gamma is a mean over the WHOLE matrix ([Production] "1. Absmean Weight
 * Quantization"), so every shard must ternarise with the same gamma: each
 * GPU forms the exact bucket sums of its own rows, the buckets are summed
 * over the GPUs as 64-bit integers (an all-reduce; integer addition makes the
 * result independent of the order and the number of shards), and every GPU
 * derives the identical gamma from the totals.  pack_weights(W) equals
 * absmean_buckets(W) -> gamma_from_buckets(count = N*K) -> ternarise_pack,
 * and on any row split the shards' packed bytes and gamma are bit-identical
 * to those of the whole matrix.
 *
 * Bucket layout: 256 uint64 (2048 bytes, 8-byte aligned).  Bucket b
 * (1..254) holds the sum of the integer significands m (< 2^24) of every
 * |W| = m * 2^(b-150), b the biased fp32 exponent
 * (subnormals in bucket 1).  Buckets 0 and 255 hold no finite values
 * (NaN/Inf weights are outside the contract).  Two's-complement int64
 * addition of the buckets (what an int64 sum all-reduce does) gives the
 * same totals as unsigned addition.
 */

/* Step 1: zero `buckets`, then add the shard's |W| (fp32, N x K row-major,
 * N*K <= 2^40).  Errors as bitlinear_pack_weights (buckets in place of
 * workspace). */
bl_status bitlinear_absmean_buckets(const float* W, int64_t N, int64_t K, void* buckets,
                                    void* stream);

/* Step 2: gamma = max(RN32(RN64(S) / count), 1e-5), S the exact total the
 * buckets hold and count >= 1 the number of elements of the whole matrix
 * (<= 2^40).  One fp32 written on the device.  Errors: BL_ERR_INVALID_ARG for
 * null pointers or count < 1; BL_ERR_UNSUPPORTED for count > 2^40;
 * BL_ERR_ALIGNMENT if buckets is not 8-byte or gamma not 4-byte aligned. */
bl_status bitlinear_gamma_from_buckets(const void* buckets, int64_t count, float* gamma,
                                       void* stream);

/* Step 3: ternarise rows of W (N x K) with the given device gamma and pack
 * them as bitlinear_pack_weights does (N x ceil(K/4) bytes).  Errors:
 * BL_ERR_INVALID_ARG for null pointers or N, K < 1; BL_ERR_UNSUPPORTED for
 * N*K > 2^40; BL_ERR_ALIGNMENT if W or gamma is not 4-byte aligned. */
bl_status bitlinear_ternarise_pack(const float* W, int64_t N, int64_t K, const float* gamma,
                                   uint8_t* packed, void* stream);

/*
 * bitlinear_pack_weights for callers that cannot allocate device memory:
 * for example a library running inside a host framework that owns every
 * byte of device memory through its own pool, or a latency-critical path
 * that must not call cudaMalloc (which can synchronise the device).  The
 * pages have no counterpart; this is a property of the library, not of the
 * method.
 *
 * Same arguments, results and errors as bitlinear_pack_weights, minus the
 * workspace: the 2064-byte pack scratch (256 x 64-bit buckets, an fp64 sum,
 * a flag) is a file-scope device array of the library, held on every GPU
 * that loads the library until the process exits.  The call allocates nothing (no cudaMalloc, cudaFree
 * or allocating library routine).
 *   - Limit: N*K <= 2^40 (the exact sum's 64-bit buckets); larger sizes return
 *     BL_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture on the device.
 *   - Every call on a device shares the one array and clears it first.  Calls
 *     that may overlap on the GPU (other streams, or other threads' streams,
 *     without ordering between them) race on it and give wrong gamma values;
 *     order them, or use bitlinear_pack_weights with separate workspaces.
 */
bl_status bitlinear_pack_weights_noalloc(const float* W, int64_t N, int64_t K,
                                         uint8_t* packed, float* gamma, void* stream);

/*
 * Per-token absmax int8 quantisation of activations.
 * [Production] "2. Absmax Dynamic Activation Quantization" and
 * ActivationQuantizerSTE: eta per token (last dimension), clamp at 1e-5,
 * Round(x * 127 / eta) evaluated as two fp32 roundings in that order.
 *
 *   x     in   M x K row-major, fp32 (xdt = BL_F32) or bf16 (BL_BF16).
 *   M     in   tokens >= 0 (M = 0 is a no-op returning BL_OK; the M-sized
 *              buffers may then be NULL).
 *   K     in   in_features >= 1.
 *   xq    out  int8, M x K row-major: clip(RNE(RN32(RN32(x*127)/eta_m)), -127, 127).
 *   eta   out  fp32, M: max(max_k |x[m,k]|, 1e-5).
 *   xsum  out  int32, M: sum_k xq[m,k] (used by the accumulate kernels);
 *              may not be NULL.
 * Errors: BL_ERR_INVALID_ARG for null pointers, M < 0, K < 1 or an unknown
 * dtype; BL_ERR_ALIGNMENT if x is not aligned to its element size.
 */
bl_status bitlinear_quant_act(const void* x, bl_dtype xdt, int64_t M, int64_t K,
                              int8_t* xq, float* eta, int32_t* xsum, void* stream);

/*
 * RMSNorm without affine parameters, fused with the per-token quantiser.
 * [Production] "2. Absmax Dynamic Activation Quantization" (the activations
 * are RMS-normalised before absmax quantisation) and BitLinear158.forward
 * (norm = rsqrt(mean(x^2) + 1e-6), x_norm = x * norm), per token:
 *   mean  = RN32(RN64(exact sum_k x^2) / K)   (the division in fp64)
 *   r     = RN32(1 / RN32(sqrt(RN32(mean + 1e-6))))
 *   x_norm = RN32(x * r), then bitlinear_quant_act's rule on x_norm.
 * The sum of squares is formed exactly, so the result does not depend on
 * the summation order and is identical on every device.
 *
 *   x     in   M x K row-major, bf16 (xdt = BL_BF16).
 *   M     in   tokens >= 0 (M = 0 is a no-op returning BL_OK; the M-sized
 *              buffers may then be NULL).
 *   K     in   in_features, 1 <= K <= 2^24.
 *   xq    out  int8, M x K row-major: the codes of x_norm.
 *   eta   out  fp32, M: max(max_k |x_norm[m,k]|, 1e-5).
 *   xsum  out  int32, M: sum_k xq[m,k].
 * Errors: BL_ERR_INVALID_ARG for null pointers, M < 0, K < 1 or an unknown
 * dtype; BL_ERR_UNSUPPORTED for fp32 x or K > 2^24; BL_ERR_ALIGNMENT if x is
 * not 2-byte aligned or eta/xsum not 4-byte aligned.
 */
bl_status bitlinear_rmsnorm_quant_act(const void* x, bl_dtype xdt, int64_t M, int64_t K,
                                      int8_t* xq, float* eta, int32_t* xsum, void* stream);

/*
 * Per-token half of the layer: integer accumulation and rescale.
 * [Production] "The MatMul-Free Breakthrough" (add where W~ = +1, subtract
 * where W~ = -1, skip zeros), [Additive] "3. Additive Integer Accumulation",
 * and [Production] pipeline step 5 / BitLinear158.forward (rescale by
 * (eta * gamma) / 127).
 *
 *   xq, eta, xsum  in   as written by bitlinear_quant_act (M x K, M, M).
 *   M, K           in   M >= 0 (0 = no-op; xq, eta, xsum, y may then be
 *                       NULL), K >= 1, 127*K < 2^31.
 *   packed, gamma  in   as written by bitlinear_pack_weights for N x K.
 *   N              in   out_features >= 1.
 *   y              out  M x N row-major, fp32 (ydt = BL_F32) or bf16
 *                       (BL_BF16, round to nearest even of the fp32 y).
 *   y_int          out  optional int32 M x N row-major (NULL = not written).
 * The fast kernels need K % 64 == 0 and 16-byte aligned xq, packed, y and
 * y_int; other inputs run a generic kernel with the same results.
 * Errors: BL_ERR_INVALID_ARG for null pointers (other than y_int), N or
 * K < 1, M < 0 or an unknown dtype; BL_ERR_UNSUPPORTED if 127*K >= 2^31.
 */
bl_status bitlinear_forward(const int8_t* xq, const float* eta, const int32_t* xsum,
                            int64_t M, int64_t K,
                            const uint8_t* packed, const float* gamma, int64_t N,
                            void* y, bl_dtype ydt, int32_t* y_int, void* stream);

/*
 * Flag for bitlinear_forward_path and bitlinear_linear: the caller promises
 * that `packed` and `gamma` are not written by any work still pending on
 * `stream` (true for weights packed earlier and synchronised, the normal
 * inference case).  The decode and tensor-core kernels may then start
 * streaming the packed weights (and read gamma) before the preceding kernel
 * on the stream has finished (programmatic dependent launch); activations
 * are always read only after it has finished.
 */
#define BL_FLAG_WEIGHTS_STATIC 1u

/*
 * bitlinear_forward with the accumulate kernel and flags chosen by the
 * caller.  BL_PATH_GEMV and BL_PATH_TCGEN05 return BL_ERR_UNSUPPORTED when
 * the inputs do not meet their layout needs (K % 64 == 0, 16-byte
 * alignment; for BL_PATH_GEMV also either M <= 4 and K * M' <= 131072,
 * M' = M rounded up to 1, 2 or 4, or 2 <= M <= 16 with a shape the
 * register-resident (2..8) or warp-MMA (9..16) kernel takes, see
 * bitlinear_decode_regm_shape and bitlinear_decode_mma_shape
 *); the results of every path are identical.
 * flags: 0 or BL_FLAG_WEIGHTS_STATIC.
 */
bl_status bitlinear_forward_path(const int8_t* xq, const float* eta, const int32_t* xsum,
                                 int64_t M, int64_t K,
                                 const uint8_t* packed, const float* gamma, int64_t N,
                                 void* y, bl_dtype ydt, int32_t* y_int,
                                 bl_path path, unsigned flags, void* stream);

/*
 * The whole per-token layer in one call: quantise x per token
 * ([Production] "2. Absmax Dynamic Activation Quantization"), accumulate
 * with add / subtract / skip ([Production] "The MatMul-Free Breakthrough")
 * and rescale ([Production] pipeline step 5).  Same results, bit for bit, as
 * bitlinear_quant_act followed by bitlinear_forward.  x is quantised as
 * given; for the pages' BitLinear158 layer, which RMS-normalises first, call
 * bitlinear_rmsnorm_quant_act and then bitlinear_forward.
 *
 *   x, xdt, M, K      in   activations as for bitlinear_quant_act.
 *   packed, gamma, N  in   as for bitlinear_forward.
 *   y, ydt, y_int     out  as for bitlinear_forward (y_int optional).
 *   xq, eta, xsum     out  the quantised activations (M x K int8, M fp32,
 *                          M int32).  For bf16 decode batches one fused
 *                          kernel runs and these are optional (NULL = not
 *                          written): one token whose layer fits the
 *                          register-resident kernel (see
 *                          bitlinear_decode_reg_shape), two tokens whose
 *                          layer fits the multi-token one (see
 *                          bitlinear_decode_regm_shape; 16-byte aligned x,
 *                          packed, y, y_int and xq), and otherwise one or
 *                          two tokens with K % 64 == 0, K * M' <= 131072
 *                          (M' = M rounded up to 1 or 2) and 16-byte
 *                          aligned x, packed, y.  Otherwise two kernels run
 *                          (quantiser, then the accumulate kernel
 *                          bitlinear_forward would pick) and they are
 *                          required scratch (BL_ERR_INVALID_ARG if NULL).
 *   flags             in   0 or BL_FLAG_WEIGHTS_STATIC.
 */
bl_status bitlinear_linear(const void* x, bl_dtype xdt, int64_t M, int64_t K,
                           const uint8_t* packed, const float* gamma, int64_t N,
                           void* y, bl_dtype ydt,
                           int8_t* xq, float* eta, int32_t* xsum,
                           int32_t* y_int, unsigned flags, void* stream);

/*
 * Launch shape of the decode kernel (BL_PATH_GEMV and the fused decode of
 * bitlinear_linear) for M tokens, K inputs and N outputs on the current
 * device; fused = 1 for bitlinear_linear's fused kernel (bf16 activations),
 * 0 for bitlinear_forward's.  The pages have no counterpart: this describes
 * how the library spreads the add / subtract / skip accumulation over a
 * GPU.  shape (host, 10 int32) receives: team_warps G (warps splitting one
 * row block's K), rows_per_block RB, teams, words per lane, rows per CTA,
 * CTAs, row blocks per ring stage, ring stages, activations staged in
 * shared memory (0/1), shared memory bytes per CTA.
 * Errors: BL_ERR_INVALID_ARG for shape == NULL or N < 1; BL_ERR_UNSUPPORTED
 * when the decode kernel does not take (M, K) or the forced shape (below)
 * does not fit; BL_ERR_CUDA / BL_ERR_UNSUPPORTED without a B200-class GPU.
 */
bl_status bitlinear_decode_shape(int64_t M, int64_t K, int64_t N, int fused, int32_t* shape);

/*
 * The same for a GPU with `sms` SMs, without querying a device (host logic
 * only; usable without a GPU).  Errors as above, plus BL_ERR_INVALID_ARG for
 * sms < 1.
 */
bl_status bitlinear_decode_shape_for(int64_t M, int64_t K, int64_t N, int fused, int sms,
                                     int32_t* shape);

/*
 * Shape of the one-token fused kernel of bitlinear_linear that holds each
 * CTA's weights in registers, for K inputs and N outputs on a GPU with `sms`
 * SMs (host logic only; usable without a GPU).  The pages have no
 * counterpart: this describes how the library lays the add / subtract /
 * skip accumulation of one token out on the GPU.  bitlinear_linear uses this
 * kernel for M = 1 (bf16 x, K % 64 == 0, the fused conditions above) when
 * this query succeeds and no decode shape is forced
 * (bitlinear_set_decode_shape); otherwise the shared-memory decode kernel.
 * shape (host, 4 int32) receives: rows per warp RB (1, 2 or 4; 16 warps per
 * CTA), 32-bit weight words per lane and row NJ (K <= 512 NJ), rows per CTA,
 * CTAs.  Errors: BL_ERR_INVALID_ARG for shape == NULL, K < 1, N < 1 or
 * sms < 1; BL_ERR_UNSUPPORTED when the kernel does not take (K, N): K not a
 * multiple of 64, more than 64 rows per CTA, or more weight words than its
 * register budget.
 */
bl_status bitlinear_decode_reg_shape(int64_t K, int64_t N, int sms, int32_t* shape);

/*
 * Shape of the register-resident kernel for 2 to 8 tokens (BL_PATH_GEMV of
 * bitlinear_forward with x~ given; bitlinear_linear runs it after the
 * quantiser kernel from three tokens on, and with the quantiser fused for
 * two bf16 tokens: every CTA quantises both rows), for M tokens, K inputs
 * and N outputs
 * on a GPU with `sms` SMs (host logic only; usable without a GPU).  The
 * pages have no counterpart.  The library uses this kernel for 2 <= M <= 8
 * on the decode path when this query succeeds and no decode shape is forced
 * (bitlinear_set_decode_shape); otherwise the shared-memory decode kernel
 * (M <= 4) or the tensor-core kernel (BL_PATH_AUTO, M > 4).
 * shape (host, 5 int32) receives: token slots MT (2, 4 or 8), rows per warp RB
 * (16 warps per CTA), 32-bit weight words per lane and row NJ (K <= 512 NJ),
 * rows per CTA, CTAs.  Errors: BL_ERR_INVALID_ARG for shape == NULL, K < 1,
 * N < 1 or sms < 1; BL_ERR_UNSUPPORTED when the kernel does not take
 * (M, K, N): M outside 2..8, K not a multiple of 64, more than 64 rows per
 * CTA, RB * MT above 32, or more weight words than its register budget.
 */
bl_status bitlinear_decode_regm_shape(int64_t M, int64_t K, int64_t N, int sms, int32_t* shape);

/*
 * Shape of the warp-MMA decode kernel for 9 to 16 tokens whose x~ is given
 * (mma.sync m16n8k32 s8 with each CTA's weights in registers), for M
 * tokens, K inputs and N outputs on a GPU with `sms` SMs (host logic only).
 * The pages have no counterpart.  The library uses this kernel for
 * 9 <= M <= 16 on the decode path (BL_PATH_GEMV, which BL_PATH_AUTO picks
 * for these M when a decode kernel takes the shape) when this query
 * succeeds, the kernel is on (bitlinear_set_decode_mma), the register-
 * resident kernels are on and no decode shape is forced; otherwise the
 * 2..8-token register kernel, the shared-memory decode kernel (M <= 4) or
 * the tensor-core kernel.  shape (host, 7 int32) receives: token slots (16),
 * row blocks of 16 per CTA RBK, K parts per block (16 / RBK),
 * steps of 64 K per warp, rows per CTA, CTAs, dynamic shared memory bytes.
 * Errors: BL_ERR_INVALID_ARG for shape == NULL, K < 1, N < 1 or sms < 1;
 * BL_ERR_UNSUPPORTED when the kernel does not take (M, K, N): M outside
 * 9..16, K not a multiple of 64, more than 64 rows per CTA, more K steps
 * per warp than the register budget (24), or activation slots beyond the
 * shared memory of one CTA.
 */
bl_status bitlinear_decode_mma_shape(int64_t M, int64_t K, int64_t N, int sms, int32_t* shape);

/*
 * Turn the warp-MMA decode kernel on (1, the default) or off (0) for every
 * later launch in this process (off: the 2..8-token register kernel, the
 * shared-memory decode kernel or the tensor-core kernel take those calls).
 * Results are identical either way; this exists to compare the kernels.
 * No counterpart on the pages.  Not synchronised with launches in flight
 * on other host threads.
 * Errors: BL_ERR_INVALID_ARG for values other than 0 and 1.
 */
bl_status bitlinear_set_decode_mma(int enable);

/*
 * Turn the register-resident kernels on (1, the default) or off (0) for
 * every later launch in this process: the one-token kernel of
 * bitlinear_linear (quantiser fused), the 2..8-token kernel and the
 * warp-MMA kernel of the decode path (x~ given).  Off, those calls run the
 * shared-memory decode kernel (or, above 4 tokens, the tensor-core kernel).  Results are identical either way; this exists to compare the
 * kernels.  No counterpart on the pages.
 * Not synchronised with launches in flight on other host threads.
 * Errors: BL_ERR_INVALID_ARG for values other than 0 and 1.
 */
bl_status bitlinear_set_decode_reg(int enable);

/*
 * Force the decode kernel's shape for every later launch in this process:
 * team_warps G in 1..16 and rows_per_block RB in {1, 2, 4, 8, 16} (RB * M'
 * <= 16 with M' = M rounded up to 1, 2 or 4); 0 for either leaves that
 * choice to the library (the default).  A forced shape that a launch cannot
 * use makes that launch return BL_ERR_UNSUPPORTED.  While a shape is forced,
 * bitlinear_linear runs the shared-memory decode kernel for one token too.  Results are identical
 * for every shape; this exists to test and tune the shapes.  Not
 * synchronised with launches in flight on other host threads.
 * Errors: BL_ERR_INVALID_ARG for values outside those ranges.
 */
bl_status bitlinear_set_decode_shape(int team_warps, int rows_per_block);

/*
 * Force the K split of the tensor-core kernel (BL_PATH_TCGEN05) for every
 * later launch in this process: k_split in 1..8 CTAs per cluster, each
 * accumulating its share of the K tiles of 128, the partial int32 tiles
 * added in distributed shared memory; 0 leaves the choice to the library
 * (the default: split only when the output tiles cannot fill the GPU).  The
 * split is capped by the K tiles and by the partial tiles the first CTA can
 * hold.  The pages have no counterpart; results are identical for every
 * split (integer sums).  Not synchronised with launches in flight on other
 * host threads.
 * Errors: BL_ERR_INVALID_ARG for k_split outside 0..8.
 */
bl_status bitlinear_set_tc_split(int k_split);

/*
 * bitlinear_linear for up to 4 matrices that share one activation input
 * (a decoder layer's Wq|Wk|Wv, or gate|up) in ONE launch of the fused decode
 * kernel: every CTA quantises x itself and works on rows of one matrix,
 * each with its own gamma and output.  The page "BitNet b1.58 & 1-Bit LLM
 * Architectures: Eliminating Matrix Multiplication and Running 70B Models on
 * CPU in 2026", section 2, names the seven BitLinear projections of a
 * Transformer block (Wq, Wk, Wv, Wo and Wgate, Wup, Wdown), of which Wq|Wk|Wv
 * and Wgate|Wup read the same input; it gives no fused form.  The results are
 * those of bitlinear_linear on each matrix, bit for bit.
 *
 *   x         in   bf16 M x K row-major, 16-byte aligned (xdt must be
 *                  BL_BF16; BL_ERR_UNSUPPORTED otherwise).
 *   M, K      in   1 <= M <= 4, K % 64 == 0, K * M' <= 131072 (the fused
 *                  decode kernel's range; BL_ERR_UNSUPPORTED otherwise).
 *                  M = 0 is a no-op.
 *   nseg      in   1..4 matrices.
 *   packed[s], gamma[s], N[s]   in   host arrays of nseg device pointers /
 *                  row counts: matrix s as bitlinear_pack_weights wrote it
 *                  (N[s] x ceil(K/4), 16-byte aligned) and its gamma.
 *   y[s]      out  host array of nseg device pointers: M x N[s] row-major,
 *                  fp32 or bf16 (ydt), 16-byte aligned.
 *   flags     in   0 or BL_FLAG_WEIGHTS_STATIC (for every matrix).
 * x~, eta, xsum and y_int are not returned (use bitlinear_linear).
 * Errors: BL_ERR_INVALID_ARG for nseg outside 1..4, null pointers or
 * arrays, N[s] < 1, unknown dtypes; BL_ERR_UNSUPPORTED as above;
 * BL_ERR_ALIGNMENT for misaligned pointers.
 */
bl_status bitlinear_linear_group(const void* x, bl_dtype xdt, int64_t M, int64_t K, int nseg,
                                 const uint8_t* const* packed, const float* const* gamma,
                                 const int64_t* N, void* const* y, bl_dtype ydt, unsigned flags,
                                 void* stream);

/*
 * Base-3 "compact ternary packing" (five trits per byte, 1.6 bits per
 * weight): the measured alternative to the 2-bit codes.  The page "1-Bit
 * Large Language Models and BitNet b1.58: How Ternary Weights and Additive
 * Kernels Eliminate Matrix Multiplications", section "Energy, Memory
 * Bandwidth, and Serving Economics", names the packing but gives no layout;
 * this library's layout: byte g of row n holds the trits of columns
 * 5g .. 5g+4 as sum_j (t + 1) * 3^j (least significant first), trits past K
 * are 0, and a row is bitlinear_packed3_stride(K) = 16 * ceil(ceil(K/5)/16)
 * bytes (padding bytes hold five zero trits, value 121).
 */

/* Row stride of the base-3 layout in bytes (0 if K < 1). */
int64_t bitlinear_packed3_stride(int64_t K);

/*
 * bitlinear_pack_weights into the base-3 layout: the same gamma and the same
 * trits, packed3 = N x bitlinear_packed3_stride(K) uint8.  Same arguments,
 * workspace and errors as bitlinear_pack_weights.
 */
bl_status bitlinear_pack_weights3(const float* W, int64_t N, int64_t K, uint8_t* packed3,
                                  float* gamma, void* workspace, void* stream);

/*
 * bitlinear_forward on base-3 packed weights (x~ given): the same y and
 * y_int, bit for bit, as bitlinear_forward on the 2-bit packing of the same
 * trits.  One CUDA-core kernel per 4 tokens or fewer (meant for decode
 * batches; fewer per launch for long rows).
 *   packed3   in   N x bitlinear_packed3_stride(K) uint8, 16-byte aligned.
 *   other arguments as bitlinear_forward (y_int optional).
 * Errors: BL_ERR_INVALID_ARG for null pointers, M < 0, K or N < 1 or an
 * unknown ydt; BL_ERR_UNSUPPORTED when K is too large for the activation
 * slots in shared memory (K above 29360) or N > 2^30;
 * BL_ERR_ALIGNMENT for misaligned pointers.  M = 0 is a no-op.
 */
bl_status bitlinear_forward3(const int8_t* xq, const float* eta, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* packed3, const float* gamma, int64_t N,
                             void* y, bl_dtype ydt, int32_t* y_int, void* stream);

/* The path bitlinear_forward would pick for these sizes and pointers on the
 * current device (without a usable device, as if the register-resident
 * kernel for 5..8 tokens were unavailable). */
bl_path bitlinear_select_path(int64_t M, int64_t K, int64_t N,
                              const void* xq, const void* packed, const void* y,
                              const void* y_int);

/*
 * Reads and clears the library's device-side error word for the current
 * device (synchronises `stream`).  The tensor-core kernel gives every wait
 * on a barrier a time limit; a wait that runs out records BL_ERR_TIMEOUT
 * there and the kernel returns early instead of hanging.  *code receives
 * BL_OK or BL_ERR_TIMEOUT.  Returns BL_ERR_CUDA if the copy fails.
 */
bl_status bitlinear_device_error(int32_t* code, void* stream);

/* Library version as "major.minor.patch" (static storage). */
const char* bitlinear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */

/*
 * bitlinear_oracle.c -- plain, slow, scalar CPU oracle for the BitNet b1.58
 * BitLinear forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header, table or helper with the CUDA sources.
 *
 * What it computes, and where the pages define it.  Pages are cited by title
 * and section, with these short tags:
 *   [Production]  "BitNet b1.58 & 1-Bit LLMs in Production: Ternary
 *                 Quantization, MatMul-Free Kernels, and Edge AI Silicon
 *                 Deployment"
 *   [Additive]    "1-Bit Large Language Models and BitNet b1.58: How Ternary
 *                 Weights and Additive Kernels Eliminate Matrix
 *                 Multiplications"
 *   [No-Multiply] "BitNet b1.58: Ternary Weight LLMs That Eliminate Matrix
 *                 Multiplication"
 *
 *  - [Production] "1. Absmean Weight Quantization": gamma = mean |W| over
 *    the whole n x m matrix; W~ = Clip(Round(W / gamma), -1, +1).  Its
 *    PyTorch WeightQuantizerSTE clamps gamma at a minimum of 1e-5 and uses
 *    torch.round (round half to even).
 *  - [Production] "2. Absmax Dynamic Activation Quantization" and its
 *    ActivationQuantizerSTE: eta = per-token max |x| (clamped at 1e-5),
 *    x~ = Round(x * 127 / eta), evaluated as (x*127)/eta in fp32.  The clip
 *    range taken is [-127, 127] (the pages disagree; the clip never binds).
 *  - [Production] "The MatMul-Free Breakthrough": y_int is the sum of x~
 *    where W~ = +1 minus the sum of x~ where W~ = -1; zeros are skipped.
 *  - [Production] "Production Deployment Standards" guideline 1, and
 *    [No-Multiply] "Kernel Implementation: The Lookup Table Approach":
 *    2-bit codes 00 = -1, 01 = 0, 10 = +1, four per byte, element j of a
 *    byte in bits 2j..2j+1.
 *  - [Production] pipeline figure step 5 and BitLinear158.forward:
 *    y = y_int * ((eta * gamma) / 127).
 *
 * Precision: the pages compute in fp32 (PyTorch float tensors), so every
 * floating-point step below is one IEEE fp32 operation rounded to nearest
 * even, in the order written, except the gamma reduction, which is exact
 * (see oracle_absmean_gamma).  Compile without -ffast-math and with
 * -ffp-contract=off so no step is fused or reordered.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_CODE 2 /* a packed code 11 was found: not a valid trit */
#define ORACLE_ERR_NONFINITE 3

/* ------------------------------------------------------------------------ */
/* Exact sum of |W| (Kulisch-style fixed-point accumulator).                 */
/*                                                                           */
/* Every finite fp32 value is an integer multiple of 2^-149 below 2^128, so */
/* a fixed-point number with its least significant bit at 2^-149 and 384    */
/* bits in all holds any sum of up to 2^100 such values without loss.       */
/* Limbs are 32 bits wide, least significant first; carries are propagated */
/* on every add, so the accumulator is always normalised.                   */
/* ------------------------------------------------------------------------ */
#define ACC_LIMBS 12

typedef struct { uint32_t limb[ACC_LIMBS]; } exact_acc;

static void acc_add_u64_at(exact_acc* a, uint64_t v, int bit) {
    /* add v * 2^bit (bit counted from the 2^-149 position) */
    int li = bit / 32, sh = bit % 32;
    /* v < 2^24 here, so v << sh < 2^56 spans at most two limbs */
    unsigned __int128 w = ((unsigned __int128)v) << sh;
    uint64_t carry = 0;
    for (int i = li; i < ACC_LIMBS; ++i) {
        uint64_t add = (uint64_t)(w & 0xffffffffu);
        w >>= 32;
        uint64_t s = (uint64_t)a->limb[i] + add + carry;
        a->limb[i] = (uint32_t)s;
        carry = s >> 32;
        if (w == 0 && carry == 0) break;
    }
}

static void acc_add_abs_float(exact_acc* a, float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t e = (u >> 23) & 0xffu;
    uint32_t frac = u & 0x7fffffu;
    if (e == 0) {
        /* zero or subnormal: value = frac * 2^-149 */
        if (frac) acc_add_u64_at(a, frac, 0);
    } else {
        /* normal: value = (2^23 + frac) * 2^(e - 150) = m * 2^-149 * 2^(e-1) */
        acc_add_u64_at(a, (uint64_t)(frac | 0x800000u), (int)e - 1);
    }
}

static int acc_get_bit(const exact_acc* a, int bit) {
    return (int)((a->limb[bit / 32] >> (bit % 32)) & 1u);
}

/* Round the exact fixed-point value to the nearest double, ties to even. */
static double acc_to_double_rn(const exact_acc* a) {
    int top = -1;
    for (int i = ACC_LIMBS - 1; i >= 0 && top < 0; --i) {
        if (a->limb[i]) {
            for (int b = 31; b >= 0; --b)
                if ((a->limb[i] >> b) & 1u) { top = i * 32 + b; break; }
        }
    }
    if (top < 0) return 0.0;
    if (top <= 52) {
        /* fits in 53 bits: exact */
        uint64_t m = 0;
        for (int b = top; b >= 0; --b) m = (m << 1) | (uint64_t)acc_get_bit(a, b);
        return ldexp((double)m, -149);
    }
    /* keep bits top .. top-52, guard bit top-53, sticky = anything below */
    uint64_t m = 0;
    for (int b = top; b >= top - 52; --b) m = (m << 1) | (uint64_t)acc_get_bit(a, b);
    int guard = acc_get_bit(a, top - 53);
    int sticky = 0;
    for (int b = top - 54; b >= 0 && !sticky; --b) sticky = acc_get_bit(a, b);
    if (guard && (sticky || (m & 1u))) m += 1; /* may become 2^53: still exact */
    return ldexp((double)m, (top - 52) - 149);
}

/*
 * gamma = max(RN32(RN64(S) / (n*m)), 1e-5f), S = exact sum of |W|.
 *
 * [Production] "1. Absmean Weight Quantization" (gamma formula) and its
 * WeightQuantizerSTE.forward (mean of |W| over the whole matrix,
 * clamp at min 1e-5).  The pages do not fix a summation order; the reading
 * taken is the exact sum, rounded once to fp64, divided by the element count
 * in fp64 and rounded once to fp32, which is reproducible on any device.
 */
int oracle_absmean_gamma(const float* W, int64_t count, float* gamma_out, double* sum_out) {
    if (!W || count <= 0 || !gamma_out) return ORACLE_ERR_ARG;
    exact_acc acc;
    memset(&acc, 0, sizeof(acc));
    for (int64_t i = 0; i < count; ++i) {
        if (!isfinite(W[i])) return ORACLE_ERR_NONFINITE;
        acc_add_abs_float(&acc, W[i]);
    }
    double s = acc_to_double_rn(&acc);
    double g = s / (double)count;
    float gf = (float)g;
    if (gf < 1e-5f) gf = 1e-5f;
    *gamma_out = gf;
    if (sum_out) *sum_out = s;
    return ORACLE_OK;
}

/* Round half to even, written from its definition (not via the FP env):
 * on a = |q| the fractional part a - floor(a) is exact, ties go to the even
 * neighbour, and the sign is put back afterwards. */
static float round_half_even(float q) {
    float a = fabsf(q);
    float f = floorf(a);
    float d = a - f;
    float r;
    if (d > 0.5f) r = f + 1.0f;
    else if (d < 0.5f) r = f;
    else r = (fmodf(f, 2.0f) == 0.0f) ? f : f + 1.0f;
    return q < 0.0f ? -r : r;
}

static float clip(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/*
 * W~[n,k] = Clip(Round(RN32(W[n,k] / gamma)), -1, 1), packed as 2-bit codes
 * code = W~ + 1 into byte n*P + k/4 at bits 2*(k%4), P = ceil(K/4).
 * Bits of a trailing partial byte are code 01 (zero).
 *
 * Ternarisation: [Production] "1. Absmean Weight Quantization" (Round then
 * Clip).  Packing: [Production] "Production Deployment Standards" guideline
 * 1; [No-Multiply] "Kernel Implementation: The Lookup Table Approach" (its
 * ternary_dot_packed reads byte i>>2 and element j from bits 2j).
 */
int oracle_ternarise_pack(const float* W, int64_t N, int64_t K, float gamma,
                          uint8_t* packed, int8_t* ternary_out /* optional N*K */) {
    if (!W || N <= 0 || K <= 0 || !packed) return ORACLE_ERR_ARG;
    int64_t P = (K + 3) / 4;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < P; ++b) {
            uint8_t byte = 0;
            for (int j = 0; j < 4; ++j) {
                int64_t k = 4 * b + j;
                int code = 1; /* zero trit for the tail */
                if (k < K) {
                    float q = W[n * K + k] / gamma;
                    float t = clip(round_half_even(q), -1.0f, 1.0f);
                    code = (int)t + 1;
                    if (ternary_out) ternary_out[n * K + k] = (int8_t)t;
                }
                byte |= (uint8_t)(code << (2 * j));
            }
            packed[n * P + b] = byte;
        }
    }
    return ORACLE_OK;
}

/*
 * Per-token absmax int8 quantisation of activations x (M x K, fp32 values;
 * bf16 inputs are widened to fp32 exactly by the caller):
 *   eta_m = max(max_k |x[m,k]|, 1e-5f)
 *   x~[m,k] = Clip(Round(RN32(RN32(x*127) / eta_m)), -127, 127)
 *   xsum_m  = sum_k x~[m,k]
 * [Production] "2. Absmax Dynamic Activation Quantization" and its
 * ActivationQuantizerSTE (per-token max over the last dimension,
 * clamp at 1e-5, x * 127.0 / eta).  xsum is a by-product used by the
 * accumulation checks; it is the plain integer sum of the row.
 */
int oracle_quant_act(const float* x, int64_t M, int64_t K,
                     int8_t* xq, float* eta, int32_t* xsum, int nthreads) {
    if (!x || M < 0 || K <= 0 || !xq || !eta) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static) if (nthreads != 1)
#endif
    for (int64_t m = 0; m < M; ++m) {
        const float* row = x + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (!isfinite(row[k])) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                err = ORACLE_ERR_NONFINITE;
            }
            float a = fabsf(row[k]);
            if (a > amax) amax = a;
        }
        float e = amax < 1e-5f ? 1e-5f : amax;
        eta[m] = e;
        int64_t s = 0;
        for (int64_t k = 0; k < K; ++k) {
            float scaled = row[k] * 127.0f;
            float q = scaled / e;
            float r = clip(round_half_even(q), -127.0f, 127.0f);
            xq[m * K + k] = (int8_t)r;
            s += (int64_t)r;
        }
        if (xsum) xsum[m] = (int32_t)s;
    }
    return err;
}

/*
 * y_int[m,n] = sum_{k: code==2} x~[m,k] - sum_{k: code==0} x~[m,k]
 * (code 01 skipped), read from the packed bytes exactly as [No-Multiply]'s
 * ternary_dot_packed decodes them, then the rescale of [Production] step 5:
 *   s_m = RN32(RN32(eta_m * gamma) / 127);  y = RN32(RN32(float(y_int)) * s_m)
 * Accumulation identity: [Production] "The MatMul-Free Breakthrough".
 * Rescale: [Production] pipeline figure step 5 and BitLinear158.forward.
 * Returns ORACLE_ERR_CODE if a code 11 is met (never produced by packing).
 */
int oracle_forward(const int8_t* xq, const float* eta, int64_t M, int64_t K,
                   const uint8_t* packed, float gamma, int64_t N,
                   int32_t* y_int, float* y, int nthreads) {
    if (!xq || !eta || M < 0 || K <= 0 || !packed || N <= 0) return ORACLE_ERR_ARG;
    int64_t P = (K + 3) / 4;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static) if (nthreads != 1)
#endif
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t* wrow = packed + n * P;
        for (int64_t m = 0; m < M; ++m) {
            const int8_t* xrow = xq + m * K;
            int32_t acc = 0;
            for (int64_t k = 0; k < K; ++k) {
                int code = (wrow[k >> 2] >> (2 * (k & 3))) & 3;
                if (code == 2) acc += xrow[k];
                else if (code == 0) acc -= xrow[k];
                else if (code == 3) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                    err = ORACLE_ERR_CODE;
                }
                /* code 1: zero weight, skipped */
            }
            if (y_int) y_int[m * N + n] = acc;
            if (y) {
                float eg = eta[m] * gamma;
                float s = eg / 127.0f;
                y[m * N + n] = (float)acc * s;
            }
        }
    }
    return err;
}

/* Same as oracle_forward, restricted to a list of (m, n) output positions, for
 * spot checks of outputs too large to compute whole. */
int oracle_forward_at(const int8_t* xq, const float* eta, int64_t M, int64_t K,
                      const uint8_t* packed, float gamma, int64_t N,
                      const int64_t* ms, const int64_t* ns, int64_t count,
                      int32_t* y_int, float* y) {
    if (!xq || !eta || K <= 0 || !packed || N <= 0 || count < 0) return ORACLE_ERR_ARG;
    int64_t P = (K + 3) / 4;
    int err = ORACLE_OK;
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        if (m < 0 || m >= M || n < 0 || n >= N) return ORACLE_ERR_ARG;
        const uint8_t* wrow = packed + n * P;
        const int8_t* xrow = xq + m * K;
        int32_t acc = 0;
        for (int64_t k = 0; k < K; ++k) {
            int code = (wrow[k >> 2] >> (2 * (k & 3))) & 3;
            if (code == 2) acc += xrow[k];
            else if (code == 0) acc -= xrow[k];
            else if (code == 3) err = ORACLE_ERR_CODE;
        }
        if (y_int) y_int[i] = acc;
        if (y) {
            float eg = eta[m] * gamma;
            float s = eg / 127.0f;
            y[i] = (float)acc * s;
        }
    }
    return err;
}

/* fp32 -> bf16, round to nearest even, on the bit pattern (finite inputs). */
void oracle_f32_to_bf16(const float* in, uint16_t* out, int64_t count) {
    for (int64_t i = 0; i < count; ++i) {
        uint32_t u;
        memcpy(&u, &in[i], 4);
        uint32_t lower = u & 0xffffu;
        uint32_t upper = u >> 16;
        if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
        out[i] = (uint16_t)upper;
    }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

// Host driver for the division-free rules of the kernels, compiled from the
// kernels' own __host__ __device__ routines (quant.cuh, pack.cuh,
// common.cuh), used by tests/test_fast_rules.py.
//   quant   : code_bits_bf16_r against RNE(RN32(RN32(127 x) / eta)) (IEEE
//             division) for every bf16 x with |x| <= eta, eta = every bf16
//             significand at several exponents, and reciprocals r that are
//             off RN32(1/eta) by -8..+8 ulps (the rule needs r within
//             2^-21 relative; the hardware approximation is within 1 ulp).
//   div127  : div127_rn(a) against the IEEE quotient a / 127 for every
//             normal fp32 a >= 2^-119.
//   vote    : code_bits_bf16_n (the tie test voted over groups of 4 or 8
//             values) against code_bits_bf16_r value by value, on the same
//             values as quant, in two groupings (consecutive values, and
//             values 997 apart), counting the groups that held a tie.
//   widen   : widen_f32_mag on every fp32 magnitude pattern and
//             widen_bf16_mag on every bf16 one: the exact value for normal
//             values, a value in [2^-127, 2^-126) for exponent field 0.
//   thresh  : ternary_code(w, ternary_threshold(gamma)) against
//             Clip(RNE(RN32(w / gamma)), -1, 1) (IEEE division) for 4096
//             values of gamma and every fp32 w within 64 ulps of
//             +-gamma (0.5 + 2^-25), of +-gamma / 2 and of +-1.5 gamma.
// Prints counts; the test requires zero mismatches.
#include <cmath>
#include <cstdio>
#include <cstring>

#include "pack.cuh"
#include "quant.cuh"

static float from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}
static uint32_t to_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

static int run_quant() {
  long long checked = 0, bad = 0, ties = 0;
  const int exps[] = {-12, -3, 0, 5, 20};
  for (int E : exps) {
    for (int m = 128; m < 256; ++m) {
      const float eta = std::ldexp(static_cast<float>(m) / 128.0f, E);  // a bf16 value
      const float heta = eta * 0.5f;
      const float r0 = 1.0f / eta;
      for (int k = -8; k <= 8; ++k) {
        const float r = from_bits(to_bits(r0) + k);
        const float s = bl::f32_mul(127.0f, r);
        for (uint32_t b = 0; b < 0x7F80u; ++b) {
          const float v = from_bits(b << 16);
          if (!(v <= eta)) continue;
          for (int sg = 0; sg < 2; ++sg) {
            const float x = sg ? -v : v;
            volatile float a = x * 127.0f;
            volatile float q = a / eta;
            float rq = std::nearbyint(q);
            rq = std::fmin(127.0f, std::fmax(-127.0f, rq));
            if (k == 0 && std::fabs(q - std::trunc(q)) == 0.5f) ++ties;
            const int got = static_cast<int>(bl::code_bits_bf16_r(x, eta, heta, s, r) - bl::kRneMagicBits);
            bad += (got != static_cast<int>(rq));
            ++checked;
          }
        }
      }
    }
  }
  printf("quant checked=%lld mismatches=%lld ties=%lld\n", checked, bad, ties);
  return 0;
}

static int run_div127() {
  const uint32_t lo = to_bits(std::ldexp(1.0f, -119)), hi = 0x7F7FFFFFu;
  long long bad = 0, checked = 0;
#pragma omp parallel for reduction(+ : bad, checked) schedule(static)
  for (long long u = lo; u <= static_cast<long long>(hi); ++u) {
    const float a = from_bits(static_cast<uint32_t>(u));
    volatile float ref = a / 127.0f;
    bad += (to_bits(bl::div127_rn(a)) != to_bits(ref));
    ++checked;
  }
  // the constant is the correctly rounded reciprocal
  const float c = 1.0f / 127.0f;
  const double e0 = std::fabs(static_cast<double>(c) - 1.0 / 127.0);
  const double e1 = std::fabs(static_cast<double>(from_bits(to_bits(c) + 1)) - 1.0 / 127.0);
  const double e2 = std::fabs(static_cast<double>(from_bits(to_bits(c) - 1)) - 1.0 / 127.0);
  printf("div127 checked=%lld mismatches=%lld inv127_nearest=%d\n", checked, bad, (e0 < e1 && e0 < e2) ? 1 : 0);
  return 0;
}

template <int G>
static void vote_groups(const float* xs, long long n, long long stride, float eta, float heta, float s,
                        float r, long long& checked, long long& bad, long long& tie_groups) {
  for (long long start = 0; start + G <= n; start += G) {
    float f[G];
    uint32_t b[G];
    bool has_tie = false;
    for (int i = 0; i < G; ++i) {
      f[i] = xs[((start + i) * stride) % n];
      volatile float a = f[i] * 127.0f;
      volatile float q = a / eta;
      has_tie |= std::fabs(q - std::trunc(q)) == 0.5f;
    }
    bl::code_bits_bf16_n<G>(f, b, eta, heta, s, r);
    for (int i = 0; i < G; ++i) bad += (b[i] != bl::code_bits_bf16_r(f[i], eta, heta, s, r));
    checked += G;
    tie_groups += has_tie;
  }
}

static int run_vote() {
  long long checked = 0, bad = 0, tie_groups = 0;
  const int exps[] = {-12, 0, 20};
  static float xs[2 * 0x7F80];
  for (int E : exps) {
    for (int m = 128; m < 256; ++m) {
      const float eta = std::ldexp(static_cast<float>(m) / 128.0f, E);
      const float heta = eta * 0.5f;
      for (int k = -1; k <= 1; ++k) {
        const float r = from_bits(to_bits(1.0f / eta) + k);
        const float s = bl::f32_mul(127.0f, r);
        long long n = 0;
        for (uint32_t bb = 0; bb < 0x7F80u; ++bb) {
          const float v = from_bits(bb << 16);
          if (!(v <= eta)) continue;
          xs[n++] = v;
          xs[n++] = -v;
        }
        vote_groups<8>(xs, n, 1, eta, heta, s, r, checked, bad, tie_groups);
        vote_groups<4>(xs, n, 1, eta, heta, s, r, checked, bad, tie_groups);
        vote_groups<8>(xs, n, 997, eta, heta, s, r, checked, bad, tie_groups);
      }
    }
  }
  printf("vote checked=%lld mismatches=%lld tie_groups=%lld\n", checked, bad, tie_groups);
  return 0;
}

static int run_widen() {
  long long bad = 0, checked = 0, zero_field = 0;
#pragma omp parallel for reduction(+ : bad, checked, zero_field) schedule(static)
  for (long long u = 0; u < 0x80000000LL; ++u) {
    const uint32_t a = static_cast<uint32_t>(u);
    const double w = bl::widen_f32_mag(a | 0x80000000u);  // the sign is ignored
    if ((a >> 23) == 0) {
      bad += !(w >= 0x1p-127 && w < 0x1p-126);
      ++zero_field;
    } else if ((a >> 23) != 0xFF) {
      bad += (w != static_cast<double>(from_bits(a)));
    }
    ++checked;
  }
  for (uint32_t h = 0; h < 0x10000u; ++h) {
    const double w = bl::widen_bf16_mag(h);
    const uint32_t e = (h >> 7) & 0xFFu;
    if (e == 0) bad += !(w >= 0x1p-127 && w < 0x1p-126);
    else if (e != 0xFF) bad += (w != static_cast<double>(std::fabs(from_bits(h << 16))));
    ++checked;
  }
  printf("widen checked=%lld mismatches=%lld zero_field=%lld\n", checked, bad, zero_field);
  return 0;
}

static int run_thresh() {
  long long bad = 0, checked = 0, nonzero = 0;
  uint32_t state = 12345u;
  for (int i = 0; i < 4096; ++i) {
    state = state * 1664525u + 1013904223u;
    // gamma: 1e-5 .. about 1e5, every significand pattern reachable
    const float gamma = std::ldexp(1.0f + static_cast<float>(state >> 9) * 0x1p-23f, -17 + static_cast<int>(i % 34));
    const float thr = bl::ternary_threshold(gamma);
    const float centers[3] = {static_cast<float>(static_cast<double>(gamma) * (0.5 + 0x1p-25)), gamma * 0.5f,
                              gamma * 1.5f};
    for (float c : centers) {
      for (int k = -64; k <= 64; ++k) {
        for (int sg = 0; sg < 2; ++sg) {
          const float w0 = from_bits(to_bits(c) + k);
          const float w = sg ? -w0 : w0;
          volatile float q = w / gamma;
          const float t = std::fmin(1.0f, std::fmax(-1.0f, std::nearbyint(q)));
          const int want = static_cast<int>(t) + 1;
          const int got = static_cast<int>(bl::ternary_code(w, thr));
          bad += (got != want);
          nonzero += (want != 1);
          ++checked;
        }
      }
    }
  }
  printf("thresh checked=%lld mismatches=%lld nonzero=%lld\n", checked, bad, nonzero);
  return 0;
}

int main(int argc, char** argv) {
  if (argc > 1 && strcmp(argv[1], "div127") == 0) return run_div127();
  if (argc > 1 && strcmp(argv[1], "vote") == 0) return run_vote();
  if (argc > 1 && strcmp(argv[1], "widen") == 0) return run_widen();
  if (argc > 1 && strcmp(argv[1], "thresh") == 0) return run_thresh();
  return run_quant();
}

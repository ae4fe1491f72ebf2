// Host driver for the exact sum-of-squares rounding of the RMSNorm kernel
// (rmsnorm.cuh's __host__ __device__ routines), used by
// tests/test_rmsnorm_exact_sum.py.  Reads lines
//   hi lo wb n  b1 v1 ... bn vn
// (a 128-bit window value hi:lo in units of 2^(2 wb - 268), plus n bucket
// values v at exponents b < wb) and prints the fp64 bit patterns of
// sumsq_rn64 and, for n = 0, of u128_rn64.
#include <cstdio>
#include <cstring>

#include "rmsnorm.cuh"

int main() {
  unsigned long long hi, lo;
  int wb, n;
  while (scanf("%llu %llu %d %d", &hi, &lo, &wb, &n) == 4) {
    unsigned long long sb[256];
    memset(sb, 0, sizeof sb);
    for (int i = 0; i < n; ++i) {
      int b;
      unsigned long long v;
      if (scanf("%d %llu", &b, &v) != 2 || b < 1 || b >= wb) return 2;
      sb[b] += v;
    }
    const unsigned __int128 win = (static_cast<unsigned __int128>(hi) << 64) | lo;
    const double s = bl::sumsq_rn64(win, wb, sb, 1, wb - 1);
    const double w = bl::u128_rn64(win, 2 * wb - 268);
    unsigned long long us, uw;
    memcpy(&us, &s, 8);
    memcpy(&uw, &w, 8);
    printf("%016llx %016llx\n", us, uw);
  }
  return 0;
}

// Host check of the integer fixed-point terms (csrc/fixed_point.h) against the fp64 route
// rint(ldexp(v * v, e)) / rint(ldexp(|v|, e)) (exact in fp64 for fp32 v, then rounded half to
// even by the host's rint in the default rounding mode), on random fp32 values of every
// exponent (subnormals included), exact .5 ties, and every grid exponent e that keeps the
// largest term below 2^62.  Built and run by tests/test_fixed_point.py.
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <random>

#include "fixed_point.h"

static float from_bits(uint32_t b) {
  float v;
  std::memcpy(&v, &b, 4);
  return v;
}

int main() {
  std::fesetround(FE_TONEAREST);
  std::mt19937_64 rng(12345);
  long long checked = 0, bad = 0;
  auto check = [&](float v, int e, bool sq) {
    const double d = std::fabs((double)v);
    const double t = sq ? std::ldexp(d * d, e) : std::ldexp(d, e);
    if (!(t < 4.611686018427387904e18)) return;  // the grid keeps terms below 2^62
    const long long want = (long long)std::nearbyint(t);
    const long long got = sq ? bitnet::fixed_sq_term(v, e) : bitnet::fixed_abs_term(v, e);
    ++checked;
    if (got != want) {
      if (bad < 10) std::printf("FAIL v=%a e=%d sq=%d got=%lld want=%lld\n", (double)v, e, (int)sq, got, want);
      ++bad;
    }
  };
  for (int it = 0; it < 2000000; ++it) {
    const uint32_t bits = (uint32_t)rng() & 0xFFFFFFFFu;
    const float v = from_bits(bits);
    if (!std::isfinite(v)) continue;
    // e around the value's own grid: 62 - E - L for L in 0..20, plus shifts that round
    int E;
    std::frexp(std::fabs((double)v) * std::fabs((double)v), &E);
    const int e0 = (v == 0.0f) ? 0 : 62 - E - (int)(rng() % 21);
    check(v, e0 - (int)(rng() % 64), true);
    int Ea;
    std::frexp(std::fabs((double)v), &Ea);
    const int ea = (v == 0.0f) ? 0 : 62 - Ea - (int)(rng() % 21);
    check(v, ea - (int)(rng() % 64), false);
  }
  // exact ties: v^2 2^e = k + 1/2 and |v| 2^e = k + 1/2
  for (int k = 0; k < 4096; ++k) {
    const float v = (float)(2 * k + 1);  // |v| 2^-1 = k + 1/2
    check(v, -1, false);
    check(v, -2, false);
    check(v, -1, true);   // v^2 / 2 = (4k^2 + 4k + 1) / 2
    check(v, -2, true);
    check(from_bits(0x00000001u + (uint32_t)k), 160, true);  // subnormals
    check(from_bits(0x00000001u + (uint32_t)k), 170, false);
  }
  if (bad) {
    std::printf("%lld of %lld terms differ\n", bad, checked);
    return 1;
  }
  std::printf("OK %lld terms\n", checked);
  return 0;
}

// The terms of the exact fixed-point sums (sum of x^2 for RMSNorm, sum of |w| for the absmean
// scale) in integer arithmetic.  The sums are taken on the grid 2^-e: each term is v^2 2^e
// or |v| 2^e rounded half to even to an integer.  A finite fp32 v is m 2^(x - 150) with its
// 24-bit significand m (biased exponent x; for subnormals x = 1 and no implicit bit), so
// v^2 2^e = m^2 2^(2x - 300 + e) with m^2 < 2^48 exact in 64 bits, and |v| 2^e =
// m 2^(x - 150 + e): a shift, or a shift whose dropped bits are rounded.  These are the
// values rint(ldexp(v * v, e)) takes in fp64 (v^2 and the scaling are exact there), without
// fp64 multiplies or fp64 -> int64 conversions.  Valid while the result is below 2^62, which
// the choice of e guarantees.  Plain C++ (host and device), so a host test checks it.
#pragma once
#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define FP_HD __host__ __device__ __forceinline__
#else
#define FP_HD inline
#endif

namespace bitnet {

FP_HD uint32_t f32_bits(float v) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(v);
#else
  uint32_t b;
  memcpy(&b, &v, 4);
  return b;
#endif
}

// rint(n * 2^s) (round half to even) for an integer n < 2^48 whose result is below 2^62.
FP_HD long long round_shift(unsigned long long n, int s) {
  if (n == 0ull) return 0;
  if (s >= 0) return (long long)(n << s);
  const int r = -s;
  if (r > 63) return 0;  // n 2^s < 2^-15
  const unsigned long long q = n >> r, rem = n & ((1ull << r) - 1ull), half = 1ull << (r - 1);
  return (long long)(q + ((rem > half || (rem == half && (q & 1ull))) ? 1ull : 0ull));
}

// rint(v^2 2^e)
FP_HD long long fixed_sq_term(float v, int e) {
  const uint32_t b = f32_bits(v) & 0x7FFFFFFFu;
  const int x = (int)(b >> 23);
  const uint32_t m = x ? ((b & 0x7FFFFFu) | 0x800000u) : b;
  return round_shift((unsigned long long)m * m, 2 * (x ? x : 1) - 300 + e);
}

// rint(|v| 2^e)
FP_HD long long fixed_abs_term(float v, int e) {
  const uint32_t b = f32_bits(v) & 0x7FFFFFFFu;
  const int x = (int)(b >> 23);
  const uint32_t m = x ? ((b & 0x7FFFFFu) | 0x800000u) : b;
  return round_shift((unsigned long long)m, (x ? x : 1) - 150 + e);
}

}  // namespace bitnet

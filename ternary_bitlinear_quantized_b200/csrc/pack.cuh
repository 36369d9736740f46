// K-pack: absmean ternarisation and I2_S packing of latent fp32 weights.
//
// "fix: I2_S ARM kernel layout + squared-ReLU FFN - passes the gate on the official
// 2B4T GGUF", description bullet "ggml: llama-quantize I2_S emits the canonical
// layout": one call per tensor (the scale is per tensor and stored after the packed
// data), the interleaved 128-weight / 32-byte layout, 28 zeroed trailer bytes; "Known
// gaps": rows divisible by 128.  Bit order inside a block: element 32 g + i of block b
// lives in byte 32 b + i, bits (7 - 2g):(6 - 2g).
//
// Four launches on the caller's stream (offline path, not latency critical):
//   k_pack_absmax  max|W| by atomicMax on the fp32 bit pattern (exact),
//   k_pack_sum     the order-free fixed-point sum of |W| (int64 atomics),
//   k_pack_codes   beta, s_w and the codes, one 32-bit output word per thread,
//   k_pack_trailer fp32 beta and the 28 zero bytes.
// The trailer doubles as scratch for max|W| (bytes 4..7) and the sum (bytes 8..15)
// until k_pack_trailer overwrites it.
//
// Prescaled mode ("Known gaps": quantize_i2_s keeps the BitNet convention, scale = first
// non-zero |w|, so inputs must already be ternary x scale): k_pack_first_nz finds the
// row-major index of the first non-zero weight (64-bit atomicMin into the scratch's sum
// word, all ones = none), beta = that |w| (1e-5 when there is none), then the same codes
// and trailer kernels.
//
// k_validate_i2s: the checks of an I2_S tensor that llama.cpp's row-data validation
// gains for I2_S in the same pull request: 2-bit fields holding 3 (no ternary weight maps
// to it), non-zero trailer bytes after the scale, a scale that is not finite and positive.
#pragma once
#include "common.cuh"

namespace bitnet {

struct PackScratch {
  uint32_t beta_bits;  // written last
  uint32_t max_bits;
  unsigned long long sum;
};

__global__ void k_pack_clear(PackScratch* sc) {
  sc->beta_bits = 0;
  sc->max_bits = 0;
  sc->sum = 0ull;
}

__global__ void __launch_bounds__(256) k_pack_absmax(const float* __restrict__ W, long long n, PackScratch* sc) {
  __shared__ float red[32];
  float m = 0.0f;
  const long long n4 = n / 4;  // n is a multiple of 128
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  m = block_reduce(m, red, MaxOp());
  if (threadIdx.x == 0) atomicMax(&sc->max_bits, __float_as_uint(m));  // m >= 0: bits order like values
}

__global__ void __launch_bounds__(256) k_pack_sum(const float* __restrict__ W, long long n, PackScratch* sc) {
  __shared__ long long red[32];
  const float M32 = __uint_as_float(sc->max_bits);
  if (M32 == 0.0f) return;
  const double p2e = pow2_f64(fixed_point_exponent((double)M32, n));
  long long part = 0;
  const long long n4 = n / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    part += fixed_abs_term(v.x, p2e) + fixed_abs_term(v.y, p2e) + fixed_abs_term(v.z, p2e) + fixed_abs_term(v.w, p2e);
  }
  part = block_reduce(part, red, AddOpLL());
  if (threadIdx.x == 0) atomicAdd(&sc->sum, (unsigned long long)part);
}

constexpr unsigned long long PACK_NO_NONZERO = ~0ull;

__global__ void k_pack_first_nz_clear(PackScratch* sc) {
  sc->beta_bits = 0;
  sc->max_bits = 0;
  sc->sum = PACK_NO_NONZERO;
}

__global__ void __launch_bounds__(256) k_pack_first_nz(const float* __restrict__ W, long long n, PackScratch* sc) {
  __shared__ unsigned long long red[32];
  unsigned long long best = PACK_NO_NONZERO;
  const long long n4 = n / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    const unsigned long long b = 4ull * (unsigned long long)i;
    const unsigned long long c = v.x != 0.0f ? b : (v.y != 0.0f ? b + 1 : (v.z != 0.0f ? b + 2 : (v.w != 0.0f ? b + 3 : best)));
    if (c < best) best = c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, best, o);
    best = w < best ? w : best;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) best = red[i] < best ? red[i] : best;
    atomicMin(&sc->sum, best);
  }
}

// beta = max(mean|W|, 1e-5) from the scratch; in the prescaled mode |W[first non-zero]|.
BN_DEV float pack_beta(const PackScratch* sc, long long n, const float* W = nullptr, int prescaled = 0) {
  if (prescaled) return sc->sum == PACK_NO_NONZERO ? 1e-5f : fabsf(__ldg(W + sc->sum));
  const float M32 = __uint_as_float(sc->max_bits);
  float mean = 0.0f;
  if (M32 != 0.0f) mean = fixed_point_mean((long long)sc->sum, fixed_point_exponent((double)M32, n), n);
  return fmaxf(mean, 1e-5f);
}

BN_DEV uint32_t ternary_code(float w, float s_w) {
  int c = __float2int_rn(__fmul_rn(w, s_w));
  c = min(1, max(-1, c));
  return (uint32_t)(c + 1);
}

// One thread per output word: word m (0..7) of block b holds bytes 4m..4m+3, whose
// field g carries elements 128 b + 32 g + 4 m + j, j = 0..3.
__global__ void __launch_bounds__(256) k_pack_codes(const float* __restrict__ W, long long n,
                                                   const PackScratch* sc, uint32_t* __restrict__ out, int prescaled) {
  const float beta = pack_beta(sc, n, W, prescaled);
  const float s_w = __fdiv_rn(1.0f, beta);
  const long long nwords = n / 16;
  for (long long wi = blockIdx.x * (long long)blockDim.x + threadIdx.x; wi < nwords; wi += (long long)gridDim.x * blockDim.x) {
    const long long b = wi >> 3;
    const int m = (int)(wi & 7);
    uint32_t word = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(W + 128 * b + 32 * g + 4 * m));
      const int sh = 6 - 2 * g;
      word |= ternary_code(v.x, s_w) << (sh + 0);
      word |= ternary_code(v.y, s_w) << (sh + 8);
      word |= ternary_code(v.z, s_w) << (sh + 16);
      word |= ternary_code(v.w, s_w) << (sh + 24);
    }
    out[wi] = word;
  }
}

__global__ void k_pack_trailer(PackScratch* sc, long long n, const float* W, int prescaled) {
  const float beta = pack_beta(sc, n, W, prescaled);
  uint32_t* t = reinterpret_cast<uint32_t*>(sc);
  t[0] = __float_as_uint(beta);
#pragma unroll
  for (int i = 1; i < 8; ++i) t[i] = 0u;
}

__global__ void k_validate_clear(unsigned long long* counts) {
  counts[0] = counts[1] = counts[2] = 0ull;
}

__global__ void __launch_bounds__(256) k_validate_i2s(const uint32_t* __restrict__ words, long long nwords,
                                                     const uint8_t* __restrict__ trailer,
                                                     unsigned long long* counts) {
  __shared__ long long red[32];
  long long bad = 0;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nwords; i += (long long)gridDim.x * blockDim.x) {
    const uint32_t w = __ldg(words + i);
    bad += __popc(w & (w >> 1) & 0x55555555u);  // a field is 3 when both of its bits are set
  }
  bad = block_reduce(bad, red, AddOpLL());
  if (threadIdx.x == 0 && bad != 0) atomicAdd(&counts[0], (unsigned long long)bad);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    unsigned long long nz = 0;
    for (int i = 4; i < 32; ++i) nz += trailer[i] != 0;
    counts[1] = nz;
    const float beta = __uint_as_float(*reinterpret_cast<const uint32_t*>(trailer));
    counts[2] = (isfinite(beta) && beta > 0.0f) ? 0ull : 1ull;
  }
}

}  // namespace bitnet

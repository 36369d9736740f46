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
  const int e = fixed_point_exponent((double)M32, n);
  const double p2e = pow2_f64(e);
  long long part = 0;
  const long long n4 = n / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    part += __double2ll_rn(__dmul_rn((double)fabsf(v.x), p2e));
    part += __double2ll_rn(__dmul_rn((double)fabsf(v.y), p2e));
    part += __double2ll_rn(__dmul_rn((double)fabsf(v.z), p2e));
    part += __double2ll_rn(__dmul_rn((double)fabsf(v.w), p2e));
  }
  part = block_reduce(part, red, AddOpLL());
  if (threadIdx.x == 0) atomicAdd(&sc->sum, (unsigned long long)part);
}

// beta = max(mean|W|, 1e-5) from the scratch.
BN_DEV float pack_beta(const PackScratch* sc, long long n) {
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
                                                   const PackScratch* sc, uint32_t* __restrict__ out) {
  const float beta = pack_beta(sc, n);
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

__global__ void k_pack_trailer(PackScratch* sc, long long n) {
  const float beta = pack_beta(sc, n);
  uint32_t* t = reinterpret_cast<uint32_t*>(sc);
  t[0] = __float_as_uint(beta);
#pragma unroll
  for (int i = 1; i < 8; ++i) t[i] = 0u;
}

}  // namespace bitnet

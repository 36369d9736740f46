// Tensor-parallel pieces of the BitNet FFN: ffn_sub_norm + absmax int8 of h when h is split
// over ranks by columns (each rank holds the columns its gate/up shard produced), and the
// dequantisation of int32 accumulators that were summed over ranks.
//
// "Add optional RMSNorm support to BitNet quantization": BitNetMLP.forward =
// down(ffn_sub_norm(act(gate(x)) * up(x))).  The norm reduces over the whole row of h, so a
// rank only holds part of each reduction.  The row's reductions are exact (a maximum and an
// integer fixed-point sum), hence they can be finished across ranks by an all-reduce (MAX,
// then SUM of int64) without changing a bit:
//   1. shard_amax:   amax_r[t]  = max |h[t, k]| over the rank's columns      -> all-reduce MAX
//   2. shard_sumsq:  S_r[t]     = sum rint(h^2 2^e), e from the GLOBAL amax and
//                                 the GLOBAL row length (the same grid on every rank) -> SUM
//   3. shard_ymax:   inv[t] = 1 / sqrt(mean + eps) from the global S; y = (h inv) g;
//                    ymax_r[t] = max |y| over the rank's columns             -> all-reduce MAX
//   4. shard_quant:  s[t] = 127 / max(ymax, 1e-5); q = clamp(rint(y s)); the rank's
//                    partial sum of q (the down product subtracts it per shard)
// The down projection is split by its input columns the same way: each rank's int32
// accumulators sum q * w over its columns only; their sum over ranks is the full integer
// product, and dequant_acc rescales it: out = fp32(acc) * (beta / s).
#pragma once
#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int SHARD_THREADS = 256;

// max |h| of each row of h [T, Ks] (Ks % 4 == 0, rows 16-byte aligned).
__global__ void __launch_bounds__(SHARD_THREADS) k_shard_amax(const float* __restrict__ h, int T, int Ks,
                                                             float* __restrict__ amax) {
  __shared__ float red[32];
  pdl_launch_dependents();
  pdl_wait();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float4* row = reinterpret_cast<const float4*>(h + (long long)t * Ks);
    float m = 0.0f;
    for (int i = threadIdx.x; i < Ks / 4; i += blockDim.x) {
      const float4 v = row[i];
      m = fmaxf(fmaxf(m, fabsf(v.x)), fmaxf(fabsf(v.y), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    m = block_reduce(m, red, MaxOp());
    if (threadIdx.x == 0) amax[t] = m;
  }
}

// The rank's part of the exact fixed-point sum of h^2 on the grid of the whole row: M is
// the square of the row's global max |h|, n the global row length.
__global__ void __launch_bounds__(SHARD_THREADS) k_shard_sumsq(const float* __restrict__ h, int T, int Ks,
                                                              const float* __restrict__ amax_g, long long K_total,
                                                              long long* __restrict__ S) {
  __shared__ long long red[32];
  pdl_launch_dependents();
  pdl_wait();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float am = amax_g[t];
    long long part = 0;
    if (am > 0.0f) {
      const double p2e = pow2_f64(fixed_point_exponent(__dmul_rn((double)am, (double)am), K_total));
      const float4* row = reinterpret_cast<const float4*>(h + (long long)t * Ks);
      if (K_total >= kFixedSmallMinN) {
        for (int i = threadIdx.x; i < Ks / 4; i += blockDim.x) {
          const float4 v = row[i];
          part += fixed_sq_term_t<true>(v.x, p2e) + fixed_sq_term_t<true>(v.y, p2e) + fixed_sq_term_t<true>(v.z, p2e) +
                  fixed_sq_term_t<true>(v.w, p2e);
        }
      } else {
        for (int i = threadIdx.x; i < Ks / 4; i += blockDim.x) {
          const float4 v = row[i];
          part += fixed_sq_term(v.x, p2e) + fixed_sq_term(v.y, p2e) + fixed_sq_term(v.z, p2e) + fixed_sq_term(v.w, p2e);
        }
      }
    }
    part = block_reduce(part, red, AddOpLL());
    if (threadIdx.x == 0) S[t] = part;
  }
}

// inv = 1 / sqrt(mean + eps) from the all-reduced sum, and the rank's max |y| with
// y = (h * inv) * g (gain NULL: no norm, inv = 1 and y = h).
__global__ void __launch_bounds__(SHARD_THREADS) k_shard_ymax(const float* __restrict__ h, const float* __restrict__ gain,
                                                             int T, int Ks, const float* __restrict__ amax_g,
                                                             const long long* __restrict__ S_g, long long K_total,
                                                             float eps, float* __restrict__ inv_out,
                                                             float* __restrict__ ymax) {
  __shared__ float red[32];
  pdl_launch_dependents();
  pdl_wait();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float am = amax_g[t];
    if (gain == nullptr) {
      if (threadIdx.x == 0) {
        inv_out[t] = 1.0f;
        ymax[t] = am;
      }
      continue;
    }
    float ms = 0.0f;
    if (am > 0.0f) ms = fixed_point_mean(S_g[t], fixed_point_exponent(__dmul_rn((double)am, (double)am), K_total), K_total);
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    const float4* row = reinterpret_cast<const float4*>(h + (long long)t * Ks);
    const float4* g4 = reinterpret_cast<const float4*>(gain);
    float m = 0.0f;
    for (int i = threadIdx.x; i < Ks / 4; i += blockDim.x) {
      const float4 v = row[i], g = __ldg(g4 + i);
      m = fmaxf(m, fabsf(__fmul_rn(__fmul_rn(v.x, inv), g.x)));
      m = fmaxf(m, fabsf(__fmul_rn(__fmul_rn(v.y, inv), g.y)));
      m = fmaxf(m, fabsf(__fmul_rn(__fmul_rn(v.z, inv), g.z)));
      m = fmaxf(m, fabsf(__fmul_rn(__fmul_rn(v.w, inv), g.w)));
    }
    m = block_reduce(m, red, MaxOp());
    if (threadIdx.x == 0) {
      inv_out[t] = inv;
      ymax[t] = m;
    }
  }
}

// q = clamp(rint(y * s), -128, 127) with s = 127 / max(global max |y|, 1e-5), the rank's
// partial sum of q, and s itself.
__global__ void __launch_bounds__(SHARD_THREADS) k_shard_quant(const float* __restrict__ h, const float* __restrict__ gain,
                                                              int T, int Ks, const float* __restrict__ inv_in,
                                                              const float* __restrict__ ymax_g, int8_t* __restrict__ q,
                                                              float* __restrict__ s_out, int32_t* __restrict__ sum_q) {
  __shared__ int red[32];
  pdl_launch_dependents();
  pdl_wait();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float inv = inv_in[t];
    const float s = __fdiv_rn(127.0f, fmaxf(ymax_g[t], 1e-5f));
    const float4* row = reinterpret_cast<const float4*>(h + (long long)t * Ks);
    const float4* g4 = reinterpret_cast<const float4*>(gain);
    int sum = 0;
    for (int i = threadIdx.x; i < Ks / 4; i += blockDim.x) {
      const float4 v = row[i];
      float y[4] = {v.x, v.y, v.z, v.w};
      if (gain != nullptr) {
        const float4 g = __ldg(g4 + i);
        y[0] = __fmul_rn(__fmul_rn(v.x, inv), g.x);
        y[1] = __fmul_rn(__fmul_rn(v.y, inv), g.y);
        y[2] = __fmul_rn(__fmul_rn(v.z, inv), g.z);
        y[3] = __fmul_rn(__fmul_rn(v.w, inv), g.w);
      }
      uint32_t w = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int qv = quant_code(__fmul_rn(y[j], s));
        sum += qv;
        w |= (uint32_t)(qv & 0xFF) << (8 * j);
      }
      reinterpret_cast<uint32_t*>(q + (long long)t * Ks)[i] = w;
    }
    sum = block_reduce(sum, red, AddOpI());
    if (threadIdx.x == 0) {
      s_out[t] = s;
      sum_q[t] = sum;
    }
  }
}

// out[t, n] = fp32(acc[t, n]) * (beta / s[t]), bf16 (nearest even) or fp32.
__global__ void __launch_bounds__(SHARD_THREADS) k_dequant_acc(const int32_t* __restrict__ acc, const float* __restrict__ s,
                                                              const float* __restrict__ beta_p, long long T, int N,
                                                              void* __restrict__ out, int out_dtype) {
  pdl_launch_dependents();
  pdl_wait();
  const float beta = __ldg(beta_p);
  const long long total = T * (long long)N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / N;
    store_out(out, out_dtype, i, dequant(acc[i], __fdiv_rn(beta, s[t])));
  }
}

}  // namespace bitnet

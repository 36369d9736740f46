// K-quant: fused BitNetRMSNorm + per-token absmax + int8 quantisation.
//
// "Add optional RMSNorm support to BitNet quantization (config + layers)": BitLinear
// applies BitNetRMSNorm (eps 1e-6 by default) to the activations before they are
// quantised; with use_rms_norm off (gain == nullptr) the activations go straight to
// the absmax quantiser.  "More BitNet-like IQ1_S quantizations": the activations of
// BitNet b1.58 are 8-bit.
//
// One CTA per token.  The row is staged once in shared memory as fp32; the three
// reductions (max|x|, the fixed-point sum of x^2, max|y|) and the sum of q are exact,
// so the result is independent of the thread count and of the order of summation.
#pragma once
#include "common.cuh"

namespace bitnet {

template <typename TIn>
struct RowLoader;

template <>
struct RowLoader<__nv_bfloat16> {
  static constexpr int V = 8;  // elements per 16-byte vector
  BN_DEV static void load(const __nv_bfloat16* p, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  BN_DEV static float load1(const __nv_bfloat16* p) { return bf16_to_f32(*reinterpret_cast<const uint16_t*>(p)); }
};

template <>
struct RowLoader<float> {
  static constexpr int V = 8;
  BN_DEV static void load(const float* p, float* o) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
  BN_DEV static float load1(const float* p) { return *p; }
};

// Quantise one staged row xs[0..K) in place of nothing: writes q, s_x, sum_q of the row.
// `vec` says whether K % 8 == 0 and the row pointers are 16-byte aligned.
BN_DEV void quantise_staged_row(float* xs, int K, const float* gain, float eps, int8_t* qrow,
                                float* s_out, int32_t* sum_out, bool vec, void* red_scratch,
                                float amax_x) {
  float* redf = reinterpret_cast<float*>(red_scratch);
  long long* redl = reinterpret_cast<long long*>(red_scratch);
  int* redi = reinterpret_cast<int*>(red_scratch);
  const int tid = threadIdx.x, nt = blockDim.x;

  float a;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (amax_x > 0.0f) {
      const double M = __dmul_rn((double)amax_x, (double)amax_x);
      const int e = fixed_point_exponent(M, K);
      const double p2e = pow2_f64(e);
      long long part = 0;
      for (int k = tid; k < K; k += nt) {
        const double v = (double)xs[k];
        part += __double2ll_rn(__dmul_rn(__dmul_rn(v, v), p2e));
      }
      const long long S = block_reduce(part, redl, AddOpLL());
      ms = fixed_point_mean(S, e, K);
    }
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float am = 0.0f;
    for (int k = tid; k < K; k += nt) {
      const float y = __fmul_rn(__fmul_rn(xs[k], inv), __ldg(gain + k));
      xs[k] = y;
      am = fmaxf(am, fabsf(y));
    }
    a = block_reduce(am, redf, MaxOp());
  } else {
    a = amax_x;  // y = x
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
  if (vec) {
    for (int k = tid * 8; k < K; k += nt * 8) {
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t packed = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int v = __float2int_rn(__fmul_rn(xs[k + 4 * h + j], s));
          v = min(127, max(-128, v));
          sum += v;
          packed |= (uint32_t)(v & 0xFF) << (8 * j);
        }
        w[h] = packed;
      }
      *reinterpret_cast<uint2*>(qrow + k) = make_uint2(w[0], w[1]);
    }
  } else {
    for (int k = tid; k < K; k += nt) {
      int v = __float2int_rn(__fmul_rn(xs[k], s));
      v = min(127, max(-128, v));
      sum += v;
      qrow[k] = (int8_t)v;
    }
  }
  sum = block_reduce(sum, redi, AddOpI());
  if (tid == 0) {
    *s_out = s;
    *sum_out = sum;
  }
}

// Stage row `x` [K] into xs as fp32; returns max|x| over the block.
template <typename TIn>
BN_DEV float stage_row(const TIn* x, int K, float* xs, bool vec, void* red_scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  float am = 0.0f;
  if (vec) {
    for (int k = tid * 8; k < K; k += nt * 8) {
      float v[8];
      RowLoader<TIn>::load(x + k, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        xs[k + j] = v[j];
        am = fmaxf(am, fabsf(v[j]));
      }
    }
  } else {
    for (int k = tid; k < K; k += nt) {
      const float v = RowLoader<TIn>::load1(x + k);
      xs[k] = v;
      am = fmaxf(am, fabsf(v));
    }
  }
  return block_reduce(am, reinterpret_cast<float*>(red_scratch), MaxOp());
}

template <typename TIn>
__global__ void __launch_bounds__(1024) k_rmsnorm_quant(const TIn* __restrict__ x, const float* __restrict__ gain,
                                                        float eps, int K, int8_t* __restrict__ q,
                                                        float* __restrict__ s_x, int32_t* __restrict__ sum_q,
                                                        int vec) {
  extern __shared__ float xs[];
  __shared__ long long red[32];
  const long long t = blockIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const float amax = stage_row<TIn>(x + t * K, K, xs, vec != 0, red);
  quantise_staged_row(xs, K, gain, eps, q + t * K, s_x + t, sum_q + t, vec != 0, red, amax);
}

// The same arithmetic for rows of K <= 2048 * NG values held in registers by 256 threads
// (thread i owns elements 8(i + 256 j) .. +7, j < NG), so a CTA reads its row once and
// several tokens fit on one SM.  Reductions use one barrier each (two scratch halves used
// in turn).
constexpr int QR_THREADS = 256;
constexpr int QR_WARPS = QR_THREADS / 32;

template <typename T>
BN_DEV T qr_reduce(T v, T* scratch, int& flip, bool is_max) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const T w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? (v > w ? v : w) : v + w;
  }
  T* b = scratch + flip * QR_WARPS;
  flip ^= 1;
  if ((threadIdx.x & 31) == 0) b[threadIdx.x >> 5] = v;
  __syncthreads();
  T r = b[0];
#pragma unroll
  for (int w = 1; w < QR_WARPS; ++w) r = is_max ? (r > b[w] ? r : b[w]) : r + b[w];
  return r;
}

template <typename TIn, int NG>
__global__ void __launch_bounds__(QR_THREADS) k_rmsnorm_quant_regs(const TIn* __restrict__ x,
                                                                  const float* __restrict__ gain, float eps, int K,
                                                                  int8_t* __restrict__ q, float* __restrict__ s_x,
                                                                  int32_t* __restrict__ sum_q) {
  __shared__ float redf[2 * QR_WARPS];
  __shared__ long long redl[2 * QR_WARPS];
  __shared__ int redi[2 * QR_WARPS];
  int ff = 0, fl = 0, fi = 0;
  const long long t = blockIdx.x;
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const TIn* xr = x + t * K;
  float v[NG][8];
  float am = 0.0f;
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    const int k = 8 * (tid + QR_THREADS * j);
    if (k < K) {
      RowLoader<TIn>::load(xr + k, v[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[j][i]));
  }
  am = qr_reduce(am, redf, ff, true);
  float a = am;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (am > 0.0f) {
      const double M = __dmul_rn((double)am, (double)am);
      const int e = fixed_point_exponent(M, K);
      const double p2e = pow2_f64(e);
      long long part = 0;
#pragma unroll
      for (int j = 0; j < NG; ++j)
        if (8 * (tid + QR_THREADS * j) < K) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const double d = (double)v[j][i];
            part += __double2ll_rn(__dmul_rn(__dmul_rn(d, d), p2e));
          }
        }
      ms = fixed_point_mean(qr_reduce(part, redl, fl, false), e, K);
    }
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float ay = 0.0f;
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      const int k = 8 * (tid + QR_THREADS * j);
      if (k < K) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[j][i] = __fmul_rn(__fmul_rn(v[j][i], inv), __ldg(gain + k + i));
          ay = fmaxf(ay, fabsf(v[j][i]));
        }
      }
    }
    a = qr_reduce(ay, redf, ff, true);
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
  int8_t* qr = q + t * K;
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    const int k = 8 * (tid + QR_THREADS * j);
    if (k < K) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qv = __float2int_rn(__fmul_rn(v[j][i], s));
        qv = min(127, max(-128, qv));
        sum += qv;
        w[i >> 2] |= (uint32_t)(qv & 0xFF) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2*>(qr + k) = make_uint2(w[0], w[1]);
    }
  }
  sum = qr_reduce(sum, redi, fi, false);
  if (tid == 0) {
    s_x[t] = s;
    sum_q[t] = sum;
  }
}

}  // namespace bitnet

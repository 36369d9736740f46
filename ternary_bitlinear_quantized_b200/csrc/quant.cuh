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
      if (K >= kFixedSmallMinN)
        for (int k = tid; k < K; k += nt) part += fixed_sq_term_t<true>(xs[k], p2e);
      else
        for (int k = tid; k < K; k += nt) part += fixed_sq_term(xs[k], p2e);
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
          int v = quant_code(__fmul_rn(xs[k + 4 * h + j], s));
          sum += v;
          packed |= (uint32_t)(v & 0xFF) << (8 * j);
        }
        w[h] = packed;
      }
      *reinterpret_cast<uint2*>(qrow + k) = make_uint2(w[0], w[1]);
    }
  } else {
    for (int k = tid; k < K; k += nt) {
      int v = quant_code(__fmul_rn(xs[k], s));
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

// Long fp32 rows (the FFN's h at prefill): one CTA per SM, persistent over rows blockIdx.x,
// blockIdx.x + gridDim.x, ...; two row buffers in shared memory, the next row fetched with a
// set of bulk copies (completing on the buffer's mbarrier) while the current one is reduced,
// so the row reads stream at the HBM rate instead of waiting behind each row's reduction
// chain.  Thread i owns the four elements 4 (i + QL_THREADS j) .. + 3 of every group j, read
// from shared memory with 16-byte loads; its gain values stay in registers for all rows
// (reading them from L2 per row put a memory round trip behind every element of the y pass).
// The y pass writes y over the row; the q pass writes four codes per 4-byte store.  The
// reductions use one barrier each and are the row's only barriers.  The arithmetic is
// quantise_staged_row's.  K % 4 == 0, K <= 4 QL_THREADS QL_MAXV, rows 16-byte aligned,
// 2 K floats of shared memory.
constexpr int QL_THREADS = 1024;
constexpr int QL_MAXV = 7;  // K <= 28672
constexpr int QL_PARTS = 8;  // bulk copies per row
__global__ void __launch_bounds__(QL_THREADS, 1) k_rmsnorm_quant_long(const float* __restrict__ x,
                                                                     const float* __restrict__ gain, float eps,
                                                                     int T, int K, int8_t* __restrict__ q,
                                                                     float* __restrict__ s_x,
                                                                     int32_t* __restrict__ sum_q) {
  extern __shared__ __align__(16) float ql_buf[];  // [2][K]
  __shared__ long long red[2][32];  // the two scratch areas of the reductions, used in turn
  int ra = 0;
  __shared__ __align__(8) unsigned long long ql_bar[2];  // one per row buffer: its bulk copy landed
  volatile __shared__ int ql_abort;
  const int tid = threadIdx.x;
  const int K4 = K >> 2;
  float4 gr[QL_MAXV];
#pragma unroll
  for (int j = 0; j < QL_MAXV; ++j) {
    const int k4 = tid + QL_THREADS * j;
    gr[j] = (gain != nullptr && k4 < K4) ? __ldg(reinterpret_cast<const float4*>(gain) + k4)
                                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  if (tid == 0) {
    mbar_init(smem_addr(&ql_bar[0]), 1);
    mbar_init(smem_addr(&ql_bar[1]), 1);
    ql_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();
  // A row is fetched by thread 0 as QL_PARTS bulk copies (several in flight stream faster than
  // one long copy), all completing on the buffer's barrier.
  const uint32_t row_bytes = (uint32_t)K * 4u;
  const uint32_t part = (row_bytes + 16u * QL_PARTS - 1u) / (16u * QL_PARTS) * 16u;  // multiple of 16
  auto fetch = [&](long long row, int b) {
    const uint32_t bar = smem_addr(&ql_bar[b]), dst = smem_addr(ql_buf + b * K);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(x + row * K);
    mbar_arrive_expect_tx(bar, row_bytes);
    for (uint32_t o = 0; o < row_bytes; o += part) bulk_g2s(dst + o, src + o, min(part, row_bytes - o), bar);
  };
  long long row = blockIdx.x;
  int issued = 0;
  if (tid == 0 && row < T) {
    fetch(row, 0);
    issued = 1;
  }
  for (int it = 0; row < T; ++it, row += gridDim.x) {
    const int b = it & 1;
    float4* cur = reinterpret_cast<float4*>(ql_buf + b * K);
    const long long next = row + gridDim.x;
    if (tid == 0 && next < T) {  // the other buffer was released by the last barrier of it - 1
      fetch(next, b ^ 1);
      ++issued;
    }
    // A wait that gives up is seen by every thread after the first reduction's barrier (the
    // max pass before it may read an incomplete row; its result is not used).
    if (!mbar_wait_bounded(smem_addr(&ql_bar[b]), (uint32_t)((it >> 1) & 1))) ql_abort = 1;
    float am = 0.0f;
#pragma unroll
    for (int j = 0; j < QL_MAXV; ++j) {
      const int k4 = tid + QL_THREADS * j;
      if (k4 < K4) {
        const float4 v = cur[k4];
        am = fmaxf(am, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
    am = block_reduce_alt(am, reinterpret_cast<float*>(red[ra++ & 1]), MaxOp());
    if (ql_abort) break;
    float a = am, inv = 1.0f;
    if (gain != nullptr) {
      float ms = 0.0f;
      if (am > 0.0f) {
        const int e = fixed_point_exponent(__dmul_rn((double)am, (double)am), K);
        const double p2e = pow2_f64(e);
        long long part = 0;
        if (K >= kFixedSmallMinN) {
          // Each term rint(v^2 2^e) < 2^51 as the bits of the fp64 sum 1.5 * 2^52 + v^2 2^e:
          // v (v 2^e) is exact (a power-of-two scaling, or below 2^-1022 where the term is 0
          // either way), so one fused multiply-add rounds exactly once, like the rounding add
          // of fixed_sq_term_t.  The bits are summed as they are (mod 2^64) and the offset of
          // every term taken off once.
          unsigned long long bits = 0ull;
          int n = 0;
#pragma unroll
          for (int j = 0; j < QL_MAXV; ++j) {
            const int k4 = tid + QL_THREADS * j;
            if (k4 < K4) {
              const float4 v = cur[k4];
              const double d0 = (double)v.x, d1 = (double)v.y, d2 = (double)v.z, d3 = (double)v.w;
              constexpr double kRound = 6755399441055744.0;  // 1.5 * 2^52
              bits += (unsigned long long)__double_as_longlong(__fma_rn(d0, __dmul_rn(d0, p2e), kRound)) +
                      (unsigned long long)__double_as_longlong(__fma_rn(d1, __dmul_rn(d1, p2e), kRound)) +
                      (unsigned long long)__double_as_longlong(__fma_rn(d2, __dmul_rn(d2, p2e), kRound)) +
                      (unsigned long long)__double_as_longlong(__fma_rn(d3, __dmul_rn(d3, p2e), kRound));
              n += 4;
            }
          }
          part = (long long)(bits - (unsigned long long)n * 0x4338000000000000ull);
        } else {
#pragma unroll
          for (int j = 0; j < QL_MAXV; ++j) {
            const int k4 = tid + QL_THREADS * j;
            if (k4 < K4) {
              const float4 v = cur[k4];
              part += fixed_sq_term(v.x, p2e) + fixed_sq_term(v.y, p2e) + fixed_sq_term(v.z, p2e) +
                      fixed_sq_term(v.w, p2e);
            }
          }
        }
        ms = fixed_point_mean(block_reduce_alt(part, red[ra++ & 1], AddOpLL()), e, K);
      }
      inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
      float ay = 0.0f;
#pragma unroll
      for (int j = 0; j < QL_MAXV; ++j) {
        const int k4 = tid + QL_THREADS * j;
        if (k4 < K4) {
          float4 v = cur[k4];
          v.x = __fmul_rn(__fmul_rn(v.x, inv), gr[j].x);
          v.y = __fmul_rn(__fmul_rn(v.y, inv), gr[j].y);
          v.z = __fmul_rn(__fmul_rn(v.z, inv), gr[j].z);
          v.w = __fmul_rn(__fmul_rn(v.w, inv), gr[j].w);
          ay = fmaxf(ay, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
          cur[k4] = v;  // y, read by the q pass
        }
      }
      fence_proxy_async_smem();  // this thread's y writes ordered before the buffer's next bulk copy
      a = block_reduce_alt(ay, reinterpret_cast<float*>(red[ra++ & 1]), MaxOp());
    }
    const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
    // quant_code's steps with its offset kept: the fp32 bits of clamp(p) + 1.5 * 2^23 are
    // 0x4B400000 + code, so their low byte is the code's byte; the bits are summed as they are
    // (mod 2^32) and the offset of every element taken off once.
    uint32_t cbits = 0u;
    int n = 0;
    uint32_t* qrow = reinterpret_cast<uint32_t*>(q + row * K);
#pragma unroll
    for (int j = 0; j < QL_MAXV; ++j) {
      const int k4 = tid + QL_THREADS * j;
      if (k4 < K4) {
        const float4 y = cur[k4];
        const float p[4] = {__fmul_rn(y.x, s), __fmul_rn(y.y, s), __fmul_rn(y.z, s), __fmul_rn(y.w, s)};
        uint32_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float c = p[i] == p[i] ? fminf(fmaxf(p[i], -128.0f), 127.0f) : 0.0f;  // NaN: code 0
          b[i] = __float_as_uint(__fadd_rn(c, 12582912.0f));
        }
        cbits += (b[0] + b[1]) + (b[2] + b[3]);
        n += 4;
        qrow[k4] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
      }
    }
    const int sum = block_reduce_alt((int)(cbits - (uint32_t)n * 0x4B400000u), reinterpret_cast<int*>(red[ra++ & 1]),
                                     AddOpI());
    if (tid == 0) {
      s_x[row] = s;
      sum_q[row] = sum;
    }
    // The buffer is refilled by the fetch of iteration it + 1, issued after the barrier of the
    // reduction above, which every thread reaches after its last read of the buffer.
  }
  // After a wait gave up, the copies still in flight land (fixed limit) before the CTA exits.
  if (tid == 0 && ql_abort)
    for (int k = (issued > 2 ? issued - 2 : 0); k < issued; ++k) mbar_drain(smem_addr(&ql_bar[k & 1]), (uint32_t)((k >> 1) & 1));
}

// The same arithmetic with W warps per row (W = 1, 2 or 4) and 8 / W rows per 256-thread
// CTA, for rows of K <= 2048 W values (K a multiple of 8, 16-byte aligned rows).  Lane l of
// the row's warp `rank` holds elements 8 (l + 32 (rank + W j)) .. +7, j < 8, in registers, so
// the row is read once; the reductions are warp shuffles, joined across the W warps by one
// named barrier each (two scratch halves used in turn).  Many rows are in flight per SM,
// which hides the latency of the loads and of the reduction chain.
constexpr int QW_THREADS = 256;
constexpr int QW_GROUPS = 8;

template <int W, typename T, typename Op>
BN_DEV T qw_reduce(T v, T* slots, int& flip, int bar_id, int rank, Op op) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (W == 1) return v;
  T* b = slots + flip * W;
  flip ^= 1;
  if ((threadIdx.x & 31) == 0) b[rank] = v;
  named_sync(bar_id, 32 * W);
  T r = b[0];
#pragma unroll
  for (int i = 1; i < W; ++i) r = op(r, b[i]);
  return r;
}

template <typename TIn, int W>
__global__ void __launch_bounds__(QW_THREADS) k_rmsnorm_quant_warps(const TIn* __restrict__ x,
                                                                   const float* __restrict__ gain, float eps, int T,
                                                                   int K, int8_t* __restrict__ q,
                                                                   float* __restrict__ s_x, int32_t* __restrict__ sum_q) {
  constexpr int ROWS = QW_THREADS / 32 / W;
  __shared__ float redf[ROWS][2 * W];
  __shared__ long long redl[ROWS][2 * W];
  __shared__ int redi[ROWS][2 * W];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = warp / W, rank = warp - rr * W;
  const long long t = (long long)blockIdx.x * ROWS + rr;
  pdl_launch_dependents();
  pdl_wait();
  if (t >= T) return;  // every warp of the row leaves together
  const int bar = 1 + rr;
  int ff = 0, fl = 0, fi = 0;
  const TIn* xr = x + t * K;
  float v[QW_GROUPS][8];
  float am = 0.0f;
#pragma unroll
  for (int j = 0; j < QW_GROUPS; ++j) {
    const int k = 8 * (lane + 32 * (rank + W * j));
    if (k < K) {
      RowLoader<TIn>::load(xr + k, v[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[j][i]));
  }
  am = qw_reduce<W>(am, &redf[rr][0], ff, bar, rank, MaxOp());
  float a = am;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (am > 0.0f) {
      const double M = __dmul_rn((double)am, (double)am);
      const int e = fixed_point_exponent(M, K);
      const double p2e = pow2_f64(e);
      long long part = 0;
      if (K >= kFixedSmallMinN) {
#pragma unroll
        for (int j = 0; j < QW_GROUPS; ++j)
          if (8 * (lane + 32 * (rank + W * j)) < K) {
#pragma unroll
            for (int i = 0; i < 8; ++i) part += fixed_sq_term_t<true>(v[j][i], p2e);
          }
      } else {
#pragma unroll
        for (int j = 0; j < QW_GROUPS; ++j)
          if (8 * (lane + 32 * (rank + W * j)) < K) {
#pragma unroll
            for (int i = 0; i < 8; ++i) part += fixed_sq_term(v[j][i], p2e);
          }
      }
      ms = fixed_point_mean(qw_reduce<W>(part, &redl[rr][0], fl, bar, rank, AddOpLL()), e, K);
    }
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float ay = 0.0f;
#pragma unroll
    for (int j = 0; j < QW_GROUPS; ++j) {
      const int k = 8 * (lane + 32 * (rank + W * j));
      if (k < K) {
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(gain + k));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(gain + k + 4));
        const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[j][i] = __fmul_rn(__fmul_rn(v[j][i], inv), g[i]);
          ay = fmaxf(ay, fabsf(v[j][i]));
        }
      }
    }
    a = qw_reduce<W>(ay, &redf[rr][0], ff, bar, rank, MaxOp());
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
  int8_t* qr = q + t * K;
#pragma unroll
  for (int j = 0; j < QW_GROUPS; ++j) {
    const int k = 8 * (lane + 32 * (rank + W * j));
    if (k < K) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qv = quant_code(__fmul_rn(v[j][i], s));
        sum += qv;
        w[i >> 2] |= (uint32_t)(qv & 0xFF) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2*>(qr + k) = make_uint2(w[0], w[1]);
    }
  }
  sum = qw_reduce<W>(sum, &redi[rr][0], fi, bar, rank, AddOpI());
  if (rank == 0 && lane == 0) {
    s_x[t] = s;
    sum_q[t] = sum;
  }
}

}  // namespace bitnet

// K-dec: the BitLinear product for few tokens (decode), on the register-fed int8
// tensor-core path (mma.sync m16n8k32, u8 weights x s8 activations -> s32).
//
// "fix: I2_S ARM kernel layout + squared-ReLU FFN - passes the gate on the official
// 2B4T GGUF", bullet "ggml-cpu: I2_S NEON kernel for the canonical layout": codes
// c = w + 1 in the interleaved 128/32 layout, and the caller subtracts the activation
// sum, so acc = sum q*c - sum q.
//
// Work split: one CTA per tile of 16 weight rows (a contiguous byte range of the
// packed tensor); its warps split K.  A warp step covers 256 in-features of the 16 rows:
// thread (gid = lane/4, r = lane%4) loads 16 bytes of rows gid and gid+8 at byte
// 64 step + 16 r, i.e. words 4(r%2)..4(r%2)+3 of block 2 step + r/2.  Field g of a
// word holds the codes of 4 consecutive in-features (k = 128 j + 32 g + 4 m + 0..3),
// so masking the word with 0x03030303 << (6 - 2g) gives an mma A register directly --
// the codes scaled by 4^(3-g), which stays in u8 range.  Each field accumulates into
// its own set of registers; the sets are combined exactly at the end
// (acc = D0/64 + D1/16 + D2/4 + D3).  The dot product is order-free, so the pairing of
// mma k-slots with in-features only has to agree between A and B: the B registers of
// thread (gid, r) hold the activations of token gid at the same in-features.
//
// Activation sum, dequantisation (out = fp32(acc) * (beta / s_x)) and, for the FFN,
// the relu2 / SiLU product h = act(g) * u are fused into the epilogue.
#pragma once
#include "common.cuh"

namespace bitnet {

constexpr int GEMV_WARPS = 8;
constexpr int GEMV_ROWS = 16;
constexpr int GEMV_TOK = 16;  // tokens per pass (two n8 mma groups)

struct GemvTensor {
  const uint8_t* packed;
  void* out;
  int32_t* acc_debug;
  int N;
  int tile_begin;
};

struct GemvArgs {
  const int8_t* q;
  const float* s_x;
  const int32_t* sum_q;
  int T;
  int K;
  int n_tensors;
  int n_tiles;
  GemvTensor t[4];
  int out_dtype;  // bitnet_dtype
  int act;        // bitnet_act (FFN mode)
  float* h;       // FFN mode output [T, N] fp32
};

BN_DEV void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ SiLU's exp
// exp in fp64 with a fixed operation sequence: k = rint(x / ln2),
// r = (x - k ln2_hi) - k ln2_lo (Cody and Waite's two-part reduction, ln2_hi keeps the
// top 32 significant bits of ln 2), the degree-17 Taylor series of exp(r) in Horner
// form, then p * 2^k.  0 below -700, +inf above 709.
constexpr double kLn2 = 0x1.62e42fefa39efp-1;
constexpr double kLn2Hi = 0x1.62e42fee00000p-1;
constexpr double kLn2Lo = 0x1.a39ef35793c76p-33;
constexpr double inv_factorial(int n) {
  double f = 1.0;
  for (int i = 2; i <= n; ++i) f *= (double)i;
  return 1.0 / f;
}
__constant__ double c_exp_taylor[18] = {
    inv_factorial(0),  inv_factorial(1),  inv_factorial(2),  inv_factorial(3),  inv_factorial(4),  inv_factorial(5),
    inv_factorial(6),  inv_factorial(7),  inv_factorial(8),  inv_factorial(9),  inv_factorial(10), inv_factorial(11),
    inv_factorial(12), inv_factorial(13), inv_factorial(14), inv_factorial(15), inv_factorial(16), inv_factorial(17)};

BN_DEV double pinned_exp(double x) {
  if (x < -700.0) return 0.0;
  if (x > 709.0) return __longlong_as_double(0x7FF0000000000000ll);
  const double k = rint(__ddiv_rn(x, kLn2));
  const double r = __dsub_rn(__dsub_rn(x, __dmul_rn(k, kLn2Hi)), __dmul_rn(k, kLn2Lo));
  double p = c_exp_taylor[17];
#pragma unroll
  for (int n = 16; n >= 0; --n) p = __dadd_rn(__dmul_rn(p, r), c_exp_taylor[n]);
  return __dmul_rn(p, pow2_f64((int)k));
}

// h = act(g) * u in fp32 (relu2: (r*r)*u with r = max(g, 0); SiLU: fp32(g / (1 + exp(-g))) * u).
BN_DEV float ffn_act(float g, float u, int act) {
  if (act == BITNET_RELU2) {
    const float r = fmaxf(g, 0.0f);
    return __fmul_rn(__fmul_rn(r, r), u);
  }
  const double gd = (double)g;
  const float s = __double2float_rn(__ddiv_rn(gd, __dadd_rn(1.0, pinned_exp(-gd))));
  return __fmul_rn(s, u);
}

BN_DEV float dequant(int acc, float f) { return __fmul_rn(__int2float_rn(acc), f); }

BN_DEV void store_out(void* out, int dtype, long long idx, float v) {
  if (dtype == BITNET_BF16)
    reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(out)[idx] = v;
}

// Accumulate one 16-row tile of one tensor over this warp's K steps, for the 16 tokens
// tok0 .. tok0+15.  d[tg][i]: combined int32 accumulators (tg = token group of 8).
BN_DEV void gemv_tile_accumulate(const uint8_t* rowA, const uint8_t* rowB, const int8_t* q, int T, int K,
                                 int tok0, int warp, int gid, int r, int (&d)[2][4]) {
  int acc[2][4][4];
#pragma unroll
  for (int tg = 0; tg < 2; ++tg)
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[tg][g][i] = 0;

  const int row_bytes = K >> 2;
  const int n_steps = (row_bytes + 63) >> 6;
  const int t_a = tok0 + gid, t_b = tok0 + 8 + gid;
  const bool ta_ok = t_a < T, tb_ok = t_b < T;
  for (int step = warp; step < n_steps; step += GEMV_WARPS) {
    const int boff = step * 64 + 16 * r;
    const bool valid = boff < row_bytes;
    uint4 wa = make_uint4(0, 0, 0, 0), wb = make_uint4(0, 0, 0, 0);
    if (valid && rowA) wa = ldg_nc_v4(rowA + boff);
    if (valid && rowB) wb = ldg_nc_v4(rowB + boff);
    const int kb = step * 256 + 128 * (r >> 1) + 16 * (r & 1);
    uint4 xa[4], xb[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      xa[g] = (valid && ta_ok) ? __ldg(reinterpret_cast<const uint4*>(q + (long long)t_a * K + kb + 32 * g)) : make_uint4(0, 0, 0, 0);
      xb[g] = (valid && tb_ok) ? __ldg(reinterpret_cast<const uint4*>(q + (long long)t_b * K + kb + 32 * g)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t mask = 0x03030303u << (6 - 2 * g);
      // pair p = 0: words 0,1 ; p = 1: words 2,3
      mma_u8s8(acc[0][g], wa.x & mask, wb.x & mask, wa.y & mask, wb.y & mask, xa[g].x, xa[g].y);
      mma_u8s8(acc[0][g], wa.z & mask, wb.z & mask, wa.w & mask, wb.w & mask, xa[g].z, xa[g].w);
      if (T > 8) {
        mma_u8s8(acc[1][g], wa.x & mask, wb.x & mask, wa.y & mask, wb.y & mask, xb[g].x, xb[g].y);
        mma_u8s8(acc[1][g], wa.z & mask, wb.z & mask, wa.w & mask, wb.w & mask, xb[g].z, xb[g].w);
      }
    }
  }
#pragma unroll
  for (int tg = 0; tg < 2; ++tg)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d[tg][i] = (acc[tg][0][i] >> 6) + (acc[tg][1][i] >> 4) + (acc[tg][2][i] >> 2) + acc[tg][3][i];
}

// Sum the per-warp accumulators of a tile through shared memory; on return, threads of
// warp 0 hold the CTA totals in d.  red: [GEMV_WARPS][32][8] ints.
BN_DEV void gemv_reduce_warps(int (&d)[2][4], int* red, int warp, int lane) {
  __syncthreads();
#pragma unroll
  for (int tg = 0; tg < 2; ++tg)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[(warp * 32 + lane) * 8 + tg * 4 + i] = d[tg][i];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int tg = 0; tg < 2; ++tg)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int s = 0;
        for (int w = 0; w < GEMV_WARPS; ++w) s += red[(w * 32 + lane) * 8 + tg * 4 + i];
        d[tg][i] = s;
      }
  }
}

template <bool FFN>
__global__ void __launch_bounds__(GEMV_WARPS * 32) k_gemv_mma(const GemvArgs a) {
  __shared__ int red[2][GEMV_WARPS * 32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, r = lane & 3;
  const int tile = blockIdx.x;
  int ti = 0;
  if (!FFN) {
    while (ti + 1 < a.n_tensors && tile >= a.t[ti + 1].tile_begin) ++ti;
  }
  const GemvTensor& TA = a.t[ti];
  const int N = TA.N;
  const int n0 = (tile - TA.tile_begin) * GEMV_ROWS;
  const int nrows = min(GEMV_ROWS, N - n0);
  const long long row_bytes = a.K >> 2;
  const uint8_t* baseA = TA.packed + (long long)n0 * row_bytes;
  const uint8_t* baseU = FFN ? a.t[1].packed + (long long)n0 * row_bytes : nullptr;

  // Weights do not depend on the previous kernel: pull this tile into L2 now.
  if (threadIdx.x == 0) {
    prefetch_l2_bulk(baseA, (uint32_t)(nrows * row_bytes));
    if (FFN) prefetch_l2_bulk(baseU, (uint32_t)(nrows * row_bytes));
  }
  pdl_launch_dependents();
  pdl_wait();

  const float betaA = *reinterpret_cast<const float*>(TA.packed + (long long)N * row_bytes);
  const float betaU = FFN ? *reinterpret_cast<const float*>(a.t[1].packed + (long long)N * row_bytes) : 0.0f;
  const uint8_t* rA0 = gid < nrows ? baseA + gid * row_bytes : nullptr;
  const uint8_t* rA1 = gid + 8 < nrows ? baseA + (gid + 8) * row_bytes : nullptr;
  const uint8_t* rU0 = FFN && gid < nrows ? baseU + gid * row_bytes : nullptr;
  const uint8_t* rU1 = FFN && gid + 8 < nrows ? baseU + (gid + 8) * row_bytes : nullptr;

  for (int tok0 = 0; tok0 < a.T; tok0 += GEMV_TOK) {
    int dA[2][4], dU[2][4];
    gemv_tile_accumulate(rA0, rA1, a.q, a.T - 0, a.K, tok0, warp, gid, r, dA);
    if (FFN) gemv_tile_accumulate(rU0, rU1, a.q, a.T, a.K, tok0, warp, gid, r, dU);
    gemv_reduce_warps(dA, red[0], warp, lane);
    if (FFN) gemv_reduce_warps(dU, red[1], warp, lane);
    if (warp == 0) {
#pragma unroll
      for (int tg = 0; tg < 2; ++tg)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = gid + ((i & 2) ? 8 : 0);
          const int t = tok0 + tg * 8 + 2 * r + (i & 1);
          if (t < a.T && row < nrows) {
            const long long n = n0 + row;
            const int sq = __ldg(a.sum_q + t);
            const float sx = __ldg(a.s_x + t);
            const int accA = dA[tg][i] - sq;
            const float vA = dequant(accA, __fdiv_rn(betaA, sx));
            if (FFN) {
              const int accU = dU[tg][i] - sq;
              const float vU = dequant(accU, __fdiv_rn(betaU, sx));
              a.h[(long long)t * N + n] = ffn_act(vA, vU, a.act);
            } else {
              store_out(TA.out, a.out_dtype, (long long)t * N + n, vA);
              if (TA.acc_debug) TA.acc_debug[(long long)t * N + n] = accA;
            }
          }
        }
    }
  }
}

}  // namespace bitnet

// The decode engine: every BitLinear step of a small-token-count forward (T <= 16) in
// ONE persistent launch.  A forward is a list of phases:
//
//   GEMV      the product of one or more I2_S tensors (or the FFN's gate/up pair with
//             h = act(g) * u fused into the epilogue) with an int8 activation batch that
//             is either given (q, s_x, sum_q in global memory) or quantised by every CTA
//             itself from the raw activations (RMSNorm + absmax int8 in registers);
//   QUANT     RMSNorm + absmax int8 of a larger activation batch, tokens split over CTAs,
//             written to global memory;
//   SUBNORM   the FFN's ffn_sub_norm + absmax int8 of h, every row split over all CTAs:
//             each CTA reduces the rows it produced in the gate/up phase, with grid
//             barriers between the global max, the exact sum of squares and max |y|.
//
// A phase may arrive on a grid barrier after its epilogue (its outputs are complete
// once every CTA has arrived) and may wait on one before it reads its inputs.  Arrival
// and wait are split, so independent work (the q/k/v projections while the o output
// is being completed) fills the wait.
//
// Weights do not depend on any phase, so a producer warp streams the packed bytes of
// ALL phases of this CTA, in phase order, through a ring of shared-memory slots; it starts
// before griddepcontrol.wait, i.e. while the previous kernel on the stream is still running.
// A slot holds one tensor's weights: whole 16-row tiles fetched as one contiguous 1-D bulk
// copy (rows of up to 2 KB), or one 16-row x 2 KB 2-D TMA box of longer rows (geometry in
// engine_sched.h).  All 15 consumer warps work on every slot, taking its 64-byte steps in
// turn (one AND per 2-bit field, mma.sync m16n8k32 u8 x s8, per-field accumulators combined
// exactly once per tile and added into the tile's shared accumulator).  The steps are dealt
// to the warps round-robin, continuing from stage to stage, so the warps' loads even out.
//
// Arithmetic and sources as in quant.cuh ("Add optional RMSNorm support to BitNet
// quantization": BitNetRMSNorm before quantisation) and gemv.cuh ("fix: I2_S ARM kernel
// layout + squared-ReLU FFN": acc = sum q*c - sum q in the interleaved 128/32 layout,
// out = fp32(acc) * (beta / s_x), relu2 / SiLU chosen by the caller).
//
// Grid barriers are counters in the caller's workspace, which must be zero before the
// first launch; the last CTA to finish zeroes them again.  Every wait is bounded (about
// a second); a wait that gives up sets BITNET_ERR_TIMEOUT in the device status word.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "engine_sched.h"
#include "gemv.cuh"

namespace bitnet {

constexpr int ENG_CONS_WARPS = 15;  // + 1 producer warp: 16 warps, 4 per SM sub-partition (128 registers each)
static_assert(ENG_CONS_WARPS == ENG_SLOT_WARPS, "the stage geometry deals slots to the consumer warps");
constexpr int ENG_CONS = ENG_CONS_WARPS * 32;
constexpr int ENG_THREADS = ENG_CONS + 32;
constexpr int ENG_MAX_PHASES = 8;
constexpr int ENG_MAX_BARRIERS = 8;
constexpr int ENG_LOCAL_MAX_K = 28672;  // rows staged in shared memory as fp32 (112 KB)
constexpr int ENG_MAX_T = 16;
constexpr int ENG_MAX_SLOTS = 32;  // ring slots at most

enum { PH_GEMV = 0, PH_GEMV_FFN = 1, PH_QUANT = 2, PH_SUBNORM = 3 };
BN_HOST_DEV inline bool ph_is_gemv(int kind) { return kind == PH_GEMV || kind == PH_GEMV_FFN; }
constexpr int ENG_MAX_GRID = 256;  // CTAs at most (per-CTA partials in the workspace)
enum { SRC_GLOBAL = 0, SRC_LOCAL = 1 };

struct EngTensor {
  const uint8_t* packed;
  void* out;
  int32_t* acc_debug;
  int N;
  int tile_begin;
};

struct EngPhase {
  int kind, K, n_tensors, n_tiles;
  EngTensor t[4];
  int src;            // GEMV: SRC_GLOBAL (q/s/sq given) or SRC_LOCAL (quantise x in every CTA)
  const void* x;      // raw activations [T, K] (SRC_LOCAL, QUANT)
  int x_f32;          // 1: fp32, 0: bf16
  const float* gain;  // RMSNorm gain, nullptr = no norm
  int8_t* q;          // int8 activations [T, K]: read (SRC_GLOBAL), written (QUANT, and by CTA 0 for SRC_LOCAL)
  float* s;
  int32_t* sq;
  int out_dtype, act;
  float* h;           // FFN output [T, N] fp32
  int wait_barrier, arrive_barrier;  // -1: none
  // SUBNORM (and the GEMV_FFN phase before it): per-CTA partials of max |h| (pmax [T][G]),
  // of the fixed-point sum of h^2 on ENG_SUB_CAND candidate grids (psum [T][G][ENG_SUB_CAND]),
  // of the sum on the global grid when the candidates do not cover it (psum_fb [T][G]) and of
  // max |y| (pmax2 [T][G]); the SUBNORM phase's inner grid barriers; the sub-norm gain, which
  // the gate/up phase prefetches for its rows (sub_gain).
  float* pmax;
  long long* psum;
  long long* psum_fb;
  float* pmax2;
  float2* pyc;  // per CTA and token: the (h, g) pair that may hold max |y| [T][G]
  int* pycnt;   // the count of such pairs [T][G] (2: more than one)
  const float* sub_gain;
  int bar_a, bar_b, bar_fb;
  // Tile split over the grid: CTA c owns tiles [start(c), start(c + 1)); by default
  // start(c) = floor(c n_tiles / G).  Balanced split (balanced = 1): every CTA gets
  // floor(n_tiles / G) tiles plus one where bit c of xmask is set, so that the host can
  // spread the remainders of consecutive phases over different CTAs.
  int balanced;
  uint32_t xmask[ENG_MAX_GRID / 32];
  EngGeom g;  // stage geometry of a product phase (engine_sched.h)
};

// One tensor map per tensor and phase (chunked mode): the packed rows viewed as
// [N, K/32] 8-byte elements, box CB/8 x 16.
struct alignas(64) EngMaps {
  CUtensorMap m[ENG_MAX_PHASES][4];
};

struct alignas(16) EngArgs {
  int T;
  float eps;
  int n_phases;
  unsigned* counters;  // ENG_MAX_BARRIERS + 1 words in the workspace (last: exit count)
  int n_slots, slot_bytes, acc_ints, qs_bytes, xs_floats;
  int sub_rows;  // rows of h a CTA keeps for the SUBNORM phase (0: none)
  int acc_priv;  // 1: every consumer warp has its own accumulator slots (small T)
  int pad_[2];
  EngPhase ph[ENG_MAX_PHASES];
};

// ------------------------------------------------------------------ consumer-group helpers
BN_DEV void cons_sync() { named_sync(1, ENG_CONS); }

// Reductions over the 256 consumer threads.  The scratch has two halves used in turn, so
// one named barrier per reduction suffices: a thread can only overwrite a half after every
// thread has passed the barrier of the reduction in between, i.e. has read that half.
struct ConsRed {
  long long* buf;  // [2][ENG_CONS_WARPS]
  int flip;
  BN_DEV long long* next() {
    long long* b = buf + flip * ENG_CONS_WARPS;
    flip ^= 1;
    return b;
  }
};

// max over non-negative floats (their bit patterns order like unsigned integers)
BN_DEV float cons_max_nonneg(float v, ConsRed& r) {
  unsigned u = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
  unsigned* b = reinterpret_cast<unsigned*>(r.next());
  if ((threadIdx.x & 31) == 0) b[threadIdx.x >> 5] = u;
  cons_sync();
  unsigned m = 0;
#pragma unroll
  for (int i = 0; i < ENG_CONS_WARPS; ++i) m = max(m, b[i]);
  return __uint_as_float(m);
}

BN_DEV int cons_sum_i32(int v, ConsRed& r) {
  int w = __reduce_add_sync(0xffffffffu, v);
  int* b = reinterpret_cast<int*>(r.next());
  if ((threadIdx.x & 31) == 0) b[threadIdx.x >> 5] = w;
  cons_sync();
  int t = 0;
#pragma unroll
  for (int i = 0; i < ENG_CONS_WARPS; ++i) t += b[i];
  return t;
}

BN_DEV long long cons_sum_i64(long long v, ConsRed& r) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  long long* b = r.next();
  if ((threadIdx.x & 31) == 0) b[threadIdx.x >> 5] = v;
  cons_sync();
  long long t = 0;
#pragma unroll
  for (int w = 0; w < ENG_CONS_WARPS; ++w) t += b[w];
  return t;
}

// Load 8 activations (bf16 or fp32) at element offset k of row x, bypassing L1 (the row
// may have been written by other CTAs earlier in this launch).
BN_DEV void load8(const void* x, int x_f32, long long k, float* o) {
  if (x_f32) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + k));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + k + 4));
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  } else {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + k));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Activation layout in shared memory.  A consumer lane r (of the four lanes that share a
// weight row in an m16n8k32 fragment) multiplies, for weight field g of 64-byte step s, the
// 16 activations k = 256 s + 128 (r >> 1) + 32 g + 16 (r & 1) + j, j < 16.  Storing those 16
// bytes at 256 s + 64 g + 16 r puts the four lanes' pieces of one field side by side, so a
// 16-byte load by every lane is served without bank conflicts.  Token rows are
// round_up(K, 256) + 64 bytes apart (also conflict-free for consecutive tokens).
BN_DEV int eng_perm(int k) {  // k a multiple of 8
  const int o = k & 255;
  return (k & ~255) + 64 * ((o >> 5) & 3) + 32 * (o >> 7) + 16 * ((o >> 4) & 1) + (o & 15);
}
BN_DEV int eng_x_pitch(int K) { return ((K + 255) & ~255) + 64; }

// RMSNorm + absmax int8 of one row of K <= ENG_REG_MAX_K values by the 256 consumer threads,
// values in registers (thread i owns elements 8(i + 256 j) .. +7, j < 4).  The activation
// and gain loads are issued together, so the row costs one memory round trip.  Writes q
// (into `qdst`, shared or global memory), s_x and sum_q (thread 0).  The same operation
// sequence as quant.cuh: exact fixed-point sum of x^2 (x^2 and its scaling by 2^e are exact
// in fp64), fp32 steps without contraction.
constexpr int ENG_REG_GROUPS = 3;
constexpr int ENG_REG_MAX_K = 8192;
static_assert(ENG_CONS * 8 * ENG_REG_GROUPS >= ENG_REG_MAX_K, "register quantiser covers the row");

__device__ __noinline__ void quant_row_regs(const void* xrow, int x_f32, int K, const float* gain, float eps,
                                            int8_t* qdst, bool perm, float* s_dst, int32_t* sq_dst, long long* red) {
  const int tid = threadIdx.x;
  ConsRed R{red, 0};
  float v[ENG_REG_GROUPS][8], g[ENG_REG_GROUPS][8];
#pragma unroll
  for (int j = 0; j < ENG_REG_GROUPS; ++j) {
    const int k = 8 * (tid + ENG_CONS * j);
    if (k < K) {
      load8(xrow, x_f32, k, v[j]);
      if (gain != nullptr) {
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(gain + k));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(gain + k + 4));
        g[j][0] = g0.x; g[j][1] = g0.y; g[j][2] = g0.z; g[j][3] = g0.w;
        g[j][4] = g1.x; g[j][5] = g1.y; g[j][6] = g1.z; g[j][7] = g1.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
    }
  }
  float am = 0.0f;
#pragma unroll
  for (int j = 0; j < ENG_REG_GROUPS; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[j][i]));
  am = cons_max_nonneg(am, R);
  float a = am;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (am > 0.0f) {
      const int e = fixed_point_exponent(__dmul_rn((double)am, (double)am), K);
      const double p2e = pow2_f64(e);
      long long part = 0;
      if (K >= kFixedSmallMinN) {
#pragma unroll
        for (int j = 0; j < ENG_REG_GROUPS; ++j) {
          if (8 * (tid + ENG_CONS * j) < K) {
#pragma unroll
            for (int i = 0; i < 8; ++i) part += fixed_sq_term_t<true>(v[j][i], p2e);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < ENG_REG_GROUPS; ++j) {
          if (8 * (tid + ENG_CONS * j) < K) {
#pragma unroll
            for (int i = 0; i < 8; ++i) part += fixed_sq_term(v[j][i], p2e);
          }
        }
      }
      ms = fixed_point_mean(cons_sum_i64(part, R), e, K);
    }
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float ay = 0.0f;
#pragma unroll
    for (int j = 0; j < ENG_REG_GROUPS; ++j) {
      if (8 * (tid + ENG_CONS * j) < K) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[j][i] = __fmul_rn(__fmul_rn(v[j][i], inv), g[j][i]);
          ay = fmaxf(ay, fabsf(v[j][i]));
        }
      }
    }
    a = cons_max_nonneg(ay, R);
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
#pragma unroll
  for (int j = 0; j < ENG_REG_GROUPS; ++j) {
    const int k = 8 * (tid + ENG_CONS * j);
    if (k < K) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qv = quant_code(__fmul_rn(v[j][i], s));
        sum += qv;
        w[i >> 2] |= (uint32_t)(qv & 0xFF) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2*>(qdst + (perm ? eng_perm(k) : k)) = make_uint2(w[0], w[1]);
    }
  }
  sum = cons_sum_i32(sum, R);
  if (tid == 0) {
    *s_dst = s;
    *sq_dst = sum;
  }
}

// The same for rows longer than ENG_REG_MAX_K: the row is staged once in shared memory as
// fp32 (`xs`, K floats) and each pass is a compact rolled loop.
__device__ __noinline__ void quant_row_staged(const void* xrow, int x_f32, int K, const float* gain, float eps,
                                              int8_t* qdst, bool perm, float* s_dst, int32_t* sq_dst, long long* red,
                                              float* xs) {
  const int tid = threadIdx.x;
  ConsRed R{red, 0};
  float am = 0.0f;
  int k = 8 * tid;
  for (; k + 3 * 8 * ENG_CONS < K; k += 4 * 8 * ENG_CONS) {  // four loads in flight per thread
    float v[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) load8(xrow, x_f32, k + j * 8 * ENG_CONS, v[j]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      *reinterpret_cast<float4*>(xs + k + j * 8 * ENG_CONS) = make_float4(v[j][0], v[j][1], v[j][2], v[j][3]);
      *reinterpret_cast<float4*>(xs + k + j * 8 * ENG_CONS + 4) = make_float4(v[j][4], v[j][5], v[j][6], v[j][7]);
#pragma unroll
      for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[j][i]));
    }
  }
  for (; k < K; k += 8 * ENG_CONS) {
    float v[8];
    load8(xrow, x_f32, k, v);
    *reinterpret_cast<float4*>(xs + k) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(xs + k + 4) = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
  }
  am = cons_max_nonneg(am, R);  // its barrier also orders the xs writes
  float a = am;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (am > 0.0f) {
      const int e = fixed_point_exponent(__dmul_rn((double)am, (double)am), K);
      const double p2e = pow2_f64(e);
      long long part = 0;
      if (K >= kFixedSmallMinN)
        for (int kk = tid; kk < K; kk += ENG_CONS) part += fixed_sq_term_t<true>(xs[kk], p2e);
      else
        for (int kk = tid; kk < K; kk += ENG_CONS) part += fixed_sq_term(xs[kk], p2e);
      ms = fixed_point_mean(cons_sum_i64(part, R), e, K);
    }
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float ay = 0.0f;
    for (int kk = tid; kk < K; kk += ENG_CONS) {
      const float y = __fmul_rn(__fmul_rn(xs[kk], inv), __ldg(gain + kk));
      xs[kk] = y;
      ay = fmaxf(ay, fabsf(y));
    }
    a = cons_max_nonneg(ay, R);  // also orders the xs rewrites
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
  for (int kk = 8 * tid; kk < K; kk += 8 * ENG_CONS) {
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int qv = quant_code(__fmul_rn(xs[kk + i], s));
      sum += qv;
      w[i >> 2] |= (uint32_t)(qv & 0xFF) << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(qdst + (perm ? eng_perm(kk) : kk)) = make_uint2(w[0], w[1]);
  }
  sum = cons_sum_i32(sum, R);
  if (tid == 0) {
    *s_dst = s;
    *sq_dst = sum;
  }
}

// `perm`: write q in the shared-memory layout of eng_perm (else plain order).
BN_DEV void quant_row(const void* xrow, int x_f32, int K, const float* gain, float eps, int8_t* qdst, bool perm,
                      float* s_dst, int32_t* sq_dst, long long* red, float* xs) {
  if (K <= ENG_REG_MAX_K)
    quant_row_regs(xrow, x_f32, K, gain, eps, qdst, perm, s_dst, sq_dst, red);
  else
    quant_row_staged(xrow, x_f32, K, gain, eps, qdst, perm, s_dst, sq_dst, red, xs);
}

// ------------------------------------------------------------------ grid barriers
// Arrival is a release add at GPU scope by one thread after the CTA barrier: the barrier
// orders the other consumer threads' writes before it, and release is cumulative, so a CTA
// whose acquire load sees the count also sees those writes (no separate full fence).
BN_DEV void grid_arrive(unsigned* ctr) {
  cons_sync();  // every consumer thread of this CTA has written its outputs
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

BN_DEV bool grid_wait(unsigned* ctr, unsigned target) {
  bool ok = true;
  if (threadIdx.x == 0) {
    long long t0 = -1;
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= target) break;
      const long long now = clock64();
      if (t0 < 0) t0 = now;
      if (now - t0 > c_wait_limit) {
        atomicExch(&g_device_status, (int)BITNET_ERR_TIMEOUT);
        ok = false;
        break;
      }
    }
    // the acquire load that saw the count orders this thread's later reads; the named
    // barrier that follows every wait passes that on to the other consumer threads
  }
  return ok;
}

// ------------------------------------------------------------------ distributed sub-norm
// Per-token scratch of the SUBNORM phase in shared memory.
constexpr int ENG_SUB_CAND = 8;  // candidate grids per CTA: local exponent e_c, e_c - 1, .., e_c - 7
static_assert(ENG_SUB_CAND == 8, "the candidate sums are reduced by a three-level lane split");
struct SubScratch {
  unsigned long long pmx[ENG_MAX_T];  // this CTA's max |h g| (exact, fp64 bits; non-negative)
  float2 yc[ENG_MAX_T];               // an (h, g) pair within 2^-20 of it
  int ycnt[ENG_MAX_T];                // and how many there are
  int yfb;                            // some CTA had more than one candidate: the barrier path
  unsigned mx[ENG_MAX_T];  // max |h|: this CTA's, then the row's (non-negative floats as bits)
  unsigned my[ENG_MAX_T];  // max |y|
  unsigned long long sum[ENG_MAX_T];
  unsigned long long cand[ENG_MAX_T][ENG_SUB_CAND];  // this CTA's sums on its candidate grids
  int e[ENG_MAX_T];        // the grid exponent: this CTA's, then the row's
  int fallback;
  float inv[ENG_MAX_T];
  float scale[ENG_MAX_T];
  int sq[ENG_MAX_T];
};

// Grid barrier between two steps of a phase: arrive, wait for every CTA, and agree on the
// outcome (false: a wait gave up).
BN_DEV bool grid_step(unsigned* ctr) {
  grid_arrive(ctr);
  const bool ok = grid_wait(ctr, gridDim.x);
  return !named_sync_or(1, ENG_CONS, !ok);
}

// ffn_sub_norm + absmax int8 of h [T, K] (fp32) into p.q / p.s / p.sq, every row split over
// the grid: this CTA owns the rows of the 16-row tiles [tb, te) it produced in the gate/up
// phase, whose epilogue kept them in shared memory (hs [T][sub_rows]) and which prefetched the
// matching gain slice (gs).  The same arithmetic as quant_row, with each reduction finished
// across the grid:
//   1. the CTA's max |h| M_c and its fixed-point sums of h^2 on the grids of the exponents
//      e_c, e_c - 1, .., e_c - 7 (e_c from M_c and the row length) -> published; grid barrier;
//   2. the global max M gives the row's grid e <= e_c; when every CTA's candidates include
//      e (or M_c = 0, whose sum is 0 on any grid) the sum is the sum of those candidates,
//      else (uniformly, from the same published maxima) every CTA sums on e itself and a
//      second barrier publishes those sums;
//   3. inv, and max |y| from the (h, g) candidate each CTA published with its sums; when
//      some CTA had more than one candidate (or after the sum fallback), max |y| of every
//      CTA's rows -> published; grid barrier; 4. s_x and q of its rows.
// Maxima and integer sums are order-free, so the result does not depend on the split.
// p.sq must be zero on entry (the kernel clears it before the gate/up phase).
__device__ __noinline__ bool eng_subnorm(const EngPhase& p, int T, float eps, int tb, int te, unsigned* counters,
                                         SubScratch& S, const float* hs, const float* gs, int sub_rows) {
  const int G = gridDim.x, K = p.K, tid = threadIdx.x, nrows = (te - tb) * GEMV_ROWS;
  const int warp = tid >> 5, lane = tid & 31;
  // Work items: (token, 32 consecutive rows), dealt to the consumer warps in turn; each warp
  // reduces its item with shuffles and adds the result into the token's shared entry.
  const int chunks = (nrows + 31) >> 5, items = T * chunks;
  cp_async_wait_all();  // this thread's part of the gain slice
  if (tid < T) {
    S.mx[tid] = S.my[tid] = 0u;
    S.sum[tid] = 0ull;
    S.pmx[tid] = 0ull;
    S.ycnt[tid] = 0;
#pragma unroll
    for (int d = 0; d < ENG_SUB_CAND; ++d) S.cand[tid][d] = 0ull;
  }
  if (tid == 0) S.fallback = S.yfb = 0;
  cons_sync();
  // 1. this CTA's max |h| and max |h g| (exact in fp64), then its sums on the candidate grids
  // e_c - d, and the (h, g) pair whose |h g| is within 2^-20 of the CTA's maximum (with the
  // count of such pairs).  max |y| over the row is taken at one of those: y = fl(fl(h inv) g)
  // is |h g| inv within a relative 2^-23 (for the y that can set the scale: |y| >= 1e-5 and
  // gains far below 2^100), so an element whose |h g| is below the row's maximum by more than
  // 2^-22 cannot hold it, and the row's argmax lies within 2^-22 of its own CTA's maximum.
  for (int it = warp; it < items; it += ENG_CONS_WARPS) {
    const int t = it / chunks, r = (it - t * chunks) * 32 + lane;
    const float hv = r < nrows ? hs[t * sub_rows + r] : 0.0f;
    const float m = warp_max(fabsf(hv));
    if (lane == 0) atomicMax(&S.mx[t], __float_as_uint(m));
    if (p.gain != nullptr) {
      const double pr = r < nrows ? fabs(__dmul_rn((double)hv, (double)gs[r])) : 0.0;
      unsigned long long pb = (unsigned long long)__double_as_longlong(pr);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) pb = max(pb, __shfl_xor_sync(0xffffffffu, pb, o));
      if (lane == 0) atomicMax(&S.pmx[t], pb);
    }
  }
  cons_sync();
  if (tid < T) {
    const float am = __uint_as_float(S.mx[tid]);
    S.e[tid] = am > 0.0f ? fixed_point_exponent(__dmul_rn((double)am, (double)am), K) : 0;
  }
  cons_sync();
  if (p.gain != nullptr) {
    for (int it = warp; it < items; it += ENG_CONS_WARPS) {
      const int t = it / chunks, r = (it - t * chunks) * 32 + lane;
      if (S.mx[t] == 0u) continue;
      const float v = r < nrows ? hs[t * sub_rows + r] : 0.0f;
      // the max |y| candidate of this row
      const double pc = __longlong_as_double((long long)S.pmx[t]);
      if (pc > 0.0 && r < nrows) {
        const float gv = gs[r];
        if (fabs(__dmul_rn((double)v, (double)gv)) >= __dsub_rn(pc, __dmul_rn(pc, 0x1p-20))) {
          if (atomicAdd(&S.ycnt[t], 1) == 0) S.yc[t] = make_float2(v, gv);
        }
      }
      const double d2 = __dmul_rn((double)v, (double)v);
      double p2e = pow2_f64(S.e[t]);
      long long c[ENG_SUB_CAND];
#pragma unroll
      for (int d = 0; d < ENG_SUB_CAND; ++d) {
        const double x2 = __dmul_rn(d2, p2e);
        c[d] = K >= kFixedSmallMinN ? rint_i64_small(x2) : __double2ll_rn(x2);
        p2e = __dmul_rn(p2e, 0.5);  // the next candidate grid: e - d - 1 (exact)
      }
      // The 8 warp sums at once (reduce-scatter): at each of the first three steps a lane keeps
      // the half of its values selected by one lane bit and adds its partner's copy of that
      // half; lane l then holds candidate (l >> 2) & 7 summed over 8 lanes, and two more steps
      // finish the sums (9 exchanges instead of 40).
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool hi = lane & 16;
        const long long send = hi ? c[i] : c[i + 4], keep = hi ? c[i + 4] : c[i];
        c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const bool hi = lane & 8;
        const long long send = hi ? c[i] : c[i + 2], keep = hi ? c[i + 2] : c[i];
        c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
      {
        const bool hi = lane & 4;
        const long long send = hi ? c[0] : c[1], keep = hi ? c[1] : c[0];
        c[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      c[0] += __shfl_xor_sync(0xffffffffu, c[0], 2);
      c[0] += __shfl_xor_sync(0xffffffffu, c[0], 1);
      if ((lane & 3) == 0) atomicAdd(&S.cand[t][(lane >> 2) & 7], (unsigned long long)c[0]);
    }
    cons_sync();
    if (tid < T * ENG_SUB_CAND)
      p.psum[((long long)(tid / ENG_SUB_CAND) * G + blockIdx.x) * ENG_SUB_CAND + tid % ENG_SUB_CAND] =
          (long long)S.cand[tid / ENG_SUB_CAND][tid % ENG_SUB_CAND];
    if (tid < T) {
      p.pyc[tid * G + blockIdx.x] = S.yc[tid];
      p.pycnt[tid * G + blockIdx.x] = min(S.ycnt[tid], 2);
    }
  }
  if (tid < T) p.pmax[tid * G + blockIdx.x] = __uint_as_float(S.mx[tid]);
  if (!grid_step(counters + p.bar_a)) return false;
  // 2. + 3. A warp per token loads every CTA's published max |h|, candidate count and (h, g)
  // pair at once (one round trip), reduces the max with shuffles, then loads the matching
  // candidate sums (a second round trip): the row's exact sum of squares, inv, and max |y| from
  // the candidates -- the same values in every CTA.  Two uniform exceptions take the barrier
  // path: a CTA whose candidate grids miss the row's grid (the sum is taken again on the row's
  // grid), or one with more than one max |y| candidate (max |y| over every CTA's rows).
  constexpr int GPL = ENG_MAX_GRID / 32;  // published values per lane at most
  for (int t = warp; t < T; t += ENG_CONS_WARPS) {
    float pm[GPL];
    int cn[GPL];
    float2 hg[GPL];
#pragma unroll
    for (int j = 0; j < GPL; ++j) {
      const int c = lane + 32 * j;
      const bool in = c < G;
      pm[j] = in ? __ldcg(p.pmax + t * G + c) : 0.0f;
      cn[j] = (in && p.gain != nullptr) ? __ldcg(p.pycnt + t * G + c) : 0;
      hg[j] = (in && p.gain != nullptr) ? __ldcg(p.pyc + t * G + c) : make_float2(0.0f, 0.0f);
    }
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < GPL; ++j) m = fmaxf(m, pm[j]);
    m = warp_max(m);
    const int e = m > 0.0f ? fixed_point_exponent(__dmul_rn((double)m, (double)m), K) : 0;
    if (p.gain != nullptr) {
      long long v[GPL];
      int fb = 0, over = 0;
#pragma unroll
      for (int j = 0; j < GPL; ++j) {
        v[j] = 0;
        if (cn[j] > 1) over = 1;
        if (pm[j] > 0.0f) {
          const int d = fixed_point_exponent(__dmul_rn((double)pm[j], (double)pm[j]), K) - e;
          if (d >= ENG_SUB_CAND)
            fb = 1;
          else
            v[j] = __ldcg(p.psum + ((long long)t * G + lane + 32 * j) * ENG_SUB_CAND + d);
        }
      }
      long long sum = 0;
#pragma unroll
      for (int j = 0; j < GPL; ++j) sum += v[j];
      sum = warp_sum_ll(sum);
      fb = __any_sync(0xffffffffu, fb);
      over = __any_sync(0xffffffffu, over);
      float ymax = 0.0f, inv = 0.0f;
      if (!fb && !over) {
        const float ms = m > 0.0f ? fixed_point_mean(sum, e, K) : 0.0f;
        inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
#pragma unroll
        for (int j = 0; j < GPL; ++j)
          if (cn[j] == 1) ymax = fmaxf(ymax, fabsf(__fmul_rn(__fmul_rn(hg[j].x, inv), hg[j].y)));
        ymax = warp_max(ymax);
      }
      if (lane == 0) {
        S.sum[t] = (unsigned long long)sum;
        if (fb) S.fallback = 1;
        if (over) S.yfb = 1;
        S.inv[t] = inv;
        S.my[t] = __float_as_uint(ymax);
      }
    }
    if (lane == 0) {
      S.mx[t] = __float_as_uint(m);
      S.e[t] = e;
    }
  }
  cons_sync();
  if (p.gain != nullptr) {
    if (S.fallback) {  // the same decision in every CTA (it follows from the published maxima)
      if (tid < T) S.cand[tid][0] = 0ull;
      cons_sync();
      for (int it = warp; it < items; it += ENG_CONS_WARPS) {
        const int t = it / chunks, r = (it - t * chunks) * 32 + lane;
        if (S.mx[t] == 0u) continue;
        const long long c = warp_sum_ll(r < nrows ? fixed_sq_term(hs[t * sub_rows + r], pow2_f64(S.e[t])) : 0ll);
        if (lane == 0) atomicAdd(&S.cand[t][0], (unsigned long long)c);
      }
      cons_sync();
      if (tid < T) p.psum_fb[tid * G + blockIdx.x] = (long long)S.cand[tid][0];
      if (!grid_step(counters + p.bar_fb)) return false;
      for (int t = warp; t < T; t += ENG_CONS_WARPS) {
        long long sum = 0;
        for (int c = lane; c < G; c += 32) sum += __ldcg(p.psum_fb + t * G + c);
        sum = warp_sum_ll(sum);
        if (lane == 0) S.sum[t] = (unsigned long long)sum;
      }
      cons_sync();
    }
    if (S.fallback || S.yfb) {  // uniform: max |y| over this CTA's rows and a grid barrier
      if (tid < T) {
        const float am = __uint_as_float(S.mx[tid]);
        const float ms = am > 0.0f ? fixed_point_mean((long long)S.sum[tid], S.e[tid], K) : 0.0f;
        S.inv[tid] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
        S.my[tid] = 0u;
      }
      cons_sync();
      for (int it = warp; it < items; it += ENG_CONS_WARPS) {
        const int t = it / chunks, r = (it - t * chunks) * 32 + lane;
        const float y = r < nrows ? fabsf(__fmul_rn(__fmul_rn(hs[t * sub_rows + r], S.inv[t]), gs[r])) : 0.0f;
        const float mm = warp_max(y);
        if (lane == 0) atomicMax(&S.my[t], __float_as_uint(mm));
      }
      cons_sync();
      if (tid < T) p.pmax2[tid * G + blockIdx.x] = __uint_as_float(S.my[tid]);
      if (!grid_step(counters + p.bar_b)) return false;
      for (int t = warp; t < T; t += ENG_CONS_WARPS) {
        float pm[GPL];
#pragma unroll
        for (int j = 0; j < GPL; ++j) {
          const int c = lane + 32 * j;
          pm[j] = c < G ? __ldcg(p.pmax2 + t * G + c) : 0.0f;
        }
        float mm = 0.0f;
#pragma unroll
        for (int j = 0; j < GPL; ++j) mm = fmaxf(mm, pm[j]);
        mm = warp_max(mm);
        if (lane == 0) S.my[t] = __float_as_uint(mm);
      }
      cons_sync();
    }
  } else {
    if (tid < T) {
      S.my[tid] = S.mx[tid];  // y = h
      S.inv[tid] = 1.0f;
    }
    cons_sync();
  }
  if (tid < T) {
    S.scale[tid] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(S.my[tid]), 1e-5f));
    S.sq[tid] = 0;
  }
  cons_sync();
  // 4. q of this CTA's rows: items of (token, 128 rows), four rows per lane
  const int qchunks = (nrows + 127) >> 7;
  for (int it = warp; it < T * qchunks; it += ENG_CONS_WARPS) {
    const int t = it / qchunks, r = (it - t * qchunks) * 128 + 4 * lane;
    int sum = 0;
    if (r < nrows) {
      const float inv = S.inv[t], sc = S.scale[t];
      uint32_t w = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float y = hs[t * sub_rows + r + k];
        if (p.gain != nullptr) y = __fmul_rn(__fmul_rn(y, inv), gs[r + k]);
        int qv = quant_code(__fmul_rn(y, sc));
        sum += qv;
        w |= (uint32_t)(qv & 0xFF) << (8 * k);
      }
      *reinterpret_cast<uint32_t*>(p.q + (long long)t * K + tb * GEMV_ROWS + r) = w;
    }
    sum = warp_sum_i(sum);
    if (lane == 0) atomicAdd(&S.sq[t], sum);
  }
  cons_sync();
  if (tid < T) {
    atomicAdd(p.sq + tid, S.sq[tid]);
    if (blockIdx.x == 0) p.s[tid] = S.scale[tid];
  }
  return true;
}

// ------------------------------------------------------------------ products of one stage
// Partial sums of one tile of one tensor, per 2-bit field: f[tg][g][i] is the mma
// accumulator of token group tg (tokens 8 tg + ..) and field g (codes scaled by 4^(3-g)).
template <int TG>
struct EngAcc {
  int f[TG][4][4];
  BN_DEV void zero() {
#pragma unroll
    for (int tg = 0; tg < TG; ++tg)
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int i = 0; i < 4; ++i) f[tg][g][i] = 0;
  }
  // Combine the fields exactly (field g's sums are multiples of 4^(3-g)) and add this warp's
  // share into the tile's shared accumulator at[row * T + tok] -- with an atomic add into the
  // slot all warps share, or (priv) a plain add into this warp's own slot, which the
  // epilogue sums (no contention of 15 warps on the same words); then restart.
  BN_DEV void flush(int* at, int T, int gid, int r, bool priv) {
#pragma unroll
    for (int tg = 0; tg < TG; ++tg)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = tg * 8 + 2 * r + (i & 1);
        if (tok < T) {
          const int v = (f[tg][0][i] >> 6) + (f[tg][1][i] >> 4) + (f[tg][2][i] >> 2) + f[tg][3][i];
          int* dst = at + (gid + ((i & 2) ? 8 : 0)) * T + tok;
          if (priv)
            *dst += v;
          else
            atomicAdd(dst, v);
        }
      }
    zero();
  }
  // The same for one token (T = 1): lanes with r == 0 hold token 0 of rows gid (i = 0) and
  // gid + 8 (i = 2).
  BN_DEV void flush1(int* at, int gid, int r, bool priv) {
    if (r == 0) {
      const int v0 = (f[0][0][0] >> 6) + (f[0][1][0] >> 4) + (f[0][2][0] >> 2) + f[0][3][0];
      const int v2 = (f[0][0][2] >> 6) + (f[0][1][2] >> 4) + (f[0][2][2] >> 2) + f[0][3][2];
      if (priv) {
        at[gid] += v0;
        at[gid + 8] += v2;
      } else {
        atomicAdd(at + gid, v0);
        atomicAdd(at + gid + 8, v2);
      }
    }
    zero();
  }
};

// This warp's 64-byte steps of one 16-row tile in a stage: steps t = t0, t0 + stride, .. < S.
// Lane (gid, r) holds rows gid and gid + 8 of the tile, bytes 16 r .. 16 r + 15 of each step
// (the A fragments of mma.sync m16n8k32, one AND per 2-bit field), and the activations of
// tokens gid (and 8 + gid) -- token T - 1 where those do not exist; those lanes only feed
// accumulator columns that are never used.  wrow: shared address of row gid's step 0 at
// byte 16 r; P: row pitch; xa / xb: shared address of the tokens' step 0 (+ 16 r).
template <int TG>
BN_DEV void eng_tile_steps(EngAcc<TG>& A, uint32_t wrow, int P, uint32_t xa_s, uint32_t xb_s, int t0, int S,
                           int stride) {
  for (int t = t0; t < S; t += stride) {
    const uint4 wa = lds128(wrow + 64 * t), wb = lds128(wrow + 8 * P + 64 * t);
    const uint32_t xo = 256u * t;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t m = 0x03030303u << (6 - 2 * g);
      const uint32_t a0 = wa.x & m, a1 = wb.x & m, a2 = wa.y & m, a3 = wb.y & m;
      const uint32_t a4 = wa.z & m, a5 = wb.z & m, a6 = wa.w & m, a7 = wb.w & m;
      const uint4 x0 = lds128(xa_s + xo + 64 * g);
      mma_u8s8(A.f[0][g], a0, a1, a2, a3, x0.x, x0.y);
      mma_u8s8(A.f[0][g], a4, a5, a6, a7, x0.z, x0.w);
      if (TG > 1) {
        const uint4 x1 = lds128(xb_s + xo + 64 * g);
        mma_u8s8(A.f[TG - 1][g], a0, a1, a2, a3, x1.x, x1.y);
        mma_u8s8(A.f[TG - 1][g], a4, a5, a6, a7, x1.z, x1.w);
      }
    }
  }
}

// The stages of one activation chunk range [wc0, wc1) of a product phase whose stages hold one
// 16-row tile of one tensor each (rs = 1): for every (tile, tensor) in order, its chunks; the
// warp's steps of the chunk are t0, t0 + 15, .. (t0 rotating from stage to stage); after the
// tile's last chunk the flush into `at`, which then advances by at_step.  A flat loop with the
// chunk width CBC fixed at compile time where it is known (0: run-time CBr), and the one-token
// flush for T1: the general loop nest ran about a quarter slower per stage.
template <int TG, int CBC, bool T1>
BN_DEV void eng_flat_stages(EngAcc<TG>& A, int n_tu, int wc0, int wc1, int n_chunks, int CBr, int RB, uint32_t ring_s,
                            int slot_bytes, int n_slots, uint32_t full0, uint32_t empty0, uint32_t xa0, uint32_t xb0,
                            int* at, int at_step, int T, bool priv, int warp, int gid, int r, int lane, int& slot,
                            uint32_t& par, int& rot, bool& ok) {
  const int CB = CBC ? CBC : CBr;
  const int S_full = (CB + 63) >> 6, S_last = (RB - (n_chunks - 1) * CB + 63) >> 6;
  const uint32_t row_off = gid * CB + 16 * r;
  for (int i = 0; i < n_tu; ++i) {
    for (int wc = wc0; wc < wc1; ++wc) {
      if (ok && !mbar_wait_bounded(full0 + 8u * slot, par)) ok = false;
      if (ok) {
        const int S = wc < n_chunks - 1 ? S_full : S_last;
        const uint32_t xoff = 256u * (uint32_t)((wc - wc0) * (CB >> 6));
        int t0 = warp - rot;
        if (t0 < 0) t0 += ENG_CONS_WARPS;
        eng_tile_steps<TG>(A, ring_s + slot * slot_bytes + row_off, CB, xa0 + xoff, xb0 + xoff, t0, S, ENG_CONS_WARPS);
        if (wc == wc1 - 1) {
          if (T1)
            A.flush1(at, gid, r, priv);
          else
            A.flush(at, T, gid, r, priv);
        }
        rot += S;
        while (rot >= ENG_CONS_WARPS) rot -= ENG_CONS_WARPS;
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * slot);
      }
      if (++slot == n_slots) {
        slot = 0;
        par ^= 1u;
      }
    }
    at += at_step;
  }
}

// Stage activations [k0, k1) of all T tokens from global memory (plain int8 [T, K]) into
// shared memory in the eng_perm layout, zero-padded to whole 256-in-feature steps.  The
// rows were written by this launch's QUANT / SUBNORM phase or by the previous kernel: read
// past L1.  Four 16-byte loads in flight per thread.
BN_DEV void eng_stage_acts(const int8_t* q, int K, int T, int k0, int k1, int8_t* qs, int x_pitch) {
  const int n16 = (k1 - k0) >> 4, padded = ((k1 - k0 + 255) & ~255) >> 4;
  const int total = T * padded;
  for (int base = threadIdx.x; base < total; base += 4 * ENG_CONS) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = base + j * ENG_CONS;
      v[j] = make_uint4(0u, 0u, 0u, 0u);
      if (i < total) {
        const int t = i / padded, u = i - t * padded;
        if (u < n16) v[j] = __ldcg(reinterpret_cast<const uint4*>(q + (long long)t * K + k0 + 16 * u));
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = base + j * ENG_CONS;
      if (i < total) {
        const int t = i / padded, u = i - t * padded;
        *reinterpret_cast<uint4*>(qs + t * x_pitch + eng_perm(16 * u)) = v[j];
      }
    }
  }
}

// ------------------------------------------------------------------ the kernel
template <int TG>
__global__ void __launch_bounds__(ENG_THREADS, 1) k_engine(const __grid_constant__ EngArgs args,
                                                            const __grid_constant__ EngMaps maps) {
  extern __shared__ __align__(128) uint8_t smem[];
  // The phase descriptors are read many times with run-time indices; reading them from the
  // kernel-parameter space costs a constant-cache miss (a memory round trip) on every first
  // touch of a line, so they are copied to shared memory once, with 16-byte loads.
  __shared__ EngArgs s_args;
  {
    const uint4* src = reinterpret_cast<const uint4*>(&args);
    uint4* dst = reinterpret_cast<uint4*>(&s_args);
    for (int i = threadIdx.x; i < (int)(sizeof(EngArgs) / 16); i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  const EngArgs& a = s_args;
  volatile __shared__ int s_abort;
  __shared__ __align__(16) long long s_red[2 * ENG_CONS_WARPS];
  __shared__ float s_loc_s[ENG_MAX_T];
  __shared__ int32_t s_loc_sq[ENG_MAX_T];
  __shared__ float s_beta[ENG_MAX_PHASES][4];
  __shared__ SubScratch s_sub;
  __shared__ int s_issued;                // stages the producer issued (for the drain on exit)

  // TMA boxes land 1024-byte aligned.
  uint8_t* ring = smem + ((1024u - (smem_addr(smem) & 1023u)) & 1023u);
  const uint32_t bar0 = smem_addr(ring + a.n_slots * a.slot_bytes);
  int* acc = reinterpret_cast<int*>(ring + a.n_slots * a.slot_bytes + 16 * a.n_slots);
  int8_t* qs = reinterpret_cast<int8_t*>(acc + a.acc_ints);  // activations, layout eng_perm
  float* xs = reinterpret_cast<float*>(qs + a.qs_bytes);     // fp32 staging of one activation row
  float* hs = xs + a.xs_floats;                              // this CTA's rows of h [T][sub_rows]
  float* gs = hs + a.T * a.sub_rows;                         // and the sub-norm gain of those rows
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (a.n_slots + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.n_slots; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), ENG_CONS_WARPS);
    }
    s_abort = 0;
    s_issued = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  auto tile_range = [&](const EngPhase& p, int& tb, int& te) {
    if (p.balanced) {
      const int base = p.n_tiles / (int)gridDim.x, c = blockIdx.x;
      int below = 0;
      for (int w = 0; w < (c >> 5); ++w) below += __popc(p.xmask[w]);
      below += __popc(p.xmask[c >> 5] & ((1u << (c & 31)) - 1u));
      tb = c * base + below;
      te = tb + base + (int)((p.xmask[c >> 5] >> (c & 31)) & 1u);
    } else {
      tb = (int)((long long)blockIdx.x * p.n_tiles / gridDim.x);
      te = (int)((long long)(blockIdx.x + 1) * p.n_tiles / gridDim.x);
    }
  };
  auto locate = [&](const EngPhase& p, int tile, int& ti, int& n0, int& nrows) {
    ti = 0;
    if (p.kind == PH_GEMV)
      while (ti + 1 < p.n_tensors && tile >= p.t[ti + 1].tile_begin) ++ti;
    n0 = (tile - p.t[ti].tile_begin) * GEMV_ROWS;
    nrows = min(GEMV_ROWS, p.t[ti].N - n0);
  };

  if (warp == ENG_CONS_WARPS) {
    // ------------------------------------------------------------ producer
    // First, bulk L2 prefetches (one CTA per slice of the grid) of what the per-phase
    // quantisations read: every norm gain (immutable) and the raw activation rows of the
    // phases that do not wait for this launch (L2 is coherent, so a prefetch issued while the
    // previous kernel may still write them only warms the lines).  They land ahead of the
    // weight stream, so the quantisations' loads hit L2.
    if (lane == 0 && blockIdx.x < 8) {
      for (int pi = 0; pi < a.n_phases; ++pi) {
        const EngPhase& p = a.ph[pi];
        const float* g = p.kind == PH_SUBNORM ? nullptr : p.gain;
        const uint32_t gb = (uint32_t)p.K * 4u;
        if (g != nullptr && blockIdx.x == (pi & 7)) prefetch_l2_bulk(g, gb);
        if ((p.kind == PH_QUANT || (ph_is_gemv(p.kind) && p.src == SRC_LOCAL)) && p.wait_barrier < 0 &&
            blockIdx.x == ((pi + 4) & 7)) {
          const uint32_t xb = (uint32_t)T * (uint32_t)p.K * (p.x_f32 ? 4u : 2u);
          prefetch_l2_bulk(p.x, xb);
        }
        if (p.kind == PH_GEMV_FFN && p.sub_gain != nullptr && blockIdx.x == (pi & 7))
          prefetch_l2_bulk(p.sub_gain, (uint32_t)a.ph[pi].t[0].N * 4u);
      }
    }
    // Then walks the stage order of every product phase (engine_sched.h).  Lane 0 waits for
    // the slot, sets the expected bytes and issues the copies (no multicast).
    int slot = 0, issued = 0;
    uint32_t par = 0;
    bool go = true;  // warp-uniform: false once a wait gave up or the consumers aborted
    for (int pi = 0; pi < a.n_phases && go; ++pi) {
      const EngPhase& p = a.ph[pi];
      if (!ph_is_gemv(p.kind)) continue;
      const EngGeom& G = p.g;
      const int NT = p.kind == PH_GEMV_FFN ? 2 : 1;
      int tb, te;
      tile_range(p, tb, te);
      const int nt = te - tb;
      for (int ac = 0; ac < G.n_ac && go; ++ac) {
        const int wc0 = ac * G.ac_chunks, wc1 = min(G.n_chunks, wc0 + G.ac_chunks);
        for (int tg0 = 0; tg0 < nt && go; tg0 += G.rs) {
          const int ntg = min(G.rs, nt - tg0);
          for (int u = 0; u < NT && go; ++u) {
            for (int wc = wc0; wc < wc1 && go; ++wc) {
              bool ok = true;
              if (lane == 0) {
                ok = s_abort == 0 && mbar_wait_bounded(empty(slot), par ^ 1u);
                if (ok) {
                  const uint32_t dst = smem_addr(ring + slot * a.slot_bytes);
                  if (G.full_rows && ntg == 1) {
                    // one tile: one contiguous copy of its rows
                    int ti, n0, nr;
                    locate(p, tb + tg0, ti, n0, nr);
                    const uint32_t bytes = (uint32_t)nr * G.RB;
                    mbar_arrive_expect_tx(full(slot), bytes);
                    bulk_g2s(dst, p.t[NT == 2 ? u : ti].packed + (long long)n0 * G.RB, bytes, full(slot));
                  } else if (G.full_rows) {
                    // runs of consecutive tiles of the same tensor: one contiguous copy each
                    uint32_t bytes = 0;
                    for (int pass = 0; pass < 2; ++pass) {
                      if (pass == 1) mbar_arrive_expect_tx(full(slot), bytes);
                      for (int i = 0; i < ntg;) {
                        int ti, n0, nr;
                        locate(p, tb + tg0 + i, ti, n0, nr);
                        int j = i + 1, rows = nr;
                        while (j < ntg) {
                          int tj, m0, mr;
                          locate(p, tb + tg0 + j, tj, m0, mr);
                          if (tj != ti) break;
                          rows += mr;
                          ++j;
                        }
                        if (pass == 0) {
                          bytes += (uint32_t)rows * G.RB;
                        } else {
                          const uint8_t* src = p.t[NT == 2 ? u : ti].packed + (long long)n0 * G.RB;
                          bulk_g2s(dst + (uint32_t)(i * GEMV_ROWS * G.RB), src, (uint32_t)rows * G.RB, full(slot));
                        }
                        i = j;
                      }
                    }
                  } else {
                    int ti, n0, nr;
                    locate(p, tb + tg0, ti, n0, nr);
                    mbar_arrive_expect_tx(full(slot), (uint32_t)(GEMV_ROWS * G.CB));
                    tma_load_2d(dst, &maps.m[pi][NT == 2 ? u : ti], wc * (G.CB >> 3), n0, full(slot));
                  }
                  s_issued = ++issued;
                } else {
                  s_abort = 1;
                }
              }
              go = __shfl_sync(0xffffffffu, ok, 0);
              if (++slot == a.n_slots) {
                slot = 0;
                par ^= 1u;
              }
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, r = lane & 3;
    const int t_a = gid, t_b = 8 + gid;
    if (threadIdx.x < ENG_MAX_PHASES * 4) {
      // per-tensor scales (weights: no dependency wait needed); read by the epilogues, after
      // the named barriers of the first phase
      const int pi = threadIdx.x >> 2, u = threadIdx.x & 3;
      float b = 0.0f;
      if (pi < a.n_phases && ph_is_gemv(a.ph[pi].kind) && u < a.ph[pi].n_tensors) {
        const EngTensor& t = a.ph[pi].t[u];
        b = __ldg(reinterpret_cast<const float*>(t.packed + (long long)t.N * (a.ph[pi].K >> 2)));
      }
      s_beta[pi][u] = b;
    }
    pdl_wait();  // activations and workspace belong to the previous kernel until now
    int slot = 0;       // ring position of the next stage
    uint32_t par = 0;   // and the phase parity of its barriers
    // The SUBNORM phases accumulate sum_q with atomics: clear it before any CTA can get
    // there (the grid barrier of the gate/up phase comes first).
    if (blockIdx.x == 0 && threadIdx.x < T)
      for (int i = 0; i < a.n_phases; ++i)
        if (a.ph[i].kind == PH_SUBNORM) a.ph[i].sq[threadIdx.x] = 0;
    // Every branch that leaves the phase loop is taken by all consumer threads together
    // (barrier.red.or consensus), so no thread is left at a named barrier.
    for (int pi = 0; pi < a.n_phases; ++pi) {
      const EngPhase& p = a.ph[pi];
      if (named_sync_or(1, ENG_CONS, s_abort != 0)) break;
      if (p.wait_barrier >= 0) {
        const bool ok = grid_wait(a.counters + p.wait_barrier, gridDim.x);
        if (named_sync_or(1, ENG_CONS, !ok)) {
          s_abort = 1;
          break;
        }
      }
      if (p.kind == PH_QUANT) {
        for (int t = blockIdx.x; t < T; t += gridDim.x) {
          quant_row(reinterpret_cast<const uint8_t*>(p.x) + (long long)t * p.K * (p.x_f32 ? 4 : 2), p.x_f32, p.K,
                    p.gain, a.eps, p.q + (long long)t * p.K, false, p.s + t, p.sq + t, s_red, xs);
        }
        if (p.arrive_barrier >= 0) grid_arrive(a.counters + p.arrive_barrier);
        continue;
      }
      if (p.kind == PH_SUBNORM) {
        int tb0, te0;
        tile_range(p, tb0, te0);
        if (!eng_subnorm(p, T, a.eps, tb0, te0, a.counters, s_sub, hs, gs, a.sub_rows)) {
          s_abort = 1;
          break;
        }
        grid_arrive(a.counters + p.arrive_barrier);
        continue;
      }
      const EngGeom& G = p.g;
      const int NT = p.kind == PH_GEMV_FFN ? 2 : 1;
      int tb, te;
      tile_range(p, tb, te);
      const int nt = te - tb;
      const bool local = p.src == SRC_LOCAL;
      if (local) {
        // Quantise the raw activations in this CTA (whole row, full-row geometry), straight
        // into the shared layout; zero the padding of the last 256-in-feature step.
        for (int t = 0; t < T; ++t) {
          quant_row(reinterpret_cast<const uint8_t*>(p.x) + (long long)t * p.K * (p.x_f32 ? 4 : 2), p.x_f32, p.K,
                    p.gain, a.eps, qs + t * G.x_pitch, true, s_loc_s + t, s_loc_sq + t, s_red, xs);
        }
        const int pad16 = (((p.K + 255) & ~255) - p.K) >> 4;
        for (int i = threadIdx.x; i < T * pad16; i += ENG_CONS) {
          const int t = i / pad16, u = p.K / 16 + (i - t * pad16);
          *reinterpret_cast<uint4*>(qs + t * G.x_pitch + eng_perm(16 * u)) = make_uint4(0u, 0u, 0u, 0u);
        }
        if (blockIdx.x == 0 && p.q != nullptr) {  // one plain-order copy for callers that read the intermediates
          const int K16 = p.K >> 4;
          for (int i = threadIdx.x; i < T * K16; i += ENG_CONS) {
            const int t = i / K16, k = (i - t * K16) * 16;
            *reinterpret_cast<uint4*>(p.q + (long long)t * p.K + k) =
                *reinterpret_cast<const uint4*>(qs + t * G.x_pitch + eng_perm(k));
          }
          if (threadIdx.x < T) {
            p.s[threadIdx.x] = s_loc_s[threadIdx.x];
            p.sq[threadIdx.x] = s_loc_sq[threadIdx.x];
          }
        }
      }
      // Accumulators: [tile][tensor][16 rows][T], or with private warp slots (a.acc_priv)
      // [tile][tensor][warp][16 rows][T].
      const int aw = a.acc_priv ? ENG_CONS_WARPS : 1;
      for (int i = threadIdx.x; i < nt * NT * aw * GEMV_ROWS * T; i += ENG_CONS) acc[i] = 0;
      if (p.pmax != nullptr && p.sub_gain != nullptr) {
        // the SUBNORM phase's gain for this CTA's rows, fetched while the products run
        for (int i = threadIdx.x; i < nt * GEMV_ROWS / 4; i += ENG_CONS)
          cp_async16(smem_addr(gs + 4 * i), p.sub_gain + (long long)tb * GEMV_ROWS + 4 * i);
        cp_async_commit();
      }

      {
        const uint32_t qs_s = smem_addr(qs);
        const int ta = min(t_a, T - 1), tb2 = min(t_b, T - 1);
        const uint32_t xa0 = qs_s + ta * G.x_pitch + 16 * r, xb0 = qs_s + tb2 * G.x_pitch + 16 * r;
        const uint32_t ring_s = smem_addr(ring);
        EngAcc<TG> A;
        A.zero();
        // The stage's tiles go to groups of wpt warps (per phase constants); within a group the
        // steps are dealt round-robin, continuing from stage to stage.  The stage loop's
        // parameters are taken out of the shared descriptors once.
        const int CB = G.CB, RB = G.RB, n_chunks = G.n_chunks, rs = G.rs, n_ac = G.n_ac, ac_chunks = G.ac_chunks;
        const int n_slots = a.n_slots, slot_bytes = a.slot_bytes;
        const bool priv = a.acc_priv != 0;
        const uint32_t full0 = full(0), empty0 = empty(0);
        const int wpt = ENG_CONS_WARPS / rs, my_tl = warp / wpt, my_wi = warp - my_tl * wpt;
        const int S_full = (CB + 63) >> 6;  // steps of a whole chunk
        int* const acc_w = acc + (priv ? warp : 0) * GEMV_ROWS * T;
        int rot = 0;
        // A warp whose wait gives up stops waiting and computing but keeps walking the stage
        // order, so that every consumer thread meets the same named barriers; the decision
        // to leave is taken together at the next one (barrier.red.or).
        bool ok = true;
        for (int ac = 0; ac < n_ac; ++ac) {
          const int wc0 = ac * ac_chunks, wc1 = min(n_chunks, wc0 + ac_chunks);
          if (!local) {
            // the previous chunk's readers are done, then stage this chunk
            if (named_sync_or(1, ENG_CONS, !ok)) {
              ok = false;
              break;
            }
            eng_stage_acts(p.q, p.K, T, 4 * wc0 * CB, min(p.K, 4 * wc1 * CB), qs, G.x_pitch);
          }
          if (named_sync_or(1, ENG_CONS, !ok)) {
            ok = false;
            break;
          }
          if (rs == 1) {
            const int at_step = aw * GEMV_ROWS * T;
            if (TG == 1 && T == 1) {
              if (CB == 2048)
                eng_flat_stages<TG, 2048, true>(A, nt * NT, wc0, wc1, n_chunks, CB, RB, ring_s, slot_bytes, n_slots, full0,
                                                empty0, xa0, xb0, acc_w, at_step, T, priv, warp, gid, r, lane, slot, par,
                                                rot, ok);
              else
                eng_flat_stages<TG, 0, true>(A, nt * NT, wc0, wc1, n_chunks, CB, RB, ring_s, slot_bytes, n_slots, full0,
                                             empty0, xa0, xb0, acc_w, at_step, T, priv, warp, gid, r, lane, slot, par, rot,
                                             ok);
            } else {
              if (CB == 2048)
                eng_flat_stages<TG, 2048, false>(A, nt * NT, wc0, wc1, n_chunks, CB, RB, ring_s, slot_bytes, n_slots, full0,
                                                 empty0, xa0, xb0, acc_w, at_step, T, priv, warp, gid, r, lane, slot, par,
                                                 rot, ok);
              else
                eng_flat_stages<TG, 0, false>(A, nt * NT, wc0, wc1, n_chunks, CB, RB, ring_s, slot_bytes, n_slots, full0,
                                              empty0, xa0, xb0, acc_w, at_step, T, priv, warp, gid, r, lane, slot, par, rot,
                                              ok);
            }
            continue;
          }
          for (int tg0 = 0; tg0 < nt; tg0 += rs) {
            const int ntg = min(rs, nt - tg0);
            for (int u = 0; u < NT; ++u) {
              for (int wc = wc0; wc < wc1; ++wc) {
                if (ok && !mbar_wait_bounded(full0 + 8u * slot, par)) ok = false;
                if (ok) {
                  const int S = wc < n_chunks - 1 ? S_full : (RB - wc * CB + 63) >> 6;
                  const uint32_t xoff = 256u * (uint32_t)((wc - wc0) * (CB >> 6));
                  const uint32_t sbase = ring_s + slot * slot_bytes + gid * CB + 16 * r;
                  if (my_tl < ntg) {
                    int t0 = my_wi - rot;
                    if (t0 < 0) t0 += wpt;
                    eng_tile_steps<TG>(A, sbase + my_tl * GEMV_ROWS * CB, CB, xa0 + xoff, xb0 + xoff, t0, S, wpt);
                    if (wc == wc1 - 1)
                      A.flush(acc_w + ((tg0 + my_tl) * NT + u) * aw * GEMV_ROWS * T, T, gid, r, priv);
                  }
                  rot += S;
                  while (rot >= wpt) rot -= wpt;
                  __syncwarp();
                  if (lane == 0) mbar_arrive(empty0 + 8u * slot);
                }
                if (++slot == n_slots) {
                  slot = 0;
                  par ^= 1u;
                }
              }
            }
          }
        }
        if (!ok) s_abort = 1;
      }
      if (named_sync_or(1, ENG_CONS, s_abort != 0)) break;
      // Epilogue of this phase's tiles.
      const int n_out = nt * GEMV_ROWS * T;
      for (int idx = threadIdx.x; idx < n_out; idx += ENG_CONS) {
        const int tl2 = idx / (GEMV_ROWS * T), rem = idx - tl2 * (GEMV_ROWS * T);
        const int t = rem / GEMV_ROWS, row = rem - t * GEMV_ROWS;
        int ti, n0, nrows;
        locate(p, tb + tl2, ti, n0, nrows);
        if (row >= nrows) continue;
        const long long n = n0 + row;
        const int N = p.t[ti].N;
        const int sq = local ? s_loc_sq[t] : __ldcg(p.sq + t);
        // s_x may be absent when only the int32 accumulators are asked for (no float output).
        const float sx = local ? s_loc_s[t] : (p.s != nullptr ? __ldcg(p.s + t) : 1.0f);
        const int* at = acc + tl2 * NT * aw * GEMV_ROWS * T;
        int sumA = 0, sumU = 0;
        for (int w = 0; w < aw; ++w) {
          sumA += at[(w * GEMV_ROWS + row) * T + t];
          if (NT == 2) sumU += at[((aw + w) * GEMV_ROWS + row) * T + t];
        }
        const int accA = sumA - sq;
        const float betaA = s_beta[pi][ti];
        const float vA = dequant(accA, __fdiv_rn(betaA, sx));
        if (NT == 2) {
          const float betaU = s_beta[pi][1];
          const int accU = sumU - sq;
          const float vU = dequant(accU, __fdiv_rn(betaU, sx));
          const float hv = ffn_act(vA, vU, p.act);
          p.h[(long long)t * N + n] = hv;
          if (p.pmax != nullptr) hs[t * a.sub_rows + tl2 * GEMV_ROWS + row] = hv;  // kept for the SUBNORM phase
        } else {
          if (p.t[ti].out) store_out(p.t[ti].out, p.out_dtype, (long long)t * N + n, vA);
          if (p.t[ti].acc_debug) p.t[ti].acc_debug[(long long)t * N + n] = accA;
        }
      }
      if (p.arrive_barrier >= 0)
        grid_arrive(a.counters + p.arrive_barrier);
      else
        cons_sync();  // acc and the staged activations are reused by the next phase
    }
  }

  cp_async_wait_all();
  __syncthreads();
  // After an abort, copies the producer issued may still be in flight into this CTA's shared
  // memory: wait for every slot's last fill to land (fixed limit) before the CTA exits.
  if (s_abort && threadIdx.x == 0) {
    const int issued = s_issued;
    for (int k = (issued > a.n_slots ? issued - a.n_slots : 0); k < issued; ++k)
      mbar_drain(full(k % a.n_slots), (uint32_t)((k / a.n_slots) & 1));
  }
  if (threadIdx.x == 0 && a.counters != nullptr) {
    // The last CTA out zeroes the barrier counters for the next launch.
    __threadfence();
    const unsigned prev = atomicAdd(a.counters + ENG_MAX_BARRIERS, 1u);
    if (prev == gridDim.x - 1) {
      for (int b = 0; b <= ENG_MAX_BARRIERS; ++b) atomicExch(a.counters + b, 0u);
      __threadfence();
    }
  }
}

}  // namespace bitnet

// The decode engine: every BitLinear step of a small-token-count forward (T <= 16) in
// ONE persistent launch.  A forward is a list of phases:
//
//   GEMV      the product of one or more I2_S tensors (or the FFN's gate/up pair with
//             h = act(g) * u fused into the epilogue) with an int8 activation batch that
//             is either given (q, s_x, sum_q in global memory) or quantised by every CTA
//             itself from the raw activations (RMSNorm + absmax int8 in registers);
//   QUANT     RMSNorm + absmax int8 of a larger activation batch, tokens split over CTAs,
//             written to global memory.
//
// A phase may arrive on a grid barrier after its epilogue (its outputs are complete
// once every CTA has arrived) and may wait on one before it reads its inputs.  Arrival
// and wait are split, so independent work (the q/k/v projections while the o output
// is being completed) fills the wait.
//
// Weights do not depend on any phase, so a producer warp streams the packed bytes of
// ALL phases of this CTA, in phase order, through a ring of shared-memory slots with
// cp.async.bulk; it starts before griddepcontrol.wait, i.e. while the previous kernel
// on the stream is still running.  Consumer warps (8) work through the stages exactly
// as in the single-phase decode product (gemv.cuh: one AND per 2-bit field, mma.sync
// m16n8k32 u8 x s8, per-field accumulators combined exactly).
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
#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int ENG_CONS_WARPS = 8;
constexpr int ENG_CONS = ENG_CONS_WARPS * 32;
constexpr int ENG_THREADS = ENG_CONS + 32;
constexpr int ENG_MAX_PHASES = 8;
constexpr int ENG_MAX_BARRIERS = 8;
constexpr int ENG_ROW_PAD = 64;
constexpr int ENG_LOCAL_MAX_K = 8192;  // local quantisation keeps <= 32 values per thread
constexpr int ENG_MAX_T = 16;

enum { PH_GEMV = 0, PH_GEMV_FFN = 1, PH_QUANT = 2 };
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
  int chunk_bytes, n_chunks, row_stride, stage_bytes;
};

struct EngArgs {
  int T;
  float eps;
  int n_phases;
  unsigned* counters;  // ENG_MAX_BARRIERS + 1 words in the workspace (last: exit count)
  int n_slots, slot_bytes, acc_ints, qs_bytes;
  EngPhase ph[ENG_MAX_PHASES];
};

// ------------------------------------------------------------------ consumer-group helpers
BN_DEV void cons_sync() { named_sync(1, ENG_CONS); }

template <typename T, typename Op>
BN_DEV T cons_reduce(T v, T* scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  cons_sync();
  if (lane == 0) scratch[warp] = v;
  cons_sync();
  T r = scratch[0];
#pragma unroll
  for (int w = 1; w < ENG_CONS_WARPS; ++w) r = op(r, scratch[w]);
  return r;
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

// RMSNorm + absmax int8 of one row of K <= ENG_LOCAL_MAX_K values held in registers by
// the 256 consumer threads (thread i owns elements 8(i + 256 j) .. +7).  Writes q (into
// `qdst`, shared or global), s_x and sum_q (thread 0).  Same operation sequence as
// quant.cuh: exact fixed-point sum of x^2, fp32 steps without contraction.
BN_DEV void quant_row_regs(const void* xrow, int x_f32, int K, const float* gain, float eps, int8_t* qdst,
                           float* s_dst, int32_t* sq_dst, void* red) {
  const int tid = threadIdx.x;
  float v[4][8];
  float am = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int k = 8 * (tid + ENG_CONS * j);
    if (k < K) {
      load8(xrow, x_f32, k, v[j]);
#pragma unroll
      for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[j][i]));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
    }
  }
  am = cons_reduce(am, reinterpret_cast<float*>(red), MaxOp());
  float a = am;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (am > 0.0f) {
      const double M = __dmul_rn((double)am, (double)am);
      const int e = fixed_point_exponent(M, K);
      const double p2e = pow2_f64(e);
      long long part = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double d = (double)v[j][i];
          part += __double2ll_rn(__dmul_rn(__dmul_rn(d, d), p2e));
        }
      const long long S = cons_reduce(part, reinterpret_cast<long long*>(red), AddOpLL());
      ms = fixed_point_mean(S, e, K);
    }
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float ay = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = 8 * (tid + ENG_CONS * j);
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
    a = cons_reduce(ay, reinterpret_cast<float*>(red), MaxOp());
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int k = 8 * (tid + ENG_CONS * j);
    if (k < K) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qv = __float2int_rn(__fmul_rn(v[j][i], s));
        qv = min(127, max(-128, qv));
        sum += qv;
        w[i >> 2] |= (uint32_t)(qv & 0xFF) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2*>(qdst + k) = make_uint2(w[0], w[1]);
    }
  }
  sum = cons_reduce(sum, reinterpret_cast<int*>(red), AddOpI());
  if (tid == 0) {
    *s_dst = s;
    *sq_dst = sum;
  }
}

// The same for any K, streaming the row from global memory in four passes (used when a
// CTA quantises whole tokens for everyone: the QUANT phase).
BN_DEV void quant_row_stream(const void* xrow, int x_f32, int K, const float* gain, float eps, int8_t* qdst,
                             float* s_dst, int32_t* sq_dst, void* red) {
  const int tid = threadIdx.x;
  float v[8];
  float am = 0.0f;
  for (int k = 8 * tid; k < K; k += 8 * ENG_CONS) {
    load8(xrow, x_f32, k, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
  }
  am = cons_reduce(am, reinterpret_cast<float*>(red), MaxOp());
  float a = am, inv = 1.0f;
  if (gain != nullptr) {
    float ms = 0.0f;
    if (am > 0.0f) {
      const double M = __dmul_rn((double)am, (double)am);
      const int e = fixed_point_exponent(M, K);
      const double p2e = pow2_f64(e);
      long long part = 0;
      for (int k = 8 * tid; k < K; k += 8 * ENG_CONS) {
        load8(xrow, x_f32, k, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double d = (double)v[i];
          part += __double2ll_rn(__dmul_rn(__dmul_rn(d, d), p2e));
        }
      }
      const long long S = cons_reduce(part, reinterpret_cast<long long*>(red), AddOpLL());
      ms = fixed_point_mean(S, e, K);
    }
    inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float ay = 0.0f;
    for (int k = 8 * tid; k < K; k += 8 * ENG_CONS) {
      load8(xrow, x_f32, k, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) ay = fmaxf(ay, fabsf(__fmul_rn(__fmul_rn(v[i], inv), __ldg(gain + k + i))));
    }
    a = cons_reduce(ay, reinterpret_cast<float*>(red), MaxOp());
  }
  const float s = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
  int sum = 0;
  for (int k = 8 * tid; k < K; k += 8 * ENG_CONS) {
    load8(xrow, x_f32, k, v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float y = gain != nullptr ? __fmul_rn(__fmul_rn(v[i], inv), __ldg(gain + k + i)) : v[i];
      int qv = __float2int_rn(__fmul_rn(y, s));
      qv = min(127, max(-128, qv));
      sum += qv;
      w[i >> 2] |= (uint32_t)(qv & 0xFF) << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(qdst + k) = make_uint2(w[0], w[1]);
  }
  sum = cons_reduce(sum, reinterpret_cast<int*>(red), AddOpI());
  if (tid == 0) {
    *s_dst = s;
    *sq_dst = sum;
  }
}

// ------------------------------------------------------------------ grid barriers
BN_DEV void grid_arrive(unsigned* ctr) {
  cons_sync();  // every consumer thread of this CTA has written its outputs
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
  }
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
      if (now - t0 > kWaitLimitCycles) {
        atomicExch(&g_device_status, (int)BITNET_ERR_TIMEOUT);
        ok = false;
        break;
      }
    }
    __threadfence();
  }
  return ok;
}

// ------------------------------------------------------------------ the kernel
template <int TG>
__global__ void __launch_bounds__(ENG_THREADS, TG == 1 ? 2 : 1) k_engine(const EngArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  volatile __shared__ int s_abort;
  __shared__ long long s_red[ENG_CONS_WARPS];
  __shared__ float s_loc_s[ENG_MAX_T];
  __shared__ int32_t s_loc_sq[ENG_MAX_T];

  uint8_t* ring = smem;
  const uint32_t bar0 = smem_addr(smem + a.n_slots * a.slot_bytes);
  int* acc = reinterpret_cast<int*>(smem + a.n_slots * a.slot_bytes + 16 * a.n_slots);
  int8_t* qs = reinterpret_cast<int8_t*>(acc + a.acc_ints);
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
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  auto tile_range = [&](const EngPhase& p, int& tb, int& te) {
    tb = (int)((long long)blockIdx.x * p.n_tiles / gridDim.x);
    te = (int)((long long)(blockIdx.x + 1) * p.n_tiles / gridDim.x);
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
    int st = 0;
    for (int pi = 0; pi < a.n_phases && !s_abort; ++pi) {
      const EngPhase& p = a.ph[pi];
      if (p.kind == PH_QUANT) continue;
      const int NT = p.kind == PH_GEMV_FFN ? 2 : 1;
      const int row_bytes = p.K >> 2;
      int tb, te;
      tile_range(p, tb, te);
      for (int tile = tb; tile < te && !s_abort; ++tile) {
        int ti, n0, nrows;
        locate(p, tile, ti, n0, nrows);
        for (int c = 0; c < p.n_chunks; ++c, ++st) {
          const int slot = st % a.n_slots;
          bool ok = true;
          if (lane == 0) ok = mbar_wait_bounded(empty(slot), ((st / a.n_slots) & 1) ^ 1);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            s_abort = 1;
            break;
          }
          const int cb = min(p.chunk_bytes, row_bytes - c * p.chunk_bytes);
          if (lane == 0) mbar_arrive_expect_tx(full(slot), (uint32_t)(nrows * cb * NT));
          __syncwarp();
          for (int idx = lane; idx < nrows * NT; idx += 32) {
            const int u = idx / nrows, r = idx % nrows;
            const uint8_t* src =
                p.t[NT == 2 ? u : ti].packed + (long long)(n0 + r) * row_bytes + (long long)c * p.chunk_bytes;
            bulk_g2s(smem_addr(ring + slot * a.slot_bytes + (u * GEMV_ROWS + r) * p.row_stride), src, (uint32_t)cb,
                     full(slot));
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, r = lane & 3;
    const int t_a = gid, t_b = 8 + gid;
    pdl_wait();  // activations and workspace belong to the previous kernel until now
    int st = 0;
    // Every branch that leaves the phase loop is taken by all 256 consumer threads
    // together (barrier.red.or consensus), so no thread is left at a named barrier.
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
          quant_row_stream(reinterpret_cast<const uint8_t*>(p.x) + (long long)t * p.K * (p.x_f32 ? 4 : 2), p.x_f32,
                           p.K, p.gain, a.eps, p.q + (long long)t * p.K, p.s + t, p.sq + t, s_red);
        }
        if (p.arrive_barrier >= 0) grid_arrive(a.counters + p.arrive_barrier);
        continue;
      }
      const int NT = p.kind == PH_GEMV_FFN ? 2 : 1;
      const int row_bytes = p.K >> 2;
      int tb, te;
      tile_range(p, tb, te);
      // Activations of this phase.
      const bool local = p.src == SRC_LOCAL;
      if (local) {
        for (int t = 0; t < T; ++t) {
          quant_row_regs(reinterpret_cast<const uint8_t*>(p.x) + (long long)t * p.K * (p.x_f32 ? 4 : 2), p.x_f32,
                         p.K, p.gain, a.eps, qs + t * p.K, s_loc_s + t, s_loc_sq + t, s_red);
        }
        if (blockIdx.x == 0 && p.q != nullptr) {  // one copy for callers that read the intermediates
          for (int i = threadIdx.x; i < T * p.K / 16; i += ENG_CONS)
            reinterpret_cast<uint4*>(p.q)[i] = reinterpret_cast<const uint4*>(qs)[i];
          if (threadIdx.x < T) {
            p.s[threadIdx.x] = s_loc_s[threadIdx.x];
            p.sq[threadIdx.x] = s_loc_sq[threadIdx.x];
          }
        }
      }
      for (int i = threadIdx.x; i < (te - tb) * NT * 256; i += ENG_CONS) acc[i] = 0;
      cons_sync();

      // Products: the global step index g runs over (stage, 64-byte step); warp w takes
      // the steps with g % 8 == w, so short stages still use every warp.
      int f[2][TG][4][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int i = 0; i < 4; ++i) f[u][tg][g][i] = 0;
      bool have = false;
      int gstep = 0;
      for (int tile = tb; tile < te && !s_abort; ++tile) {
        int ti, n0, nrows;
        locate(p, tile, ti, n0, nrows);
        for (int c = 0; c < p.n_chunks; ++c, ++st) {
          const int slot = st % a.n_slots;
          const int cb = min(p.chunk_bytes, row_bytes - c * p.chunk_bytes);
          const int nsteps = (cb + 63) >> 6;
          const int first = (warp - gstep % ENG_CONS_WARPS + ENG_CONS_WARPS) % ENG_CONS_WARPS;
          if (s_abort) break;
          if (first < nsteps) {
            if (!mbar_wait_bounded(full(slot), (st / a.n_slots) & 1)) {
              s_abort = 1;
              break;
            }
            const uint8_t* sbase = ring + slot * a.slot_bytes;
            for (int step = first; step < nsteps; step += ENG_CONS_WARPS) {
              const int boff = 64 * step + 16 * r;
              const bool valid = boff < cb;
              uint4 wa[2], wb[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                if (u < NT) {
                  const uint8_t* rb = sbase + u * GEMV_ROWS * p.row_stride + boff;
                  wa[u] = (valid && gid < nrows) ? *reinterpret_cast<const uint4*>(rb + gid * p.row_stride)
                                                 : make_uint4(0, 0, 0, 0);
                  wb[u] = (valid && gid + 8 < nrows) ? *reinterpret_cast<const uint4*>(rb + (gid + 8) * p.row_stride)
                                                     : make_uint4(0, 0, 0, 0);
                }
              }
              const int kb = 4 * (c * p.chunk_bytes + 64 * step) + 128 * (r >> 1) + 16 * (r & 1);
              uint4 xa[4], xb[4];
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const uint4 z = make_uint4(0, 0, 0, 0);
                if (local) {
                  xa[g] = (valid && t_a < T) ? *reinterpret_cast<const uint4*>(qs + t_a * p.K + kb + 32 * g) : z;
                  xb[g] = (TG > 1 && valid && t_b < T) ? *reinterpret_cast<const uint4*>(qs + t_b * p.K + kb + 32 * g)
                                                       : z;
                } else {
                  xa[g] = (valid && t_a < T)
                              ? __ldcg(reinterpret_cast<const uint4*>(p.q + (long long)t_a * p.K + kb + 32 * g))
                              : z;
                  xb[g] = (TG > 1 && valid && t_b < T)
                              ? __ldcg(reinterpret_cast<const uint4*>(p.q + (long long)t_b * p.K + kb + 32 * g))
                              : z;
                }
              }
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                if (u < NT) {
#pragma unroll
                  for (int g = 0; g < 4; ++g) {
                    const uint32_t m = 0x03030303u << (6 - 2 * g);
                    mma_u8s8(f[u][0][g], wa[u].x & m, wb[u].x & m, wa[u].y & m, wb[u].y & m, xa[g].x, xa[g].y);
                    mma_u8s8(f[u][0][g], wa[u].z & m, wb[u].z & m, wa[u].w & m, wb[u].w & m, xa[g].z, xa[g].w);
                    if (TG > 1) {
                      mma_u8s8(f[u][TG - 1][g], wa[u].x & m, wb[u].x & m, wa[u].y & m, wb[u].y & m, xb[g].x, xb[g].y);
                      mma_u8s8(f[u][TG - 1][g], wa[u].z & m, wb[u].z & m, wa[u].w & m, wb[u].w & m, xb[g].z, xb[g].w);
                    }
                  }
                }
              }
            }
            have = true;
          }
          gstep += nsteps;
          __syncwarp();
          if (lane == 0) mbar_arrive(empty(slot));
          if (c == p.n_chunks - 1) {
            if (have) {
              int* at = acc + (tile - tb) * NT * 256;
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                if (u < NT) {
#pragma unroll
                  for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                      const int v = (f[u][tg][0][i] >> 6) + (f[u][tg][1][i] >> 4) + (f[u][tg][2][i] >> 2) + f[u][tg][3][i];
                      const int row = gid + ((i & 2) ? 8 : 0), tok = tg * 8 + 2 * r + (i & 1);
                      if (tok < T && row < nrows) atomicAdd(at + u * 256 + row * 16 + tok, v);
#pragma unroll
                      for (int g = 0; g < 4; ++g) f[u][tg][g][i] = 0;
                    }
                }
              }
            }
            have = false;
          }
        }
      }
      if (named_sync_or(1, ENG_CONS, s_abort != 0)) break;
      // Epilogue of this phase's tiles.
      const int n_out = (te - tb) * GEMV_ROWS * T;
      for (int idx = threadIdx.x; idx < n_out; idx += ENG_CONS) {
        const int tl = idx / (GEMV_ROWS * T), rem = idx % (GEMV_ROWS * T);
        const int t = rem / GEMV_ROWS, row = rem % GEMV_ROWS;
        int ti, n0, nrows;
        locate(p, tb + tl, ti, n0, nrows);
        if (row >= nrows) continue;
        const long long n = n0 + row;
        const int N = p.t[ti].N;
        const int sq = local ? s_loc_sq[t] : __ldcg(p.sq + t);
        const float sx = local ? s_loc_s[t] : __ldcg(p.s + t);
        const int* at = acc + tl * NT * 256;
        const int accA = at[row * 16 + t] - sq;
        const float betaA = __ldg(reinterpret_cast<const float*>(p.t[ti].packed + (long long)N * row_bytes));
        const float vA = dequant(accA, __fdiv_rn(betaA, sx));
        if (NT == 2) {
          const float betaU = __ldg(reinterpret_cast<const float*>(p.t[1].packed + (long long)N * row_bytes));
          const int accU = at[256 + row * 16 + t] - sq;
          const float vU = dequant(accU, __fdiv_rn(betaU, sx));
          p.h[(long long)t * N + n] = ffn_act(vA, vU, p.act);
        } else {
          store_out(p.t[ti].out, p.out_dtype, (long long)t * N + n, vA);
          if (p.t[ti].acc_debug) p.t[ti].acc_debug[(long long)t * N + n] = accA;
        }
      }
      if (p.arrive_barrier >= 0)
        grid_arrive(a.counters + p.arrive_barrier);
      else
        cons_sync();  // acc and the local activations are reused by the next phase
    }
  }

  __syncthreads();
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

// K-dec (pipelined): the BitLinear product for up to 16 tokens, streaming the packed
// weights through shared memory with bulk copies.
//
// Arithmetic as in gemv.cuh ("fix: I2_S ARM kernel layout + squared-ReLU FFN", bullet
// "I2_S NEON kernel for the canonical layout": acc = sum q*c - sum q, codes in the
// interleaved 128/32 layout; out = fp32(acc) * (beta / s_x)).  Layout of the work:
//
//  * one CTA per SM (persistent); CTA b owns a contiguous range of 16-row tiles, whose
//    packed bytes are contiguous rows of the tensor(s);
//  * a producer warp streams each tile in K-chunks ("stages") into a ring of shared
//    memory slots with cp.async.bulk (one copy per row, rows padded by 64 bytes so
//    that the 16-byte reads of 8 rows fall on distinct banks), completing on an
//    mbarrier; it issues the first slots BEFORE griddepcontrol.wait, because weights do
//    not depend on the previous kernel -- they stream in while that kernel finishes;
//  * 8 consumer warps take the 64-byte steps of each stage (256 in-features of 16
//    rows), unpack with one AND per field and run mma.sync m16n8k32 (u8 x s8), keep
//    per-field accumulators across the chunks of a tile, and add them into a per-tile
//    shared accumulator when the tile ends;
//  * after the last stage, all consumers run the epilogue (activation-sum correction,
//    dequantisation, bf16/fp32 store, or the FFN's h = act(g) * u).
//
// Every wait is bounded (about a second); a wait that gives up sets the device status
// word to BITNET_ERR_TIMEOUT and the CTA skips its epilogue.
#pragma once
#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int DEC_CONS_WARPS = 8;
constexpr int DEC_THREADS = (DEC_CONS_WARPS + 1) * 32;
constexpr int DEC_ROW_PAD = 64;
constexpr int DEC_MAX_TILES_CTA = 16;
constexpr int DEC_MAX_T = 16;

struct DecPlan {
  int chunk_bytes;  // bytes of one row per stage (multiple of 64, except a shorter last chunk)
  int n_chunks;     // stages per tile
  int row_stride;   // chunk_bytes + DEC_ROW_PAD
  int stage_bytes;  // 16 rows x row_stride x tensors
  int n_slots;      // ring depth
  int acc_tiles;    // tile slots of the shared accumulator
  int smem_bytes;
};

template <bool FFN, int TG>  // TG: token groups of 8 (T <= 8 * TG)
__global__ void __launch_bounds__(DEC_THREADS, 1) k_decode(const GemvArgs a, const DecPlan p) {
  constexpr int NT = FFN ? 2 : 1;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_abort;
  __shared__ int s_issued;
  uint8_t* ring = smem;
  const uint32_t bar0 = smem_addr(smem + p.n_slots * p.stage_bytes);  // full[S] then empty[S]
  int* acc = reinterpret_cast<int*>(smem + p.n_slots * p.stage_bytes + 16 * p.n_slots);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (p.n_slots + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = (int)((long long)blockIdx.x * a.n_tiles / gridDim.x);
  const int t_end = (int)((long long)(blockIdx.x + 1) * a.n_tiles / gridDim.x);
  const int n_stages = (t_end - t_begin) * p.n_chunks;
  const int row_bytes = a.K >> 2;

  for (int i = threadIdx.x; i < (t_end - t_begin) * NT * 256; i += blockDim.x) acc[i] = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_slots; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), DEC_CONS_WARPS);
    }
    s_abort = 0;
    s_issued = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // Tile -> (tensor, first row, valid rows).
  auto locate = [&](int tile, int& ti, int& n0, int& nrows) {
    ti = 0;
    if (!FFN)
      while (ti + 1 < a.n_tensors && tile >= a.t[ti + 1].tile_begin) ++ti;
    n0 = (tile - a.t[ti].tile_begin) * GEMV_ROWS;
    nrows = min(GEMV_ROWS, a.t[ti].N - n0);
  };

  if (warp == DEC_CONS_WARPS) {
    // ------------------------------------------------------------ producer
    for (int st = 0; st < n_stages; ++st) {
      const int slot = st % p.n_slots;
      if (st >= p.n_slots) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(empty(slot), ((st / p.n_slots) - 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          s_abort = 1;
          break;
        }
      }
      int ti, n0, nrows;
      locate(t_begin + st / p.n_chunks, ti, n0, nrows);
      const int c = st % p.n_chunks;
      const int cb = min(p.chunk_bytes, row_bytes - c * p.chunk_bytes);
      if (lane == 0) mbar_arrive_expect_tx(full(slot), (uint32_t)(nrows * cb * NT));
      __syncwarp();
      for (int idx = lane; idx < nrows * NT; idx += 32) {
        const int u = idx / nrows, r = idx % nrows;
        const uint8_t* src = a.t[FFN ? u : ti].packed + (long long)(n0 + r) * row_bytes + (long long)c * p.chunk_bytes;
        uint8_t* dst = ring + slot * p.stage_bytes + (u * GEMV_ROWS + r) * p.row_stride;
        bulk_g2s(smem_addr(dst), src, (uint32_t)cb, full(slot));
      }
      if (lane == 0) s_issued = st + 1;
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, r = lane & 3;
    pdl_wait();  // activations come from the previous kernel
    const int T = a.T;
    const int t_a = gid, t_b = 8 + gid;
    int f[NT][TG][4][4];
#pragma unroll
    for (int u = 0; u < NT; ++u)
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int i = 0; i < 4; ++i) f[u][tg][g][i] = 0;
    bool have = false;
    for (int st = 0; st < n_stages; ++st) {
      const int slot = st % p.n_slots;
      int ti, n0, nrows;
      locate(t_begin + st / p.n_chunks, ti, n0, nrows);
      const int c = st % p.n_chunks;
      const int cb = min(p.chunk_bytes, row_bytes - c * p.chunk_bytes);
      const int nsteps = (cb + 63) >> 6;
      if (warp < nsteps) {
        bool ok = mbar_wait_bounded(full(slot), (st / p.n_slots) & 1);
        if (!ok) {
          s_abort = 1;
          break;
        }
        const uint8_t* sbase = ring + slot * p.stage_bytes;
        for (int step = warp; step < nsteps; step += DEC_CONS_WARPS) {
          const int boff = 64 * step + 16 * r;
          const bool valid = boff < cb;
          uint4 wa[NT], wb[NT];
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            const uint8_t* rb = sbase + u * GEMV_ROWS * p.row_stride + boff;
            wa[u] = (valid && gid < nrows) ? *reinterpret_cast<const uint4*>(rb + gid * p.row_stride)
                                           : make_uint4(0, 0, 0, 0);
            wb[u] = (valid && gid + 8 < nrows) ? *reinterpret_cast<const uint4*>(rb + (gid + 8) * p.row_stride)
                                               : make_uint4(0, 0, 0, 0);
          }
          const int kb = 4 * (c * p.chunk_bytes + 64 * step) + 128 * (r >> 1) + 16 * (r & 1);
          uint4 xa[4], xb[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            xa[g] = (valid && t_a < T) ? __ldg(reinterpret_cast<const uint4*>(a.q + (long long)t_a * a.K + kb + 32 * g))
                                       : make_uint4(0, 0, 0, 0);
            xb[g] = (TG > 1 && valid && t_b < T)
                        ? __ldg(reinterpret_cast<const uint4*>(a.q + (long long)t_b * a.K + kb + 32 * g))
                        : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < NT; ++u)
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
        have = true;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(slot));
      if (c == p.n_chunks - 1) {
        if (have) {
          int* at = acc + (st / p.n_chunks) * NT * 256;
#pragma unroll
          for (int u = 0; u < NT; ++u)
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
        have = false;
      }
    }
  }
  __syncthreads();
  if (s_abort) {
    // A wait gave up: let the copies this CTA issued land before it exits (bounded).
    if (warp == DEC_CONS_WARPS && lane == 0) {
      for (int st = s_issued - 1; st >= 0 && st >= s_issued - p.n_slots; --st)
        mbar_wait_bounded(full(st % p.n_slots), (st / p.n_slots) & 1);
    }
    return;
  }

  // ------------------------------------------------------------ epilogue (all threads)
  const int T = a.T;
  const int n_out = (t_end - t_begin) * GEMV_ROWS * T;
  for (int idx = threadIdx.x; idx < n_out; idx += blockDim.x) {
    const int tl = idx / (GEMV_ROWS * T), rem = idx % (GEMV_ROWS * T);
    const int t = rem / GEMV_ROWS, row = rem % GEMV_ROWS;
    int ti, n0, nrows;
    locate(t_begin + tl, ti, n0, nrows);
    if (row >= nrows) continue;
    const long long n = n0 + row;
    const int N = a.t[ti].N;
    const int sq = __ldg(a.sum_q + t);
    const float sx = __ldg(a.s_x + t);
    const int* at = acc + tl * NT * 256;
    const int accA = at[row * 16 + t] - sq;
    const float betaA = __ldg(reinterpret_cast<const float*>(a.t[ti].packed + (long long)N * row_bytes));
    const float vA = dequant(accA, __fdiv_rn(betaA, sx));
    if (FFN) {
      const float betaU = __ldg(reinterpret_cast<const float*>(a.t[1].packed + (long long)N * row_bytes));
      const int accU = at[256 + row * 16 + t] - sq;
      const float vU = dequant(accU, __fdiv_rn(betaU, sx));
      a.h[(long long)t * N + n] = ffn_act(vA, vU, a.act);
    } else {
      store_out(a.t[ti].out, a.out_dtype, (long long)t * N + n, vA);
      if (a.t[ti].acc_debug) a.t[ti].acc_debug[(long long)t * N + n] = accA;
    }
  }
}

// Launch geometry of k_decode for a problem of n_tiles 16-row tiles of K in-features.
inline DecPlan plan_decode(int n_tiles, int K, bool ffn, int sms, int* grid) {
  const int NT = ffn ? 2 : 1;
  DecPlan p = {};
  const int row_bytes = K / 4;
  const int max_chunk = ffn ? 1024 : 2048;
  p.n_chunks = (row_bytes + max_chunk - 1) / max_chunk;
  p.chunk_bytes = ((row_bytes + p.n_chunks - 1) / p.n_chunks + 63) / 64 * 64;
  p.n_chunks = (row_bytes + p.chunk_bytes - 1) / p.chunk_bytes;
  p.row_stride = p.chunk_bytes + DEC_ROW_PAD;
  p.stage_bytes = GEMV_ROWS * p.row_stride * NT;
  int g = n_tiles < sms ? n_tiles : sms;
  const int need = (n_tiles + DEC_MAX_TILES_CTA - 1) / DEC_MAX_TILES_CTA;
  if (g < need) g = need;
  *grid = g;
  p.acc_tiles = (n_tiles + g - 1) / g;
  const int stages_cta = p.acc_tiles * p.n_chunks;
  int slots = (110 * 1024) / p.stage_bytes;
  if (slots < 2) slots = 2;
  if (slots > stages_cta) slots = stages_cta;
  if (slots > 16) slots = 16;
  p.n_slots = slots;
  p.smem_bytes = p.n_slots * p.stage_bytes + 16 * p.n_slots + p.acc_tiles * NT * 256 * 4;
  return p;
}

}  // namespace bitnet

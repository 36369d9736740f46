// K-pre: the BitLinear product for many tokens (prefill) on the 5th-generation tensor
// cores: tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Arithmetic ("fix: I2_S ARM kernel layout + squared-ReLU FFN", bullet "I2_S NEON kernel
// for the canonical layout"): D[n, t] = sum_k c[n, k] q[t, k] with the 2-bit codes
// c = w + 1 expanded to u8, then acc = D - sum_q[t] and out = fp32(acc) * (beta / s_x[t]).
//
// One CTA per SM, persistent over output tiles of 128 weight rows (MMA M, one TMEM lane
// per row) x BN tokens (MMA N, TMEM columns), K in blocks of 128 in-features:
//   warp 4      TMA producer: per k-block, the BN x 128 int8 activation tile
//               (128-byte swizzle, the UMMA K-major canonical layout) and the 128 x 32
//               byte packed weight tile of each tensor;
//   warps 6-13  expanders: two threads per row turn the row's 32 packed bytes into 128 u8
//               codes and write them in the same swizzled K-major layout: field g of packed words
//               4h..4h+3 is exactly the 16-byte chunk 2g + h (in-features 32g + 16h ..
//               +15), placed at chunk position (2g + h) ^ (r % 8);
//   warp 5      MMA issuer: allocates TMEM, issues 4 MMAs (K = 32 each) per k-block and
//               tensor, commits each stage back to the producer and each finished
//               accumulator to the epilogue; two accumulator buffers, so the epilogue of
//               one tile overlaps the MMAs of the next;
//   warps 0-3   epilogue: tcgen05.ld of their 32-lane quarter, activation-sum
//               correction, dequantisation and the bf16/fp32 store (or, for the FFN,
//               h = act(g) * u from the gate and up accumulators of the same tile).
// All waits are bounded; a wait that gives up sets the device status word to
// BITNET_ERR_TIMEOUT, every role leaves its loop, and TMEM is released before exit.
// No load uses cluster multicast.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int TC_BM = 128;
constexpr int TC_BK = 128;
constexpr int TC_EXP_WARPS = 8;     // warps 6-13: two threads per tile row
constexpr int TC_EXP_PARTS = TC_EXP_WARPS * 32 / 128;  // threads per tile row
constexpr int TC_FPP = 4 / TC_EXP_PARTS;               // 2-bit fields per thread
static_assert(TC_EXP_PARTS * TC_FPP == 4, "the expander threads split a row's four fields");
constexpr int TC_THREADS = (6 + TC_EXP_WARPS) * 32;
constexpr int TC_EPI_WARPS = 4;      // warps 0-3
constexpr int TC_TMA_WARP = 4;
constexpr int TC_MMA_WARP = 5;
constexpr int TC_EXP_WARP0 = 6;
constexpr int TC_MAX_STAGES = 8;
constexpr int TC_A_BUFS = 3;        // expanded weight tiles in flight (decoupled from the TMA stages)

struct TcTensor {
  const uint8_t* packed;
  void* out;
  int32_t* acc_debug;
  int N;
  int m_tile_begin;
};

struct TcArgs {
  const float* s_x;
  const int32_t* sum_q;
  int T, K, BN;
  int n_tensors;     // plain mode: 1..4 tensors (tiles concatenated); FFN mode: gate, up
  int m_tiles;       // total 128-row tiles over all tensors (FFN: of the gate)
  int tok_tiles;     // ceil(T / BN)
  int stages;
  int out_dtype;
  int act;
  float* h;
  TcTensor t[4];
};

struct alignas(64) TcMaps {
  CUtensorMap act;   // int8 [T, K], box {128, BN}, 128-byte swizzle
  CUtensorMap w[4];  // uint8 [N, K/4], box {32, 128}, no swizzle
};

// ------------------------------------------------------------------ PTX wrappers
BN_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
BN_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

BN_DEV void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
BN_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
BN_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::i8, issued by one thread.
BN_DEV void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` when all previously issued tcgen05.mma of this thread have completed.
BN_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

BN_DEV void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
BN_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory descriptor of a K-major operand tile with 128-byte rows in the
// 128-byte-swizzle canonical layout (8-row atoms of 1024 bytes, stacked every 1024 B).
BN_DEV uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: D s32, A u8 (codes), B s8 (activations), both K-major, M = 128, N = BN.
BN_DEV uint32_t umma_idesc_i8(int bn) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
}
// The FFN's product with the roles swapped: D s32 [128 tokens x 256], A s8 (activations, M = 128
// tokens), B u8 (the gate and up codes of one 128-row tile, stacked: N = 256).  One instruction
// then covers both tensors, and at twice the N each instruction runs long enough for the single
// issuing thread to keep the tensor pipe fed.
BN_DEV uint32_t umma_idesc_i8_ffn() {
  return (2u << 4) | (1u << 7) | (0u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

template <bool FFN>
__global__ void __launch_bounds__(TC_THREADS, 1) k_gemm_tc(const __grid_constant__ TcMaps maps, const TcArgs a) {
  constexpr int NT = FFN ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  volatile __shared__ int s_abort;
  __shared__ int s_issued;  // stages the producer issued (for the drain after an abort)
  __shared__ uint32_t s_tmem;
  __shared__ float s_f[NT][256];
  __shared__ int s_sq[256];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BN = a.BN, S = a.stages, KB = a.K / TC_BK;
  // Shared layout (1024-byte aligned): TC_A_BUFS expanded weight buffers [NT][128 x 128],
  // then S TMA stages of B tile [BN x 128] + packed [NT][128 x 32].  The TMA stages run deeper
  // than the expanded buffers: the operand loads stay ahead of the expansion by S stages.
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t a_bytes = TC_BM * TC_BK, b_bytes = (uint32_t)BN * TC_BK, p_bytes = TC_BM * 32;
  const uint32_t stage_bytes = (b_bytes + NT * p_bytes + 1023u) & ~1023u;
  const uint32_t tma0 = base + TC_A_BUFS * NT * a_bytes;
  auto sA = [&](int xb, int u) { return base + (xb * NT + u) * a_bytes; };
  auto sB = [&](int s) { return tma0 + s * stage_bytes; };
  auto sP = [&](int s, int u) { return tma0 + s * stage_bytes + b_bytes + u * p_bytes; };
  const uint32_t bars = tma0 + S * stage_bytes;
  auto full_tma = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (TC_MAX_STAGES + s); };
  auto full_a = [&](int xb) { return bars + 8u * (2 * TC_MAX_STAGES + xb); };
  auto tm_full = [&](int b) { return bars + 8u * (2 * TC_MAX_STAGES + 2 * TC_A_BUFS + b); };
  auto tm_empty = [&](int b) { return bars + 8u * (2 * TC_MAX_STAGES + 2 * TC_A_BUFS + 2 + b); };
  const uint32_t mma_done = bars + 8u * (2 * TC_MAX_STAGES + 2 * TC_A_BUFS + 4);  // final commit after an abort

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_tma(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int xb = 0; xb < TC_A_BUFS; ++xb) mbar_init(full_a(xb), TC_EXP_WARPS * 32);
    for (int b = 0; b < 2; ++b) {
      mbar_init(tm_full(b), 1);
      mbar_init(tm_empty(b), 128);
    }
    mbar_init(mma_done, 1);
    s_abort = 0;
    s_issued = 0;
    fence_mbar_init();
  }
  if (warp == TC_MMA_WARP) {
    tmem_alloc(smem_addr(&s_tmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  pdl_launch_dependents();

  const int total = a.m_tiles * a.tok_tiles;
  auto tile_coords = [&](int lin, int& ti, int& m0, int& tok0) {
    const int mt = lin / a.tok_tiles;
    tok0 = (lin % a.tok_tiles) * BN;
    ti = 0;
    if (!FFN)
      while (ti + 1 < a.n_tensors && mt >= a.t[ti + 1].m_tile_begin) ++ti;
    m0 = (mt - a.t[ti].m_tile_begin) * TC_BM;
  };

  if (warp == TC_TMA_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();
      int it = 0;
      for (int lin = blockIdx.x; lin < total && !s_abort; lin += gridDim.x) {
        int ti, m0, tok0;
        tile_coords(lin, ti, m0, tok0);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait_bounded(empty(s), ((it / S) & 1) ^ 1)) {
            s_abort = 1;
            break;
          }
          mbar_arrive_expect_tx(full_tma(s), b_bytes + NT * p_bytes);
          tma_load_2d(sB(s), &maps.act, kb * TC_BK, tok0, full_tma(s));
#pragma unroll
          for (int u = 0; u < NT; ++u) tma_load_2d(sP(s, u), &maps.w[FFN ? u : ti], kb * 32, m0, full_tma(s));
          s_issued = it + 1;
        }
      }
    }
  } else if (warp >= TC_EXP_WARP0) {
    // ------------------------------------------------------------ expanders
    // Thread e: row r = e % 128 of the tile, fields 2h and 2h + 1 (h = e / 128), i.e. the
    // 16-byte chunks 4h .. 4h + 3 of the row's 128 u8 codes.
    const int e = threadIdx.x - TC_EXP_WARP0 * 32;
    const int r = e & 127, h = e >> 7;
    int it = 0;
    for (int lin = blockIdx.x; lin < total && !s_abort; lin += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % S, xb = it % TC_A_BUFS;  // TMA stage, expanded buffer
        // Buffer xb was last read by the MMAs of iteration it - TC_A_BUFS, whose commit also
        // completes that iteration's stage barrier: wait for that phase.  The MMAs are at most
        // at iteration it - 1, and the stage's next completion after it - TC_A_BUFS is at
        // it - TC_A_BUFS + S >= it (S >= TC_A_BUFS), so the parity cannot alias.
        const int pv = it - TC_A_BUFS;
        if (!mbar_wait_bounded(full_tma(s), (it / S) & 1) ||
            (pv >= 0 && !mbar_wait_bounded(empty(pv % S), (pv / S) & 1))) {
          s_abort = 1;
          break;
        }
#pragma unroll
        for (int u = 0; u < NT; ++u) {
          // Rows are 32 bytes apart: lanes 4..7 of each quarter-warp read their row's second
          // half first, so the eight 16-byte reads of a quarter-warp cover all banks once.
          const uint32_t sw = (uint32_t)((e >> 2) & 1) * 16u;
          const uint32_t pa = sP(s, u) + r * 32;
          const uint4 f0 = lds128(pa + sw), f1 = lds128(pa + (16u - sw));
          const uint4 w0 = sw ? f1 : f0, w1 = sw ? f0 : f1;
          const uint32_t rowa = sA(xb, u) + r * 128;
#pragma unroll
          for (int gg = 0; gg < TC_FPP; ++gg) {
            const int g = TC_FPP * h + gg;
            const int sh = 6 - 2 * g;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint4 w = hh ? w1 : w0;
              const uint32_t c0 = (w.x >> sh) & 0x03030303u, c1 = (w.y >> sh) & 0x03030303u;
              const uint32_t c2 = (w.z >> sh) & 0x03030303u, c3 = (w.w >> sh) & 0x03030303u;
              const uint32_t chunk = (uint32_t)(2 * g + hh) ^ (uint32_t)(r & 7);
              asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(rowa + chunk * 16), "r"(c0), "r"(c1), "r"(c2),
                           "r"(c3)
                           : "memory");
            }
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        mbar_arrive(full_a(xb));
      }
    }
  } else if (warp == TC_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // One thread runs the whole loop (stage and buffer indices and their barrier parities kept
    // incrementally): between two k-blocks it has only the waits and a commit to do, so the
    // tensor pipe's queue does not run dry.
    if (lane == 0) {
      const uint32_t idesc = FFN ? umma_idesc_i8_ffn() : umma_idesc_i8(BN);
      int s = 0, xb = 0, tcount = 0;
      uint32_t ph_s = 0, ph_x = 0;
      bool ok = true;
      for (int lin = blockIdx.x; ok && lin < total && !s_abort; lin += gridDim.x, ++tcount) {
        const int ab = tcount & 1;
        if (!mbar_wait_bounded(tm_empty(ab), ((tcount >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(ab * NT * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(full_a(xb), ph_x) || !mbar_wait_bounded(full_tma(s), ph_s)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (FFN) {
            // D[token][gate row | up row]: A = the activation tile, B = both expanded code tiles
            // (sA(xb, 0) and sA(xb, 1) are adjacent: 256 rows in the same swizzled layout).
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_i8(dcol, umma_desc_sw128(sB(s) + 32 * kk), umma_desc_sw128(sA(xb, 0) + 32 * kk), idesc,
                      (kb | kk) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_i8(dcol, umma_desc_sw128(sA(xb, 0) + 32 * kk), umma_desc_sw128(sB(s) + 32 * kk), idesc,
                      (kb | kk) ? 1u : 0u);
          }
          umma_commit(empty(s));  // frees the TMA stage and (to the expanders) the expanded buffer
          if (kb == KB - 1) umma_commit(tm_full(ab));
          if (++s == S) {
            s = 0;
            ph_s ^= 1u;
          }
          if (++xb == TC_A_BUFS) {
            xb = 0;
            ph_x ^= 1u;
          }
        }
      }
      if (!ok) s_abort = 1;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    pdl_wait();
    const int et = threadIdx.x;  // 0..127 = TMEM lane = row of the tile
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int tcount = 0;
    // The four epilogue warps leave the loop together (named-barrier consensus), so
    // none of them is left waiting at a named barrier.
    for (int lin = blockIdx.x; lin < total; lin += gridDim.x, ++tcount) {
      if (named_sync_or(1, 128, s_abort != 0)) break;
      int ti, m0, tok0;
      tile_coords(lin, ti, m0, tok0);
      const int ab = tcount & 1;
      const int N = a.t[ti].N;
      const long long row_bytes = a.K >> 2;
      if (FFN) {
        // Swapped roles: TMEM lane = token tok0 + et, columns [0, 128) gate and [128, 256) up of
        // weight rows m0 .. m0 + 127; this thread writes 16 consecutive h values per chunk.
        const int t = tok0 + et;
        const bool tok_ok = t < a.T;
        const float sx = (tok_ok && a.s_x != nullptr) ? __ldg(a.s_x + t) : 1.0f;
        const int sq = tok_ok ? __ldg(a.sum_q + t) : 0;
        const float betaG = __ldg(reinterpret_cast<const float*>(a.t[0].packed + (long long)N * row_bytes));
        const float betaU = __ldg(reinterpret_cast<const float*>(a.t[1].packed + (long long)N * row_bytes));
        const float fG = __fdiv_rn(betaG, sx), fU = __fdiv_rn(betaU, sx);
        const bool ok = mbar_wait_bounded(tm_full(ab), (tcount >> 1) & 1);
        tc_fence_after();
        for (int c0 = 0; ok && c0 < TC_BM; c0 += 16) {
          uint32_t vg[16], vu[16];
          tmem_ld16(tmem + lane_base + (uint32_t)(ab * 256 + c0), vg);
          tmem_ld16(tmem + lane_base + (uint32_t)(ab * 256 + TC_BM + c0), vu);
          tmem_wait_ld();
          if (c0 + 16 >= TC_BM) {
            tc_fence_before();
            mbar_arrive(tm_empty(ab));  // accumulator may be overwritten now
          }
          if (!tok_ok || m0 + c0 >= N) continue;
          float hv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            hv[j] = ffn_act(dequant((int)vg[j] - sq, fG), dequant((int)vu[j] - sq, fU), a.act);
          float4* dst = reinterpret_cast<float4*>(a.h + (long long)t * N + m0 + c0);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_float4(hv[4 * j], hv[4 * j + 1], hv[4 * j + 2], hv[4 * j + 3]);
        }
        if (named_sync_or(1, 128, !ok)) {
          s_abort = 1;
          break;
        }
        continue;
      }
      // Per-token factors of this tile: beta / s_x and the activation sum.
      for (int j = et; j < BN; j += 128) {
        const int t = tok0 + j;
        const float sx = (t < a.T && a.s_x != nullptr) ? __ldg(a.s_x + t) : 1.0f;  // absent: accumulators only
#pragma unroll
        for (int u = 0; u < NT; ++u) {
          const uint8_t* pk = a.t[FFN ? u : ti].packed;
          const float beta = __ldg(reinterpret_cast<const float*>(pk + (long long)N * row_bytes));
          s_f[u][j] = __fdiv_rn(beta, sx);
        }
        s_sq[j] = t < a.T ? __ldg(a.sum_q + t) : 0;
      }
      named_sync(1, 128);
      const bool ok = mbar_wait_bounded(tm_full(ab), (tcount >> 1) & 1);
      tc_fence_after();
      const int n = m0 + et;
      const bool row_ok = n < N;
      for (int c0 = 0; ok && c0 < BN; c0 += 16) {
        uint32_t va[16], vu[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(ab * NT * BN + c0), va);
        if (FFN) tmem_ld16(tmem + lane_base + (uint32_t)(ab * NT * BN + BN + c0), vu);
        tmem_wait_ld();
        if (c0 + 16 >= BN) {
          tc_fence_before();
          mbar_arrive(tm_empty(ab));  // accumulator may be overwritten now
        }
        if (!row_ok) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = tok0 + c0 + j;
          if (t >= a.T) break;
          const int accA = (int)va[j] - s_sq[c0 + j];
          const float vA = dequant(accA, s_f[0][c0 + j]);
          if (FFN) {
            const int accU = (int)vu[j] - s_sq[c0 + j];
            const float vU = dequant(accU, s_f[1][c0 + j]);
            a.h[(long long)t * N + n] = ffn_act(vA, vU, a.act);
          } else {
            if (a.t[ti].out) store_out(a.t[ti].out, a.out_dtype, (long long)t * N + n, vA);
            if (a.t[ti].acc_debug) a.t[ti].acc_debug[(long long)t * N + n] = accA;
          }
        }
      }
      if (named_sync_or(1, 128, !ok)) {  // s_f / s_sq are rewritten for the next tile
        s_abort = 1;
        break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (s_abort) {
    // After an abort: let every issued MMA finish (a final commit covers all of them) and
    // every issued TMA copy land in this CTA's shared memory before TMEM is released and
    // the CTA exits (fixed drain limit).
    if (warp == TC_MMA_WARP && lane == 0) {
      umma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
    if (warp == TC_TMA_WARP && lane == 0) {
      const int issued = s_issued;
      for (int k = (issued > S ? issued - S : 0); k < issued; ++k) mbar_drain(full_tma(k % S), (uint32_t)((k / S) & 1));
    }
  }
  __syncthreads();
  if (warp == TC_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bitnet

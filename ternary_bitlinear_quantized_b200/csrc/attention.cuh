// The attention between a decoder block's q/k/v and o projections, for decode (a few new
// tokens against a KV cache).  The BitNet pages keep the transformer's attention and only
// replace its linear layers ("Add BitNet" in flash-linear-attention: the transformer code
// with nn.Linear swapped for BitLinear; "More BitNet-like IQ1_S quantizations": the per-block
// attn_q / attn_k / attn_v / attn_output tensors), so this is the textbook computation:
//   rotary embedding   (x_i, x_{i+d/2}) -> (x_i cos a - x_{i+d/2} sin a, x_{i+d/2} cos a + x_i sin a),
//                      a = p * theta^(-2i/d), on q and k at token position p;
//   attention          out = softmax(q . k / sqrt(d)) v over cache rows 0..p (causal), query
//                      head h reading key/value head h / (Hq / Hkv).
// Head size d = 128.  Everything is fp32 on the GPU (angles and their sine and cosine in
// fp64); the KV cache holds bf16 [Hkv][L_max][128].
//
// The attention is split over the cache: k_attn_partial handles one key/value head and
// ATT_CHUNK cache rows for all query rows of that head (T tokens x Hq/Hkv heads), keeping
// the chunk's running maximum, exponent sum and weighted value sum; k_attn_combine merges
// the chunks of each query row.  It is bound by the cache read (2 x 256 bytes per row and
// head).
#pragma once
#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int ATT_D = 128;
constexpr int ATT_CHUNK = 64;                  // cache rows per CTA
constexpr int ATT_THREADS = 256;
constexpr int ATT_MAX_ROWS = 128;              // query rows per key/value head (T x Hq/Hkv)
constexpr int ATT_KP = ATT_D + 4;              // fp32 pitch of a staged key/value row (bank spread)

// ------------------------------------------------------------------ rotary embedding + append
// One thread per (token, head, i < d/2) of q, k and v.  q_out fp32 [T, Hq, d]; the rotated k
// and v go to cache rows pos0 + t (bf16, nearest even).
template <typename TIn>
__global__ void __launch_bounds__(256) k_rope_append(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                     const TIn* __restrict__ v, int T, int Hq, int Hkv, long long pos0,
                                                     double theta, float* __restrict__ q_out,
                                                     __nv_bfloat16* __restrict__ k_cache,
                                                     __nv_bfloat16* __restrict__ v_cache, long long L_max) {
  pdl_launch_dependents();
  pdl_wait();
  const int half = ATT_D / 2;
  const long long total = (long long)T * (Hq + 2 * Hkv) * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx % half);
    const long long th = idx / half;
    const int hh = (int)(th % (Hq + 2 * Hkv));
    const int t = (int)(th / (Hq + 2 * Hkv));
    const long long p = pos0 + t;
    auto ld = [](const TIn* base, long long off) -> float {
      if constexpr (sizeof(TIn) == 2) return bf16_to_f32(reinterpret_cast<const uint16_t*>(base)[off]);
      else return reinterpret_cast<const float*>(base)[off];
    };
    if (hh >= Hq + Hkv) {  // v: copied
      const int h = hh - Hq - Hkv;
      const long long src = ((long long)t * Hkv + h) * ATT_D;
      const long long dst = ((long long)h * L_max + p) * ATT_D;
      v_cache[dst + i] = __float2bfloat16_rn(ld(v, src + i));
      v_cache[dst + i + half] = __float2bfloat16_rn(ld(v, src + i + half));
      continue;
    }
    // a = p theta^(-2i/d) in fp64; sine and cosine in fp64, rounded to fp32
    const double inv_freq = pow(theta, -2.0 * (double)i / (double)ATT_D);
    double sd, cd;
    sincos((double)p * inv_freq, &sd, &cd);
    const float s = __double2float_rn(sd), c = __double2float_rn(cd);
    if (hh < Hq) {
      const long long off = ((long long)t * Hq + hh) * ATT_D;
      const float x1 = ld(q, off + i), x2 = ld(q, off + i + half);
      q_out[off + i] = __fsub_rn(__fmul_rn(x1, c), __fmul_rn(x2, s));
      q_out[off + i + half] = __fadd_rn(__fmul_rn(x2, c), __fmul_rn(x1, s));
    } else {
      const int h = hh - Hq;
      const long long off = ((long long)t * Hkv + h) * ATT_D;
      const float x1 = ld(k, off + i), x2 = ld(k, off + i + half);
      const long long dst = ((long long)h * L_max + p) * ATT_D;
      k_cache[dst + i] = __float2bfloat16_rn(__fsub_rn(__fmul_rn(x1, c), __fmul_rn(x2, s)));
      k_cache[dst + i + half] = __float2bfloat16_rn(__fadd_rn(__fmul_rn(x2, c), __fmul_rn(x1, s)));
    }
  }
}

// Dynamic shared memory of k_attn_partial for R query rows.
BN_HOST_DEV inline size_t attn_partial_smem(int R) {
  return ((size_t)R * ATT_KP + 2 * ATT_CHUNK * ATT_KP + (size_t)R * ATT_CHUNK) * sizeof(float);
}

// ------------------------------------------------------------------ attention, one chunk
// Partial result of query row j (token t = j / G, head kv * G + j % G) over cache rows
// [c0, c1): m = max score, l = sum exp(score - m), o[d] = sum exp(score - m) v[d].
// Layout of the partials: [chunk][kv][row] x (ATT_D + 2) floats (o, then m, l).
__global__ void __launch_bounds__(ATT_THREADS) k_attn_partial(const float* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                                                              const __nv_bfloat16* __restrict__ vc, int T, int Hq,
                                                              int Hkv, long long pos0, long long L_max,
                                                              float* __restrict__ part) {
  extern __shared__ float att_sm[];
  const int G = Hq / Hkv, R = T * G;
  const int chunk = blockIdx.x, kv = blockIdx.y;
  const long long L = pos0 + T;  // cache rows in use
  const long long c0 = (long long)chunk * ATT_CHUNK;
  const int n = (int)min((long long)ATT_CHUNK, L - c0);
  float* Qs = att_sm;                              // [R][ATT_KP]
  float* Ks = Qs + R * ATT_KP;                     // [ATT_CHUNK][ATT_KP]
  float* Vs = Ks + ATT_CHUNK * ATT_KP;             // [ATT_CHUNK][ATT_KP]
  float* Ss = Vs + ATT_CHUNK * ATT_KP;             // [R][ATT_CHUNK] scores, then weights
  __shared__ float s_m[ATT_MAX_ROWS], s_l[ATT_MAX_ROWS];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x;
  // stage q rows (fp32) and the chunk's keys and values (bf16 -> fp32), 16 bytes at a time
  for (int i = tid; i < R * (ATT_D / 4); i += ATT_THREADS) {
    const int j = i / (ATT_D / 4), d4 = (i % (ATT_D / 4)) * 4;
    const int t = j / G, h = kv * G + j % G;
    *reinterpret_cast<float4*>(Qs + j * ATT_KP + d4) =
        __ldg(reinterpret_cast<const float4*>(q + ((long long)t * Hq + h) * ATT_D + d4));
  }
  // every thread issues all of its 16-byte loads first (one memory round trip), then widens
  constexpr int KV_LOADS = 2 * ATT_CHUNK * (ATT_D / 8) / ATT_THREADS;
  static_assert(KV_LOADS * ATT_THREADS == 2 * ATT_CHUNK * (ATT_D / 8), "whole loads per thread");
  uint4 w[KV_LOADS];
#pragma unroll
  for (int j = 0; j < KV_LOADS; ++j) {
    const int i = tid + j * ATT_THREADS;
    const int which = i / (ATT_CHUNK * (ATT_D / 8)), rem = i % (ATT_CHUNK * (ATT_D / 8));
    const int p = rem / (ATT_D / 8), d8 = (rem % (ATT_D / 8)) * 8;
    w[j] = make_uint4(0u, 0u, 0u, 0u);
    if (p < n) w[j] = __ldg(reinterpret_cast<const uint4*>((which ? vc : kc) + ((long long)kv * L_max + c0 + p) * ATT_D + d8));
  }
#pragma unroll
  for (int j = 0; j < KV_LOADS; ++j) {
    const int i = tid + j * ATT_THREADS;
    const int which = i / (ATT_CHUNK * (ATT_D / 8)), rem = i % (ATT_CHUNK * (ATT_D / 8));
    const int p = rem / (ATT_D / 8), d8 = (rem % (ATT_D / 8)) * 8;
    float* dst = (which ? Vs : Ks) + p * ATT_KP + d8;
    const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dst[2 * e] = __uint_as_float(ww[e] << 16);
      dst[2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
    }
  }
  __syncthreads();
  // scores: thread = (row group rg, cache row p); rows rg, rg + 4, ...
  const float scale = __fdiv_rn(1.0f, __fsqrt_rn((float)ATT_D));
  {
    const int p = tid % ATT_CHUNK, rg = tid / ATT_CHUNK;
    const float* kr = Ks + p * ATT_KP;
    for (int j = rg; j < R; j += ATT_THREADS / ATT_CHUNK) {
      const float* qr = Qs + j * ATT_KP;
      // four independent partial sums (short dependency chains), added at the end
      float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll 8
      for (int d = 0; d < ATT_D; d += 4) {
        const float4 a = *reinterpret_cast<const float4*>(qr + d), b = *reinterpret_cast<const float4*>(kr + d);
        a0 = __fadd_rn(a0, __fmul_rn(a.x, b.x));
        a1 = __fadd_rn(a1, __fmul_rn(a.y, b.y));
        a2 = __fadd_rn(a2, __fmul_rn(a.z, b.z));
        a3 = __fadd_rn(a3, __fmul_rn(a.w, b.w));
      }
      const float acc = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
      const long long qpos = pos0 + j / G;
      Ss[j * ATT_CHUNK + p] = (p < n && c0 + p <= qpos) ? __fmul_rn(acc, scale) : -INFINITY;
    }
  }
  __syncthreads();
  // per row: max, weights, sum (a warp per row)
  {
    const int w = tid >> 5, lane = tid & 31;
    for (int j = w; j < R; j += ATT_THREADS / 32) {
      float* sr = Ss + j * ATT_CHUNK;
      float m = -INFINITY;
      for (int p = lane; p < ATT_CHUNK; p += 32) m = fmaxf(m, sr[p]);
      m = warp_max(m);
      float l = 0.0f;
      for (int p = lane; p < ATT_CHUNK; p += 32) {
        const float e = (m == -INFINITY || sr[p] == -INFINITY) ? 0.0f : expf(__fsub_rn(sr[p], m));
        sr[p] = e;
        l = __fadd_rn(l, e);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, o));
      if (lane == 0) {
        s_m[j] = m;
        s_l[j] = l;
      }
    }
  }
  __syncthreads();
  // weighted values: thread = (row half, dim)
  {
    const int d = tid % ATT_D, rh = tid / ATT_D;
    for (int j = rh; j < R; j += ATT_THREADS / ATT_D) {
      const float* sr = Ss + j * ATT_CHUNK;
      float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
      int p = 0;
      for (; p + 3 < n; p += 4) {
        a0 = __fadd_rn(a0, __fmul_rn(sr[p], Vs[p * ATT_KP + d]));
        a1 = __fadd_rn(a1, __fmul_rn(sr[p + 1], Vs[(p + 1) * ATT_KP + d]));
        a2 = __fadd_rn(a2, __fmul_rn(sr[p + 2], Vs[(p + 2) * ATT_KP + d]));
        a3 = __fadd_rn(a3, __fmul_rn(sr[p + 3], Vs[(p + 3) * ATT_KP + d]));
      }
      for (; p < n; ++p) a0 = __fadd_rn(a0, __fmul_rn(sr[p], Vs[p * ATT_KP + d]));
      const float acc = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
      float* dst = part + (((long long)chunk * Hkv + kv) * R + j) * (ATT_D + 2);
      dst[d] = acc;
      if (d == 0) {
        dst[ATT_D] = s_m[j];
        dst[ATT_D + 1] = s_l[j];
      }
    }
  }
}

// Merge the chunks of each query row: out = (sum_c o_c e^(m_c - M)) / (sum_c l_c e^(m_c - M)).
// The chunk maxima and factors go through shared memory (each loaded once, all chunks at once
// across the 128 threads); every thread then sums its dimension over the chunks with eight
// loads in flight, so the merge costs a few memory round trips instead of one per chunk.
constexpr int ATT_MAX_CHUNKS = 1024;  // cache rows up to 64 Ki
__global__ void __launch_bounds__(ATT_D) k_attn_combine(const float* __restrict__ part, int T, int Hq, int Hkv,
                                                        int n_chunks, void* __restrict__ out, int out_dtype) {
  __shared__ float s_f[ATT_MAX_CHUNKS];
  __shared__ float s_red[ATT_D / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int G = Hq / Hkv, R = T * G;
  const int row = blockIdx.x;  // (t, h)
  const int t = row / Hq, h = row % Hq, kv = h / G, j = t * G + (h % G);
  const int d = threadIdx.x, lane = d & 31, w = d >> 5;
  auto pc = [&](int c) { return part + (((long long)c * Hkv + kv) * R + j) * (ATT_D + 2); };
  float M = -INFINITY;
  for (int c = d; c < n_chunks; c += ATT_D) {
    const float m = pc(c)[ATT_D];
    s_f[c] = m;
    M = fmaxf(M, m);
  }
  M = warp_max(M);
  if (lane == 0) s_red[w] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  __syncthreads();
  float L = 0.0f;
  for (int c = d; c < n_chunks; c += ATT_D) {
    const float m = s_f[c];
    const float f = m == -INFINITY ? 0.0f : expf(__fsub_rn(m, M));
    s_f[c] = f;
    L = __fadd_rn(L, __fmul_rn(pc(c)[ATT_D + 1], f));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L = __fadd_rn(L, __shfl_xor_sync(0xffffffffu, L, o));
  if (lane == 0) s_red[w] = L;
  __syncthreads();
  L = __fadd_rn(__fadd_rn(s_red[0], s_red[1]), __fadd_rn(s_red[2], s_red[3]));
  float O = 0.0f;
  int c = 0;
  for (; c + 7 < n_chunks; c += 8) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = pc(c + k)[d];
#pragma unroll
    for (int k = 0; k < 8; ++k) O = __fadd_rn(O, __fmul_rn(v[k], s_f[c + k]));
  }
  for (; c < n_chunks; ++c) O = __fadd_rn(O, __fmul_rn(pc(c)[d], s_f[c]));
  store_out(out, out_dtype, (long long)row * ATT_D + d, __fdiv_rn(O, L));
}

}  // namespace bitnet

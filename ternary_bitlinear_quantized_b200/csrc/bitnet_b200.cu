// The C ABI of include/bitnet_b200.h: argument checks, launch configuration and the
// order of launches on the caller's stream.  Every step of the arithmetic runs in the
// kernels of quant.cuh, pack.cuh, engine.cuh and gemm_tc.cuh (one translation unit, so
// that the device status word needs no relocatable device code).
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <algorithm>
#include <string>

#include "common.cuh"
#include "quant.cuh"
#include "pack.cuh"
#include "gemv.cuh"
#include "engine.cuh"
#include "gemm_tc.cuh"
#include "shard.cuh"
#include "attention.cuh"

namespace bitnet {

static thread_local std::string t_last_error;

static bitnet_status cuda_fail(cudaError_t e, const char* where) {
  t_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return BITNET_ERR_CUDA;
}

#define BN_CUDA(call, where)                        \
  do {                                              \
    cudaError_t _e = (call);                        \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic stream serialisation: the kernel may begin while the
// previous kernel on the stream is still running; it calls griddepcontrol.wait before
// reading anything that kernel produced.
template <typename... KArgs, typename... Args>
static cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

static int device_sm_count() {
  static thread_local int cached_dev = -1, cached_sms = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != cached_dev) {
    cudaDeviceGetAttribute(&cached_sms, cudaDevAttrMultiProcessorCount, dev);
    cached_dev = dev;
  }
  return cached_sms > 0 ? cached_sms : 148;
}

// Opt a kernel in to the full dynamic shared memory of the SM, once per device.  The
// "done" flags are atomics: several host threads may race to set the same attribute, which
// is harmless (the same value), and none of them reads a torn flag.
static cudaError_t opt_in_smem(const void* kern, int slot) {
  static std::atomic<int> done[16][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::atomic<int>& d = done[slot & 15][dev & 63];
  if (d.load(std::memory_order_acquire)) return cudaSuccess;
  int max_optin = 0;
  cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_optin - (int)fa.sharedSizeBytes);
  if (e == cudaSuccess) d.store(1, std::memory_order_release);
  return e;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (a function-local static is initialised
// exactly once even when several threads call this at the same time).
static EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// 2-D byte tensor [rows, cols] (row stride `stride` bytes) with a box of box_cols x box_rows.
static bool make_map_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t stride,
                        uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ quant
static bitnet_status enqueue_quant(const void* x, bitnet_dtype xt, const float* gain, float eps, int64_t T, int64_t K,
                                   int8_t* q, float* s_x, int32_t* sum_q, cudaStream_t s) {
  if (T == 0) return BITNET_OK;
  // Rows of up to 8192 values (K a multiple of 8, 16-byte aligned rows): values in registers,
  // one to four warps per row; four when there are too few rows to fill the GPU, so each
  // row's reductions are short.
  const size_t esz_r = xt == BITNET_BF16 ? 2 : 4;
  if (K <= 4 * 2048 && K % 8 == 0 && aligned16(x) && aligned16(q) && (K * esz_r) % 16 == 0) {
    const int w = (T <= 256 || K > 4096) ? 4 : (K <= 2048 ? 1 : 2);
    const unsigned grid = (unsigned)((T + QW_THREADS / 32 / w - 1) / (QW_THREADS / 32 / w));
    cudaError_t e;
    if (xt == BITNET_BF16) {
      auto* kern = w == 1 ? k_rmsnorm_quant_warps<__nv_bfloat16, 1>
                          : (w == 2 ? k_rmsnorm_quant_warps<__nv_bfloat16, 2> : k_rmsnorm_quant_warps<__nv_bfloat16, 4>);
      e = launch(kern, dim3(grid), dim3(QW_THREADS), 0, s, true, reinterpret_cast<const __nv_bfloat16*>(x), gain, eps,
                 (int)T, (int)K, q, s_x, sum_q);
    } else {
      auto* kern = w == 1 ? k_rmsnorm_quant_warps<float, 1>
                          : (w == 2 ? k_rmsnorm_quant_warps<float, 2> : k_rmsnorm_quant_warps<float, 4>);
      e = launch(kern, dim3(grid), dim3(QW_THREADS), 0, s, true, reinterpret_cast<const float*>(x), gain, eps, (int)T,
                 (int)K, q, s_x, sum_q);
    }
    if (e != cudaSuccess) return cuda_fail(e, "k_rmsnorm_quant_warps");
    return BITNET_OK;
  }
  // Long fp32 rows, many of them (the FFN's h at prefill): persistent, double-buffered.
  if (xt == BITNET_F32 && K % 4 == 0 && 2 * K * 4 <= 227 * 1024 - 1024 && K <= 4 * QL_THREADS * QL_MAXV &&
      T >= 2 * device_sm_count() && aligned16(x) && aligned16(q)) {
    const size_t smem_l = (size_t)2 * K * 4;
    static std::atomic<int> long_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!long_done[dev & 63].load(std::memory_order_acquire)) {
      cudaError_t ea = cudaFuncSetAttribute(k_rmsnorm_quant_long, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            227 * 1024 - 1024);
      if (ea != cudaSuccess) return cuda_fail(ea, "quant attribute (long rows)");
      long_done[dev & 63].store(1, std::memory_order_release);
    }
    const int sms = device_sm_count();
    cudaError_t el = launch(k_rmsnorm_quant_long, dim3((unsigned)(T < sms ? T : sms)), dim3(QL_THREADS), smem_l, s,
                            true, reinterpret_cast<const float*>(x), gain, eps, (int)T, (int)K, q, s_x, sum_q);
    if (el != cudaSuccess) return cuda_fail(el, "k_rmsnorm_quant_long");
    return BITNET_OK;
  }
  int threads = (int)((K / 8 + 31) / 32 * 32);
  threads = threads < 128 ? 128 : (threads > 1024 ? 1024 : threads);
  const size_t smem = (size_t)K * sizeof(float);
  const size_t esz = xt == BITNET_BF16 ? 2 : 4;
  const int vec = (K % 8 == 0) && aligned16(x) && aligned16(q) && ((K * esz) % 16 == 0);
  cudaError_t e;
  if (smem > 48 * 1024) {
    // Opt in to the large dynamic shared memory once per device and kernel.
    static std::atomic<int> done_mask[2][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    std::atomic<int>& done = done_mask[xt == BITNET_BF16 ? 0 : 1][dev & 63];
    if (!done.load(std::memory_order_acquire)) {
      e = xt == BITNET_BF16 ? cudaFuncSetAttribute(k_rmsnorm_quant<__nv_bfloat16>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, BITNET_MAX_K * 4)
                            : cudaFuncSetAttribute(k_rmsnorm_quant<float>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, BITNET_MAX_K * 4);
      if (e != cudaSuccess) return cuda_fail(e, "quant attribute");
      done.store(1, std::memory_order_release);
    }
  }
  if (xt == BITNET_BF16) {
    e = launch(k_rmsnorm_quant<__nv_bfloat16>, dim3((unsigned)T), dim3(threads), smem, s, true,
               reinterpret_cast<const __nv_bfloat16*>(x), gain, eps, (int)K, q, s_x, sum_q, vec);
  } else {
    e = launch(k_rmsnorm_quant<float>, dim3((unsigned)T), dim3(threads), smem, s, true,
               reinterpret_cast<const float*>(x), gain, eps, (int)K, q, s_x, sum_q, vec);
  }
  if (e != cudaSuccess) return cuda_fail(e, "k_rmsnorm_quant");
  return BITNET_OK;
}

// ------------------------------------------------------------------ product
// Prefill: the tcgen05 kernel, from the same arguments as the decode kernel.
static bitnet_status enqueue_gemm_tc(const GemvArgs& g, bool ffn, cudaStream_t s) {
  const int NT = ffn ? 2 : 1;
  TcArgs a = {};
  a.s_x = g.s_x;
  a.sum_q = g.sum_q;
  a.T = g.T;
  a.K = g.K;
  // Token-tile width: the candidate that minimises waves x (BN + per-tile overhead), so
  // that the last wave of 128-row tiles is not left nearly empty.
  {
    int m_tiles = 0;
    for (int i = 0; i < g.n_tensors; ++i)
      if (!ffn || i == 0) m_tiles += (g.t[i].N + TC_BM - 1) / TC_BM;
    const int sms_ = device_sm_count();
    const int bn_max = ffn ? 128 : 256;
    const int cands[4] = {256, 192, 128, 64};
    long best = -1;
    int best_bn = 64;
    for (int c : cands) {
      int bn = c;
      const int tfit = (g.T + 15) / 16 * 16;
      if (bn > bn_max) continue;
      if (bn > tfit) bn = tfit;
      const long tiles = (long)m_tiles * ((g.T + bn - 1) / bn);
      const long waves = (tiles + sms_ - 1) / sms_;
      const long cost = waves * (bn + 48);
      if (best < 0 || cost < best) {
        best = cost;
        best_bn = bn;
      }
    }
    // The FFN product runs with the roles swapped (128 tokens as the MMA's M): BN = 128.
    a.BN = ffn ? TC_BM : best_bn;
  }
  a.n_tensors = g.n_tensors;
  a.out_dtype = g.out_dtype;
  a.act = g.act;
  a.h = g.h;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_map_u8(&maps.act, g.q, (uint64_t)g.K, (uint64_t)g.T, (uint64_t)g.K, TC_BK, (uint32_t)a.BN, true))
    return cuda_fail(cudaErrorInvalidValue, "tensor map (activations)");
  int mt = 0;
  for (int i = 0; i < g.n_tensors; ++i) {
    a.t[i].packed = g.t[i].packed;
    a.t[i].out = g.t[i].out;
    a.t[i].acc_debug = g.t[i].acc_debug;
    a.t[i].N = g.t[i].N;
    a.t[i].m_tile_begin = mt;
    if (!ffn || i == 0) mt += (g.t[i].N + TC_BM - 1) / TC_BM;
    if (!make_map_u8(&maps.w[i], g.t[i].packed, (uint64_t)(g.K / 4), (uint64_t)g.t[i].N, (uint64_t)(g.K / 4), 32,
                     TC_BM, false))
      return cuda_fail(cudaErrorInvalidValue, "tensor map (weights)");
  }
  a.m_tiles = mt;
  a.tok_tiles = (g.T + a.BN - 1) / a.BN;
  // TMA stages (B tile + packed weights) after TC_A_BUFS expanded weight buffers.
  const uint32_t stage_bytes = (uint32_t)((a.BN * TC_BK + NT * TC_BM * 32 + 1023) / 1024 * 1024);
  const uint32_t abuf_bytes = (uint32_t)(TC_A_BUFS * NT * TC_BM * TC_BK);
  int dev = 0, max_optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa;
  void (*kern)(const TcMaps, const TcArgs) = ffn ? k_gemm_tc<true> : k_gemm_tc<false>;
  cudaError_t e = cudaFuncGetAttributes(&fa, (const void*)kern);
  if (e != cudaSuccess) return cuda_fail(e, "k_gemm_tc attributes");
  int stages = (int)((max_optin - (int)fa.sharedSizeBytes - 1024 - 256 - (int)abuf_bytes) / (int)stage_bytes);
  if (stages > TC_MAX_STAGES) stages = TC_MAX_STAGES;
  if (stages < TC_A_BUFS) return cuda_fail(cudaErrorInvalidConfiguration, "k_gemm_tc stages");
  a.stages = stages;
  const size_t smem = (size_t)abuf_bytes + (size_t)stages * stage_bytes + 1024 + 256;
  e = opt_in_smem((const void*)kern, 4 + (ffn ? 1 : 0));
  if (e != cudaSuccess) return cuda_fail(e, "k_gemm_tc attribute");
  const int total = a.m_tiles * a.tok_tiles;
  const int sms = device_sm_count();
  e = launch(kern, dim3(total < sms ? total : sms), dim3(TC_THREADS), smem, s, true, maps, a);
  if (e != cudaSuccess) return cuda_fail(e, "k_gemm_tc");
  return BITNET_OK;
}

// ------------------------------------------------------------------ decode engine plans
constexpr int ENG_RING_MAX = 160 * 1024;      // bytes of weights in flight per SM at most
constexpr int ENG_LOCAL_MAX_TK = 16 * 1024;   // T * K up to which every CTA quantises for itself

static EngPhase eng_gemv(int K, bool ffn, int n_tensors, const uint8_t* const* packed, const int64_t* N,
                         void* const* out, int32_t* const* dbg, int out_dtype, int act, float* h) {
  EngPhase p;
  memset(&p, 0, sizeof(p));
  p.kind = ffn ? PH_GEMV_FFN : PH_GEMV;
  p.K = K;
  p.n_tensors = n_tensors;
  int tiles = 0;
  for (int i = 0; i < n_tensors; ++i) {
    p.t[i].packed = packed[i];
    p.t[i].out = out ? out[i] : nullptr;
    p.t[i].acc_debug = dbg ? dbg[i] : nullptr;
    p.t[i].N = (int)N[i];
    p.t[i].tile_begin = tiles;
    if (!ffn || i == 0) tiles += (int)((N[i] + GEMV_ROWS - 1) / GEMV_ROWS);
  }
  p.n_tiles = tiles;
  p.out_dtype = out_dtype;
  p.act = act;
  p.h = h;
  p.wait_barrier = p.arrive_barrier = -1;
  return p;
}

static void eng_src_global(EngPhase& p, const int8_t* q, const float* s, const int32_t* sq) {
  p.src = SRC_GLOBAL;
  p.q = const_cast<int8_t*>(q);
  p.s = const_cast<float*>(s);
  p.sq = const_cast<int32_t*>(sq);
}

static void eng_src_local(EngPhase& p, const void* x, int x_f32, const float* gain, int8_t* q_copy, float* s_copy,
                          int32_t* sq_copy) {
  p.src = SRC_LOCAL;
  p.x = x;
  p.x_f32 = x_f32;
  p.gain = gain;
  p.q = q_copy;
  p.s = s_copy;
  p.sq = sq_copy;
}

static EngPhase eng_quant(const void* x, int x_f32, int K, const float* gain, int8_t* q, float* s, int32_t* sq) {
  EngPhase p;
  memset(&p, 0, sizeof(p));
  p.kind = PH_QUANT;
  p.K = K;
  p.x = x;
  p.x_f32 = x_f32;
  p.gain = gain;
  p.q = q;
  p.s = s;
  p.sq = sq;
  p.wait_barrier = p.arrive_barrier = -1;
  return p;
}

static bool eng_local_ok(int64_t T, int64_t K) { return T * K <= ENG_LOCAL_MAX_TK && K <= ENG_REG_MAX_K; }
static bool eng_quant_ok(int64_t K) { return K <= ENG_LOCAL_MAX_K; }

// Tensor map of an I2_S tensor [N, K] as 8-byte elements [N, K/32], box CB/8 x 16 rows
// (chunked stages of the decode engine).
static bool make_map_u64(CUtensorMap* m, const void* base, uint64_t N, uint64_t K, uint32_t CB) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {K / 32, N};
  const cuuint64_t strides[1] = {K / 4};
  const cuuint32_t box[2] = {CB / 8, (cuuint32_t)GEMV_ROWS};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_INT64, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch the engine over the phases in `a` (a.T, a.eps, a.n_phases, a.ph, a.counters set).
// Balanced tile split (see EngPhase::balanced) of the product phases that run back to back
// from the first one up to the first QUANT or SUBNORM phase (no grid-wide wait between them
// blocks a CTA for long): each phase's n_tiles mod G extra tiles go to the CTAs with the least
// work so far, heaviest phases first, work counted in weight bytes per tile.  A SUBNORM phase
// takes the split of the phase before it (it reduces the rows that phase produced).
static void balance_tiles(EngArgs& a, int grid) {
  int first = 0;
  while (first < a.n_phases && !ph_is_gemv(a.ph[first].kind)) ++first;
  int last = first;
  while (last < a.n_phases && ph_is_gemv(a.ph[last].kind)) ++last;  // [first, last)
  if (last - first >= 2 && grid >= 2 && grid <= ENG_MAX_GRID) {
    int order[ENG_MAX_PHASES], n = 0;
    for (int i = first; i < last; ++i) order[n++] = i;
    auto tile_bytes = [&](const EngPhase& p) {
      return (long long)(p.kind == PH_GEMV_FFN ? 2 : 1) * GEMV_ROWS * (p.K / 4);
    };
    for (int i = 1; i < n; ++i)  // heaviest tiles first (stable)
      for (int j = i; j > 0 && tile_bytes(a.ph[order[j]]) > tile_bytes(a.ph[order[j - 1]]); --j) {
        const int t = order[j];
        order[j] = order[j - 1];
        order[j - 1] = t;
      }
    long long load[ENG_MAX_GRID];
    int idx[ENG_MAX_GRID];
    for (int c = 0; c < grid; ++c) load[c] = 0;
    for (int k = 0; k < n; ++k) {
      EngPhase& p = a.ph[order[k]];
      const int base = p.n_tiles / grid, extra = p.n_tiles % grid;
      for (int c = 0; c < grid; ++c) idx[c] = c;
      std::stable_sort(idx, idx + grid, [&](int x, int y) { return load[x] < load[y]; });
      p.balanced = 1;
      memset(p.xmask, 0, sizeof(p.xmask));
      for (int j = 0; j < extra; ++j) p.xmask[idx[j] >> 5] |= 1u << (idx[j] & 31);
      for (int c = 0; c < grid; ++c)
        load[c] += tile_bytes(p) * (base + (int)((p.xmask[c >> 5] >> (c & 31)) & 1u));
    }
  }
  for (int i = 1; i < a.n_phases; ++i)
    if (a.ph[i].kind == PH_SUBNORM && ph_is_gemv(a.ph[i - 1].kind)) {
      a.ph[i].balanced = a.ph[i - 1].balanced;
      memcpy(a.ph[i].xmask, a.ph[i - 1].xmask, sizeof(a.ph[i].xmask));
    }
}

static bitnet_status enqueue_engine(EngArgs& a, cudaStream_t s) {
  static_assert(sizeof(EngArgs) % 16 == 0, "EngArgs is copied with 16-byte loads");
  const int sms = device_sm_count();
  bool multi = a.n_phases > 1;
  int max_tiles = 1;
  for (int i = 0; i < a.n_phases; ++i)
    if (ph_is_gemv(a.ph[i].kind) && a.ph[i].n_tiles > max_tiles) max_tiles = a.ph[i].n_tiles;
  const int gmax = sms < ENG_MAX_GRID ? sms : ENG_MAX_GRID;  // per-CTA partials are sized for ENG_MAX_GRID
  const int grid = multi ? gmax : (max_tiles < gmax ? max_tiles : gmax);
  balance_tiles(a, grid);
  int acc_ints = 0, qs = 0, xs = 0, slot = 0;
  EngMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int i = 0; i < a.n_phases; ++i) {
    EngPhase& p = a.ph[i];
    if ((p.kind == PH_QUANT || (ph_is_gemv(p.kind) && p.src == SRC_LOCAL)) && p.K > ENG_REG_MAX_K && p.K > xs) xs = p.K;
    if (!ph_is_gemv(p.kind)) continue;
    const int NT = p.kind == PH_GEMV_FFN ? 2 : 1;
    const int per = (p.n_tiles + grid - 1) / grid * NT * GEMV_ROWS * a.T;
    if (per > acc_ints) acc_ints = per;
    if (!eng_plan(p.K, a.T, ENG_SLOT_MAX, ENG_ACT_MAX, p.g))
      return cuda_fail(cudaErrorInvalidConfiguration, "k_engine stage geometry");
    if (p.src == SRC_LOCAL && !p.g.full_rows)  // local quantisation writes whole rows
      return cuda_fail(cudaErrorInvalidConfiguration, "k_engine local activations");
    if (a.T * p.g.x_pitch > qs) qs = a.T * p.g.x_pitch;
    const int sb = (p.g.slot_bytes + 1023) / 1024 * 1024;  // TMA destinations 1024-byte aligned
    if (sb > slot) slot = sb;
    if (!p.g.full_rows)
      for (int u = 0; u < p.n_tensors; ++u)
        if (!make_map_u64(&maps.m[i][u], p.t[u].packed, (uint64_t)p.t[u].N, (uint64_t)p.K, (uint32_t)p.g.CB))
          return cuda_fail(cudaErrorInvalidValue, "tensor map (engine weights)");
  }
  qs = (qs + 127) / 128 * 128;
  // Private accumulator slots per consumer warp when they are small (few tokens): no atomic
  // contention in the flushes; the epilogue sums the slots.
  const int acc_priv = acc_ints * ENG_CONS_WARPS * 4 <= 32 * 1024 ? 1 : 0;
  if (acc_priv) acc_ints *= ENG_CONS_WARPS;
  acc_ints = (acc_ints + 3) / 4 * 4;
  int sub_rows = 0;  // rows of h a CTA keeps for a SUBNORM phase, and their gain
  for (int i = 0; i < a.n_phases; ++i)
    if (a.ph[i].kind == PH_GEMV_FFN && a.ph[i].pmax != nullptr) {
      const int r = (a.ph[i].n_tiles + grid - 1) / grid * GEMV_ROWS;
      if (r > sub_rows) sub_rows = r;
    }
  xs = (xs + 3) / 4 * 4;  // keep what follows 16-byte aligned
  const int sub_floats = (a.T + 1) * sub_rows;
  const int tg = a.T <= 8 ? 1 : 2;
  void (*kern)(const EngArgs, const EngMaps) = tg == 1 ? k_engine<1> : k_engine<2>;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, (const void*)kern);
  if (e != cudaSuccess) return cuda_fail(e, "k_engine attributes");
  int dev = 0;
  cudaGetDevice(&dev);
  int max_optin = 0;
  cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int budget = max_optin - (int)fa.sharedSizeBytes - 1024;  // 1024: ring alignment
  const int ring = budget - acc_ints * 4 - qs - xs * 4 - sub_floats * 4;
  if (slot == 0) slot = 1024;  // no product phase (not planned by this library, but harmless)
  int slots = ring / (slot + 16);
  if (slots * slot > ENG_RING_MAX) slots = ENG_RING_MAX / slot;
  if (slots > ENG_MAX_SLOTS) slots = ENG_MAX_SLOTS;
  if (slots < 2) return cuda_fail(cudaErrorInvalidConfiguration, "k_engine shared memory");
  a.n_slots = slots;
  a.slot_bytes = slot;
  a.acc_ints = acc_ints;
  a.qs_bytes = qs;
  a.xs_floats = xs;
  a.sub_rows = sub_rows;
  a.acc_priv = acc_priv;
  const size_t smem =
      1024 + (size_t)slots * slot + 16 * slots + (size_t)acc_ints * 4 + qs + (size_t)xs * 4 + (size_t)sub_floats * 4;
  e = opt_in_smem((const void*)kern, 6 + tg - 1);
  if (e != cudaSuccess) return cuda_fail(e, "k_engine attribute");
  // Grid barriers need every CTA resident at once: one CTA per SM must fit.
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, ENG_THREADS, smem);
  if (e != cudaSuccess) return cuda_fail(e, "k_engine occupancy");
  if (per_sm < 1 || grid > per_sm * sms) return cuda_fail(cudaErrorCooperativeLaunchTooLarge, "k_engine residency");
  e = launch(kern, dim3(grid), dim3(ENG_THREADS), smem, s, true, a, maps);
  if (e != cudaSuccess) return cuda_fail(e, "k_engine");
  return BITNET_OK;
}

static bitnet_status enqueue_gemv(const int8_t* q, const float* s_x, const int32_t* sum_q, int n_tensors,
                                  const uint8_t* const* packed, const int64_t* N, void* const* out,
                                  int32_t* const* acc_debug, int64_t T, int64_t K, bitnet_dtype ot,
                                  bool ffn, bitnet_act act, float* h, cudaStream_t s) {
  if (T == 0) return BITNET_OK;
  GemvArgs a = {};
  a.q = q;
  a.s_x = s_x;
  a.sum_q = sum_q;
  a.T = (int)T;
  a.K = (int)K;
  a.n_tensors = n_tensors;
  a.out_dtype = ot;
  a.act = act;
  a.h = h;
  int tiles = 0;
  for (int i = 0; i < n_tensors; ++i) {
    a.t[i].packed = packed[i];
    a.t[i].out = out ? out[i] : nullptr;
    a.t[i].acc_debug = acc_debug ? acc_debug[i] : nullptr;
    a.t[i].N = (int)N[i];
    a.t[i].tile_begin = tiles;
    if (!ffn || i == 0) tiles += (int)((N[i] + GEMV_ROWS - 1) / GEMV_ROWS);
  }
  a.n_tiles = tiles;
  if (T <= ENG_MAX_T) {
    EngArgs ea;
    memset(&ea, 0, sizeof(ea));
    ea.T = (int)T;
    ea.n_phases = 1;
    ea.ph[0] = eng_gemv((int)K, ffn, n_tensors, packed, N, out, acc_debug, ot, act, h);
    eng_src_global(ea.ph[0], q, s_x, sum_q);
    return enqueue_engine(ea, s);
  }
  return enqueue_gemm_tc(a, ffn, s);
}

}  // namespace bitnet

using namespace bitnet;

// ====================================================================== C ABI
extern "C" {

size_t bitnet_i2s_packed_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || K % 128 != 0) return 0;
  return (size_t)(N * K / 4 + 32);
}

static bitnet_status enqueue_pack(const float* W, int64_t N, int64_t K, uint8_t* packed, int prescaled,
                                  cudaStream_t s) {
  if (!W || !packed) return BITNET_ERR_NULL;
  if (N <= 0 || K <= 0 || K % 128 != 0 || N * K >= (1ll << 40)) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed)) return BITNET_ERR_ALIGN;
  const long long n = N * K;
  PackScratch* sc = reinterpret_cast<PackScratch*>(packed + n / 4);
  const int sms = device_sm_count();
  long long want = (n / 4 + 255) / 256;
  const unsigned grid = (unsigned)(want < sms * 8 ? want : sms * 8);
  long long wantc = (n / 16 + 255) / 256;
  const unsigned gridc = (unsigned)(wantc < sms * 16 ? wantc : sms * 16);
  cudaError_t e;
  if (prescaled) {
    if ((e = launch(k_pack_first_nz_clear, dim3(1), dim3(1), 0, s, false, sc)) != cudaSuccess)
      return cuda_fail(e, "k_pack_first_nz_clear");
    if ((e = launch(k_pack_first_nz, dim3(grid), dim3(256), 0, s, false, W, n, sc)) != cudaSuccess)
      return cuda_fail(e, "k_pack_first_nz");
  } else {
    if ((e = launch(k_pack_clear, dim3(1), dim3(1), 0, s, false, sc)) != cudaSuccess) return cuda_fail(e, "k_pack_clear");
    if ((e = launch(k_pack_absmax, dim3(grid), dim3(256), 0, s, false, W, n, sc)) != cudaSuccess)
      return cuda_fail(e, "k_pack_absmax");
    if ((e = launch(k_pack_sum, dim3(grid), dim3(256), 0, s, false, W, n, sc)) != cudaSuccess)
      return cuda_fail(e, "k_pack_sum");
  }
  if ((e = launch(k_pack_codes, dim3(gridc), dim3(256), 0, s, false, W, n, (const PackScratch*)sc,
                  reinterpret_cast<uint32_t*>(packed), prescaled)) != cudaSuccess)
    return cuda_fail(e, "k_pack_codes");
  if ((e = launch(k_pack_trailer, dim3(1), dim3(1), 0, s, false, sc, n, W, prescaled)) != cudaSuccess)
    return cuda_fail(e, "k_pack_trailer");
  return BITNET_OK;
}

bitnet_status bitnet_pack_i2s(const float* W, int64_t N, int64_t K, uint8_t* packed, bitnet_stream stream) {
  return enqueue_pack(W, N, K, packed, 0, reinterpret_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_pack_i2s_prescaled(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                        bitnet_stream stream) {
  return enqueue_pack(W, N, K, packed, 1, reinterpret_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_validate_i2s(const uint8_t* packed, int64_t N, int64_t K, int64_t* counts,
                                  bitnet_stream stream) {
  if (!packed || !counts) return BITNET_ERR_NULL;
  if (N <= 0 || K <= 0 || K % 128 != 0 || N * K >= (1ll << 40)) return BITNET_ERR_SHAPE;
  if (!aligned16(packed) || (reinterpret_cast<uintptr_t>(counts) & 7)) return BITNET_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nwords = N * K / 16;
  const int sms = device_sm_count();
  const long long want = (nwords + 255) / 256;
  const unsigned grid = (unsigned)(want < sms * 8 ? want : sms * 8);
  unsigned long long* c = reinterpret_cast<unsigned long long*>(counts);
  cudaError_t e;
  if ((e = launch(k_validate_clear, dim3(1), dim3(1), 0, s, false, c)) != cudaSuccess)
    return cuda_fail(e, "k_validate_clear");
  if ((e = launch(k_validate_i2s, dim3(grid), dim3(256), 0, s, false, reinterpret_cast<const uint32_t*>(packed), nwords,
                  packed + N * K / 4, c)) != cudaSuccess)
    return cuda_fail(e, "k_validate_i2s");
  return BITNET_OK;
}

bitnet_status bitnet_rmsnorm_quant_act(const void* x, bitnet_dtype xt, const float* gain, float eps, int64_t T,
                                       int64_t K, int8_t* q, float* s_x, int32_t* sum_q, bitnet_stream stream) {
  if (xt != BITNET_BF16 && xt != BITNET_F32) return BITNET_ERR_DTYPE;
  if (T < 0 || K <= 0 || K > BITNET_MAX_K || T > 0x7FFFFFFFll) return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!x || !q || !s_x || !sum_q) return BITNET_ERR_NULL;
  if (!aligned16(x) || !aligned16(q) || !aligned16(s_x) || !aligned16(sum_q) || (gain && !aligned16(gain)))
    return BITNET_ERR_ALIGN;
  return enqueue_quant(x, xt, gain, eps, T, K, q, s_x, sum_q, reinterpret_cast<cudaStream_t>(stream));
}

static bitnet_status check_product_args(const int8_t* q, const float* s_x, const int32_t* sum_q, int64_t T,
                                        int64_t K, bitnet_dtype ot) {
  if (ot != BITNET_BF16 && ot != BITNET_F32) return BITNET_ERR_DTYPE;
  if (T < 0 || K <= 0 || K % 128 != 0 || K > BITNET_MAX_K || T > 0x7FFFFFFFll) return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!q || !s_x || !sum_q) return BITNET_ERR_NULL;
  if (!aligned16(q) || !aligned16(s_x) || !aligned16(sum_q)) return BITNET_ERR_ALIGN;
  return BITNET_OK;
}

bitnet_status bitnet_bitlinear(const int8_t* q, const float* s_x, const int32_t* sum_q, const uint8_t* packed,
                               int64_t T, int64_t N, int64_t K, void* out, bitnet_dtype ot, int32_t* acc_debug,
                               bitnet_stream stream) {
  bitnet_status st = check_product_args(q, s_x, sum_q, T, K, ot);
  if (st != BITNET_OK) return st;
  if (N <= 0 || N > (1 << 30)) return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!packed || !out) return BITNET_ERR_NULL;
  if (!aligned16(packed) || !aligned16(out) || (acc_debug && !aligned16(acc_debug))) return BITNET_ERR_ALIGN;
  const uint8_t* p[1] = {packed};
  const int64_t n[1] = {N};
  void* o[1] = {out};
  int32_t* d[1] = {acc_debug};
  return enqueue_gemv(q, s_x, sum_q, 1, p, n, o, d, T, K, ot, false, BITNET_RELU2, nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_bitlinear_group(const int8_t* q, const float* s_x, const int32_t* sum_q, int n_tensors,
                                     const uint8_t* const* packed, const int64_t* N, int64_t T, int64_t K,
                                     void* const* out, bitnet_dtype ot, bitnet_stream stream) {
  bitnet_status st = check_product_args(q, s_x, sum_q, T, K, ot);
  if (st != BITNET_OK) return st;
  if (n_tensors < 1 || n_tensors > 4) return BITNET_ERR_SHAPE;
  if (!packed || !N || !out) return BITNET_ERR_NULL;
  for (int i = 0; i < n_tensors; ++i) {
    if (N[i] <= 0 || N[i] > (1 << 30)) return BITNET_ERR_SHAPE;
    if (T > 0 && (!packed[i] || !out[i])) return BITNET_ERR_NULL;
    if (T > 0 && (!aligned16(packed[i]) || !aligned16(out[i]))) return BITNET_ERR_ALIGN;
  }
  if (T == 0) return BITNET_OK;
  return enqueue_gemv(q, s_x, sum_q, n_tensors, packed, N, out, nullptr, T, K, ot, false, BITNET_RELU2, nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_bitlinear_gate_up_act(const int8_t* q, const float* s_x, const int32_t* sum_q,
                                           const uint8_t* p_gate, const uint8_t* p_up, int64_t T, int64_t I,
                                           int64_t K, bitnet_act act, float* h, bitnet_stream stream) {
  bitnet_status st = check_product_args(q, s_x, sum_q, T, K, BITNET_F32);
  if (st != BITNET_OK) return st;
  if (act != BITNET_RELU2 && act != BITNET_SILU) return BITNET_ERR_DTYPE;
  if (I <= 0 || I > (1 << 30)) return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!p_gate || !p_up || !h) return BITNET_ERR_NULL;
  if (!aligned16(p_gate) || !aligned16(p_up) || !aligned16(h)) return BITNET_ERR_ALIGN;
  const uint8_t* gu[2] = {p_gate, p_up};
  const int64_t nI[2] = {I, I};
  return enqueue_gemv(q, s_x, sum_q, 2, gu, nI, nullptr, nullptr, T, K, BITNET_F32, true, act, h,
                      reinterpret_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_bitlinear_acc(const int8_t* q, const int32_t* sum_q, const uint8_t* packed, int64_t T, int64_t N,
                                   int64_t K, int32_t* acc, bitnet_stream stream) {
  if (T < 0 || K <= 0 || K % 128 != 0 || K > BITNET_MAX_K || T > 0x7FFFFFFFll || N <= 0 || N > (1 << 30))
    return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!q || !sum_q || !packed || !acc) return BITNET_ERR_NULL;
  if (!aligned16(q) || !aligned16(sum_q) || !aligned16(packed) || !aligned16(acc)) return BITNET_ERR_ALIGN;
  const uint8_t* p[1] = {packed};
  const int64_t n[1] = {N};
  void* o[1] = {nullptr};
  int32_t* d[1] = {acc};
  return enqueue_gemv(q, nullptr, sum_q, 1, p, n, o, d, T, K, BITNET_F32, false, BITNET_RELU2, nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- tensor-parallel pieces
static unsigned shard_grid(int64_t T) {
  const int64_t cap = (int64_t)device_sm_count() * 8;
  return (unsigned)(T < cap ? T : cap);
}

static bitnet_status shard_checks(const float* h, int64_t T, int64_t Ks) {
  if (T < 0 || T > 0x7FFFFFFFll || Ks <= 0 || Ks % 4 != 0 || Ks > (1 << 30)) return BITNET_ERR_SHAPE;
  if (T > 0 && !h) return BITNET_ERR_NULL;
  if (T > 0 && !aligned16(h)) return BITNET_ERR_ALIGN;
  return BITNET_OK;
}

bitnet_status bitnet_subnorm_shard_amax(const float* h, int64_t T, int64_t Ks, float* amax, bitnet_stream stream) {
  bitnet_status st = shard_checks(h, T, Ks);
  if (st != BITNET_OK || T == 0) return st;
  if (!amax) return BITNET_ERR_NULL;
  cudaError_t e = launch(k_shard_amax, dim3(shard_grid(T)), dim3(SHARD_THREADS), 0,
                         reinterpret_cast<cudaStream_t>(stream), true, h, (int)T, (int)Ks, amax);
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_shard_amax");
}

bitnet_status bitnet_subnorm_shard_sumsq(const float* h, int64_t T, int64_t Ks, const float* amax, int64_t K_total,
                                         int64_t* S, bitnet_stream stream) {
  bitnet_status st = shard_checks(h, T, Ks);
  if (st != BITNET_OK || T == 0) return st;
  if (K_total < Ks || K_total > (1ll << 40)) return BITNET_ERR_SHAPE;
  if (!amax || !S) return BITNET_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(S) & 7) return BITNET_ERR_ALIGN;
  cudaError_t e = launch(k_shard_sumsq, dim3(shard_grid(T)), dim3(SHARD_THREADS), 0,
                         reinterpret_cast<cudaStream_t>(stream), true, h, (int)T, (int)Ks, amax, (long long)K_total,
                         reinterpret_cast<long long*>(S));
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_shard_sumsq");
}

bitnet_status bitnet_subnorm_shard_ymax(const float* h, const float* gain, int64_t T, int64_t Ks, const float* amax,
                                        const int64_t* S, int64_t K_total, float eps, float* inv, float* ymax,
                                        bitnet_stream stream) {
  bitnet_status st = shard_checks(h, T, Ks);
  if (st != BITNET_OK || T == 0) return st;
  if (K_total < Ks || K_total > (1ll << 40)) return BITNET_ERR_SHAPE;
  if (!amax || !inv || !ymax || (gain && !S)) return BITNET_ERR_NULL;
  if ((gain && !aligned16(gain)) || (reinterpret_cast<uintptr_t>(S) & 7)) return BITNET_ERR_ALIGN;
  cudaError_t e = launch(k_shard_ymax, dim3(shard_grid(T)), dim3(SHARD_THREADS), 0,
                         reinterpret_cast<cudaStream_t>(stream), true, h, gain, (int)T, (int)Ks, amax,
                         reinterpret_cast<const long long*>(S), (long long)K_total, eps, inv, ymax);
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_shard_ymax");
}

bitnet_status bitnet_subnorm_shard_quant(const float* h, const float* gain, int64_t T, int64_t Ks, const float* inv,
                                         const float* ymax, int8_t* q, float* s_x, int32_t* sum_q,
                                         bitnet_stream stream) {
  bitnet_status st = shard_checks(h, T, Ks);
  if (st != BITNET_OK || T == 0) return st;
  if (!inv || !ymax || !q || !s_x || !sum_q) return BITNET_ERR_NULL;
  if ((gain && !aligned16(gain)) || !aligned16(q)) return BITNET_ERR_ALIGN;
  cudaError_t e = launch(k_shard_quant, dim3(shard_grid(T)), dim3(SHARD_THREADS), 0,
                         reinterpret_cast<cudaStream_t>(stream), true, h, gain, (int)T, (int)Ks, inv, ymax, q, s_x,
                         sum_q);
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_shard_quant");
}

bitnet_status bitnet_dequant_acc(const int32_t* acc, const float* s_x, const uint8_t* packed, int64_t T, int64_t N,
                                 int64_t K, void* out, bitnet_dtype ot, bitnet_stream stream) {
  if (ot != BITNET_BF16 && ot != BITNET_F32) return BITNET_ERR_DTYPE;
  if (T < 0 || T > 0x7FFFFFFFll || N <= 0 || N > (1 << 30) || K <= 0 || K % 128 != 0) return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!acc || !s_x || !packed || !out) return BITNET_ERR_NULL;
  if (!aligned16(packed)) return BITNET_ERR_ALIGN;
  const float* beta = reinterpret_cast<const float*>(packed + N * K / 4);
  const long long total = T * N;
  const long long want = (total + SHARD_THREADS - 1) / SHARD_THREADS;
  const long long cap = (long long)device_sm_count() * 8;
  cudaError_t e = launch(k_dequant_acc, dim3((unsigned)(want < cap ? want : cap)), dim3(SHARD_THREADS), 0,
                         reinterpret_cast<cudaStream_t>(stream), true, acc, s_x, beta, (long long)T, (int)N, out,
                         (int)ot);
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_dequant_acc");
}

// ---------------------------------------------------------------- attention (decode)
bitnet_status bitnet_rope_kv_append(const void* q, const void* k, const void* v, bitnet_dtype xt, int64_t T, int64_t Hq,
                                    int64_t Hkv, int64_t d, int64_t pos0, double theta, float* q_rot, void* k_cache,
                                    void* v_cache, int64_t L_max, bitnet_stream stream) {
  if (xt != BITNET_BF16 && xt != BITNET_F32) return BITNET_ERR_DTYPE;
  if (T < 0 || T > 0x7FFFFFFFll || d != ATT_D || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Hq > 4096 || pos0 < 0 ||
      L_max <= 0 || pos0 + T > L_max || !(theta > 0.0))
    return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!q || !k || !v || !q_rot || !k_cache || !v_cache) return BITNET_ERR_NULL;
  const long long total = T * (Hq + 2 * Hkv) * (ATT_D / 2);
  const long long want = (total + 255) / 256, cap = (long long)device_sm_count() * 16;
  const dim3 grid((unsigned)(want < cap ? want : cap));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (xt == BITNET_BF16)
    e = launch(k_rope_append<__nv_bfloat16>, grid, dim3(256), 0, s, true, reinterpret_cast<const __nv_bfloat16*>(q),
               reinterpret_cast<const __nv_bfloat16*>(k), reinterpret_cast<const __nv_bfloat16*>(v), (int)T, (int)Hq,
               (int)Hkv, (long long)pos0, theta, q_rot, reinterpret_cast<__nv_bfloat16*>(k_cache),
               reinterpret_cast<__nv_bfloat16*>(v_cache), (long long)L_max);
  else
    e = launch(k_rope_append<float>, grid, dim3(256), 0, s, true, reinterpret_cast<const float*>(q),
               reinterpret_cast<const float*>(k), reinterpret_cast<const float*>(v), (int)T, (int)Hq, (int)Hkv,
               (long long)pos0, theta, q_rot, reinterpret_cast<__nv_bfloat16*>(k_cache),
               reinterpret_cast<__nv_bfloat16*>(v_cache), (long long)L_max);
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_rope_append");
}

size_t bitnet_attention_workspace_bytes(int64_t T, int64_t Hq, int64_t Hkv, int64_t L) {
  if (T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L <= 0) return 0;
  const long long chunks = (L + ATT_CHUNK - 1) / ATT_CHUNK;
  return (size_t)chunks * Hkv * (T * (Hq / Hkv)) * (ATT_D + 2) * sizeof(float);
}

bitnet_status bitnet_attention_decode(const float* q_rot, const void* k_cache, const void* v_cache, int64_t T,
                                      int64_t Hq, int64_t Hkv, int64_t d, int64_t pos0, int64_t L_max, void* out,
                                      bitnet_dtype ot, void* ws, size_t ws_bytes, bitnet_stream stream) {
  if (ot != BITNET_BF16 && ot != BITNET_F32) return BITNET_ERR_DTYPE;
  if (T < 0 || d != ATT_D || Hq <= 0 || Hkv <= 0 || Hq % Hkv || pos0 < 0 || L_max <= 0 || pos0 + T > L_max ||
      T * (Hq / Hkv) > ATT_MAX_ROWS || Hq > 4096 || (pos0 + T + ATT_CHUNK - 1) / ATT_CHUNK > ATT_MAX_CHUNKS)
    return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!q_rot || !k_cache || !v_cache || !out) return BITNET_ERR_NULL;
  if (!aligned16(q_rot) || !aligned16(k_cache) || !aligned16(v_cache)) return BITNET_ERR_ALIGN;
  if (!ws || ws_bytes < bitnet_attention_workspace_bytes(T, Hq, Hkv, pos0 + T)) return BITNET_ERR_WORKSPACE;
  if (!aligned16(ws)) return BITNET_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int R = (int)(T * (Hq / Hkv));
  const int chunks = (int)((pos0 + T + ATT_CHUNK - 1) / ATT_CHUNK);
  const size_t smem = attn_partial_smem(R);
  static std::atomic<int> attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_done[dev & 63].load(std::memory_order_acquire)) {
    cudaError_t ea = cudaFuncSetAttribute(k_attn_partial, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)attn_partial_smem(ATT_MAX_ROWS));
    if (ea != cudaSuccess) return cuda_fail(ea, "k_attn_partial attribute");
    attr_done[dev & 63].store(1, std::memory_order_release);
  }
  float* part = reinterpret_cast<float*>(ws);
  cudaError_t e = launch(k_attn_partial, dim3((unsigned)chunks, (unsigned)Hkv), dim3(ATT_THREADS), smem, s, true,
                         q_rot, reinterpret_cast<const __nv_bfloat16*>(k_cache),
                         reinterpret_cast<const __nv_bfloat16*>(v_cache), (int)T, (int)Hq, (int)Hkv, (long long)pos0,
                         (long long)L_max, part);
  if (e != cudaSuccess) return cuda_fail(e, "k_attn_partial");
  e = launch(k_attn_combine, dim3((unsigned)(T * Hq)), dim3(ATT_D), 0, s, true, (const float*)part, (int)T, (int)Hq,
             (int)Hkv, chunks, out, (int)ot);
  return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "k_attn_combine");
}

static size_t align_up(size_t v) { return (v + 255) & ~(size_t)255; }

constexpr int FFN_WS_SLOTS = 8;
constexpr size_t ENG_COUNTER_BYTES = 256;  // ENG_MAX_BARRIERS + 1 counters, padded

bitnet_status bitnet_ffn_workspace_offsets(int64_t T, int64_t H, int64_t I, size_t* off) {
  if (!off) return BITNET_ERR_NULL;
  if (T < 0 || H <= 0 || I <= 0) return BITNET_ERR_SHAPE;
  size_t o = 0;
  off[0] = o; o = align_up(o + (size_t)T * H);      // q_x
  off[1] = o; o = align_up(o + (size_t)T * 4);      // s_x
  off[2] = o; o = align_up(o + (size_t)T * 4);      // sum_x
  off[3] = o; o = align_up(o + (size_t)T * I * 4);  // h
  off[4] = o; o = align_up(o + (size_t)T * I);      // q_h
  off[5] = o; o = align_up(o + (size_t)T * 4);      // s_h
  off[6] = o; o = align_up(o + (size_t)T * 4);      // sum_h
  off[7] = o;                                       // grid-barrier counters, then per-CTA partials
  return BITNET_OK;
}

// Per-CTA partial reductions of the distributed sub-norm after the counters (G = ENG_MAX_GRID):
// max |h| [T][G] fp32, max |y| [T][G] fp32, candidate fixed-point sums [T][G][ENG_SUB_CAND]
// int64, fallback sums [T][G] int64, max |y| candidates [T][G] (h, g) fp32 pairs and their counts
// [T][G] int32.
static size_t ffn_partials_bytes(int64_t T) {
  return 2 * align_up((size_t)T * ENG_MAX_GRID * 4) + align_up((size_t)T * ENG_MAX_GRID * ENG_SUB_CAND * 8) +
         2 * align_up((size_t)T * ENG_MAX_GRID * 8) +
         (size_t)T * ENG_MAX_GRID * 4;
}

size_t bitnet_ffn_workspace_bytes(int64_t T, int64_t H, int64_t I) {
  size_t off[FFN_WS_SLOTS];
  if (bitnet_ffn_workspace_offsets(T, H, I, off) != BITNET_OK) return 0;
  return off[7] + ENG_COUNTER_BYTES + ffn_partials_bytes(T);
}

// Appends the FFN phases (x [T, H] -> out [T, H]) to an engine plan; `bar` is the next
// free barrier id, `wait0` a barrier the first phase must wait for (-1: none).
static void plan_ffn(EngArgs& ea, int& bar, int wait0, const void* x, int x_f32, const float* g_ffn,
                     const uint8_t* p_gate, const uint8_t* p_up, const float* g_sub, const uint8_t* p_down, int64_t T,
                     int64_t H, int64_t I, int act, void* out, int ot, uint8_t* ws) {
  size_t off[FFN_WS_SLOTS];
  bitnet_ffn_workspace_offsets(T, H, I, off);
  int8_t* q_x = reinterpret_cast<int8_t*>(ws + off[0]);
  float* s_x = reinterpret_cast<float*>(ws + off[1]);
  int32_t* sum_x = reinterpret_cast<int32_t*>(ws + off[2]);
  float* h = reinterpret_cast<float*>(ws + off[3]);
  int8_t* q_h = reinterpret_cast<int8_t*>(ws + off[4]);
  float* s_h = reinterpret_cast<float*>(ws + off[5]);
  int32_t* sum_h = reinterpret_cast<int32_t*>(ws + off[6]);
  const uint8_t* gu[2] = {p_gate, p_up};
  const int64_t nI[2] = {I, I};
  EngPhase gate_up = eng_gemv((int)H, true, 2, gu, nI, nullptr, nullptr, BITNET_F32, act, h);
  if (eng_local_ok(T, H)) {
    eng_src_local(gate_up, x, x_f32, g_ffn, q_x, s_x, sum_x);
    gate_up.wait_barrier = wait0;
  } else {
    EngPhase qp = eng_quant(x, x_f32, (int)H, g_ffn, q_x, s_x, sum_x);
    qp.wait_barrier = wait0;
    qp.arrive_barrier = bar++;
    ea.ph[ea.n_phases++] = qp;
    eng_src_global(gate_up, q_x, s_x, sum_x);
    gate_up.wait_barrier = qp.arrive_barrier;
  }
  const int64_t nH[1] = {H};
  void* o[1] = {out};
  EngPhase down = eng_gemv((int)I, false, 1, &p_down, nH, o, nullptr, ot, act, nullptr);
  if (eng_local_ok(T, I)) {
    gate_up.arrive_barrier = bar++;
    ea.ph[ea.n_phases++] = gate_up;
    eng_src_local(down, h, 1, g_sub, q_h, s_h, sum_h);
    down.wait_barrier = gate_up.arrive_barrier;
  } else {
    // ffn_sub_norm spread over the grid: every CTA reduces the rows of h it produced (kept
    // in its shared memory, so the SUBNORM phase starts without waiting for the others).
    uint8_t* pb = ws + off[7] + ENG_COUNTER_BYTES;
    float* pmax = reinterpret_cast<float*>(pb);
    float* pmax2 = reinterpret_cast<float*>(pb + align_up((size_t)T * ENG_MAX_GRID * 4));
    long long* psum = reinterpret_cast<long long*>(pb + 2 * align_up((size_t)T * ENG_MAX_GRID * 4));
    long long* psum_fb = reinterpret_cast<long long*>(pb + 2 * align_up((size_t)T * ENG_MAX_GRID * 4) +
                                                      align_up((size_t)T * ENG_MAX_GRID * ENG_SUB_CAND * 8));
    uint8_t* pyb = reinterpret_cast<uint8_t*>(psum_fb) + align_up((size_t)T * ENG_MAX_GRID * 8);
    float2* pyc = reinterpret_cast<float2*>(pyb);
    int* pycnt = reinterpret_cast<int*>(pyb + align_up((size_t)T * ENG_MAX_GRID * 8));
    gate_up.pmax = pmax;
    gate_up.sub_gain = g_sub;
    ea.ph[ea.n_phases++] = gate_up;
    EngPhase sp;
    memset(&sp, 0, sizeof(sp));
    sp.kind = PH_SUBNORM;
    sp.K = (int)I;
    sp.n_tiles = gate_up.n_tiles;
    sp.x = h;
    sp.x_f32 = 1;
    sp.gain = g_sub;
    sp.q = q_h;
    sp.s = s_h;
    sp.sq = sum_h;
    sp.pmax = pmax;
    sp.pmax2 = pmax2;
    sp.psum = psum;
    sp.psum_fb = psum_fb;
    sp.pyc = pyc;
    sp.pycnt = pycnt;
    sp.wait_barrier = -1;
    sp.bar_a = bar++;
    sp.bar_b = bar++;
    sp.bar_fb = bar++;
    sp.arrive_barrier = bar++;
    ea.ph[ea.n_phases++] = sp;
    eng_src_global(down, q_h, s_h, sum_h);
    down.wait_barrier = sp.arrive_barrier;
  }
  ea.ph[ea.n_phases++] = down;
}

// The FFN as separate launches (prefill): quant, gate/up + act, quant, down.
static bitnet_status enqueue_ffn_launches(const void* x, bitnet_dtype xt, const float* g_ffn, const uint8_t* p_gate,
                                          const uint8_t* p_up, const float* g_sub, const uint8_t* p_down, int64_t T,
                                          int64_t H, int64_t I, bitnet_act act, float eps, void* out, bitnet_dtype ot,
                                          uint8_t* w, cudaStream_t s) {
  size_t off[FFN_WS_SLOTS];
  bitnet_ffn_workspace_offsets(T, H, I, off);
  int8_t* q_x = reinterpret_cast<int8_t*>(w + off[0]);
  float* s_x = reinterpret_cast<float*>(w + off[1]);
  int32_t* sum_x = reinterpret_cast<int32_t*>(w + off[2]);
  float* h = reinterpret_cast<float*>(w + off[3]);
  int8_t* q_h = reinterpret_cast<int8_t*>(w + off[4]);
  float* s_h = reinterpret_cast<float*>(w + off[5]);
  int32_t* sum_h = reinterpret_cast<int32_t*>(w + off[6]);
  bitnet_status st = enqueue_quant(x, xt, g_ffn, eps, T, H, q_x, s_x, sum_x, s);
  if (st != BITNET_OK) return st;
  const uint8_t* gu[2] = {p_gate, p_up};
  const int64_t nI[2] = {I, I};
  st = enqueue_gemv(q_x, s_x, sum_x, 2, gu, nI, nullptr, nullptr, T, H, BITNET_F32, true, act, h, s);
  if (st != BITNET_OK) return st;
  st = enqueue_quant(h, BITNET_F32, g_sub, eps, T, I, q_h, s_h, sum_h, s);
  if (st != BITNET_OK) return st;
  const uint8_t* pd[1] = {p_down};
  const int64_t nH[1] = {H};
  void* o[1] = {out};
  return enqueue_gemv(q_h, s_h, sum_h, 1, pd, nH, o, nullptr, T, I, ot, false, act, nullptr, s);
}

// Checks of bitnet_ffn_block's arguments other than the workspace (BITNET_OK also for T = 0).
static bitnet_status ffn_check_args(const void* x, bitnet_dtype xt, const uint8_t* p_gate, const uint8_t* p_up,
                                    const uint8_t* p_down, int64_t T, int64_t H, int64_t I, bitnet_act act,
                                    const void* out, bitnet_dtype ot, const float* g_ffn, const float* g_sub) {
  if (xt != BITNET_BF16 && xt != BITNET_F32) return BITNET_ERR_DTYPE;
  if (ot != BITNET_BF16 && ot != BITNET_F32) return BITNET_ERR_DTYPE;
  if (act != BITNET_RELU2 && act != BITNET_SILU) return BITNET_ERR_DTYPE;
  if (T < 0 || T > 0x7FFFFFFFll || H <= 0 || I <= 0 || H % 128 || I % 128 || H > BITNET_MAX_K || I > BITNET_MAX_K)
    return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  if (!x || !p_gate || !p_up || !p_down || !out) return BITNET_ERR_NULL;
  if (!aligned16(x) || !aligned16(p_gate) || !aligned16(p_up) || !aligned16(p_down) || !aligned16(out) ||
      (g_ffn && !aligned16(g_ffn)) || (g_sub && !aligned16(g_sub)))
    return BITNET_ERR_ALIGN;
  return BITNET_OK;
}

bitnet_status bitnet_ffn_block(const void* x, bitnet_dtype xt, const float* g_ffn, const uint8_t* p_gate,
                               const uint8_t* p_up, const float* g_sub, const uint8_t* p_down, int64_t T, int64_t H,
                               int64_t I, bitnet_act act, float eps, void* out, bitnet_dtype ot, void* ws,
                               size_t ws_bytes, bitnet_stream stream) {
  bitnet_status st0 = ffn_check_args(x, xt, p_gate, p_up, p_down, T, H, I, act, out, ot, g_ffn, g_sub);
  if (st0 != BITNET_OK || T == 0) return st0;
  if (!ws) return BITNET_ERR_WORKSPACE;
  if (ws_bytes < bitnet_ffn_workspace_bytes(T, H, I)) return BITNET_ERR_WORKSPACE;
  if (!aligned16(ws)) return BITNET_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  if (T > ENG_MAX_T || !eng_quant_ok(H) || !eng_quant_ok(I))
    return enqueue_ffn_launches(x, xt, g_ffn, p_gate, p_up, g_sub, p_down, T, H, I, act, eps, out, ot, w, s);
  size_t off[FFN_WS_SLOTS];
  bitnet_ffn_workspace_offsets(T, H, I, off);
  EngArgs ea;
  memset(&ea, 0, sizeof(ea));
  ea.T = (int)T;
  ea.eps = eps;
  ea.counters = reinterpret_cast<unsigned*>(w + off[7]);
  int bar = 0;
  plan_ffn(ea, bar, -1, x, xt == BITNET_F32, g_ffn, p_gate, p_up, g_sub, p_down, T, H, I, act, out, ot, w);
  return enqueue_engine(ea, s);
}

// ---------------------------------------------------------------- FFN without a caller workspace
// For callers that cannot allocate device memory themselves (for example a plugin inside a
// host framework that owns all device memory and forbids allocation while it serves, or a
// process under a hard memory cap): the FFN block's workspace lives in this file-scope
// array instead.  Every GPU that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB: every FFN up to 16 tokens of the
                                                    // configured model shapes fits
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  The array's name in host
// code is only a host-side stand-in, so the address is looked up once per device, with
// that device current, by the first call made on it.
static bitnet_status noalloc_scratch(uint8_t** out) {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return cuda_fail(cudaErrorInvalidDevice, "no-alloc scratch (device id)");
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    addr[dev] = reinterpret_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return BITNET_OK;
}

size_t bitnet_ffn_block_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

bitnet_status bitnet_ffn_block_noalloc(const void* x, bitnet_dtype xt, const float* g_ffn, const uint8_t* p_gate,
                                       const uint8_t* p_up, const float* g_sub, const uint8_t* p_down, int64_t T,
                                       int64_t H, int64_t I, bitnet_act act, float eps, void* out, bitnet_dtype ot,
                                       bitnet_stream stream) {
  // The same argument checks as bitnet_ffn_block, all before the shared scratch is touched,
  // so that an invalid call writes nothing and returns the same status.
  bitnet_status st = ffn_check_args(x, xt, p_gate, p_up, p_down, T, H, I, act, out, ot, g_ffn, g_sub);
  if (st != BITNET_OK || T == 0) return st;
  const size_t need = bitnet_ffn_workspace_bytes(T, H, I);
  if (need == 0) return BITNET_ERR_SHAPE;
  if (need > kNoAllocScratchBytes) {
    t_last_error = "bitnet_ffn_block_noalloc: the workspace for these sizes exceeds the built-in scratch of " +
                   std::to_string(kNoAllocScratchBytes) + " bytes; pass a workspace to bitnet_ffn_block";
    return BITNET_ERR_WORKSPACE;
  }
  uint8_t* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != BITNET_OK) return st;
  // The grid-barrier counters must start at zero; the previous call normally leaves them
  // zero, but clear them anyway (a call that timed out would not have).
  size_t off[FFN_WS_SLOTS];
  bitnet_ffn_workspace_offsets(T, H, I, off);
  cudaError_t e = cudaMemsetAsync(ws + off[7], 0, ENG_COUNTER_BYTES, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-alloc counters)");
  return bitnet_ffn_block(x, xt, g_ffn, p_gate, p_up, g_sub, p_down, T, H, I, act, eps, out, ot, ws,
                          kNoAllocScratchBytes, stream);
}

// ---------------------------------------------------------------- decoder block
bitnet_status bitnet_block_workspace_offsets(int64_t T, int64_t H, int64_t NQ, int64_t I, size_t* off) {
  if (!off) return BITNET_ERR_NULL;
  if (T < 0 || H <= 0 || NQ <= 0 || I <= 0) return BITNET_ERR_SHAPE;
  size_t o = 0;
  off[0] = o; o = align_up(o + (size_t)T * H);    // q of x (attn_norm)
  off[1] = o; o = align_up(o + (size_t)T * 4);
  off[2] = o; o = align_up(o + (size_t)T * 4);
  off[3] = o; o = align_up(o + (size_t)T * NQ);   // q of the attention output (attn_sub_norm)
  off[4] = o; o = align_up(o + (size_t)T * 4);
  off[5] = o; o = align_up(o + (size_t)T * 4);
  off[6] = o;                                     // the FFN's workspace
  return BITNET_OK;
}

size_t bitnet_block_workspace_bytes(int64_t T, int64_t H, int64_t NQ, int64_t I) {
  size_t off[7];
  if (bitnet_block_workspace_offsets(T, H, NQ, I, off) != BITNET_OK) return 0;
  return off[6] + bitnet_ffn_workspace_bytes(T, H, I);
}

bitnet_status bitnet_decoder_block(const void* x, const void* attn_out, bitnet_dtype xt, const float* g_attn_norm,
                                   const float* g_attn_sub_norm, const float* g_ffn_norm, const float* g_ffn_sub_norm,
                                   const uint8_t* p_q, const uint8_t* p_k, const uint8_t* p_v, const uint8_t* p_o,
                                   const uint8_t* p_gate, const uint8_t* p_up, const uint8_t* p_down, int64_t T,
                                   int64_t H, int64_t NQ, int64_t NKV, int64_t I, bitnet_act act, float eps,
                                   void* out_q, void* out_k, void* out_v, void* out_o, void* out_ffn, bitnet_dtype ot,
                                   void* ws, size_t ws_bytes, bitnet_stream stream) {
  if (xt != BITNET_BF16 && xt != BITNET_F32) return BITNET_ERR_DTYPE;
  if (ot != BITNET_BF16 && ot != BITNET_F32) return BITNET_ERR_DTYPE;
  if (act != BITNET_RELU2 && act != BITNET_SILU) return BITNET_ERR_DTYPE;
  if (T < 0 || T > 0x7FFFFFFFll || H <= 0 || NQ <= 0 || NKV <= 0 || I <= 0 || H % 128 || NQ % 128 || I % 128 ||
      H > BITNET_MAX_K || NQ > BITNET_MAX_K || I > BITNET_MAX_K || NQ > (1 << 30) || NKV > (1 << 30))
    return BITNET_ERR_SHAPE;
  if (T == 0) return BITNET_OK;
  const void* need[] = {x, attn_out, p_q, p_k, p_v, p_o, p_gate, p_up, p_down, out_q, out_k, out_v, out_o, out_ffn};
  for (const void* p : need)
    if (!p) return BITNET_ERR_NULL;
  if (!ws) return BITNET_ERR_WORKSPACE;
  if (ws_bytes < bitnet_block_workspace_bytes(T, H, NQ, I)) return BITNET_ERR_WORKSPACE;
  for (const void* p : need)
    if (!aligned16(p)) return BITNET_ERR_ALIGN;
  const void* gains[] = {g_attn_norm, g_attn_sub_norm, g_ffn_norm, g_ffn_sub_norm};
  for (const void* p : gains)
    if (p && !aligned16(p)) return BITNET_ERR_ALIGN;
  if (!aligned16(ws)) return BITNET_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  size_t off[7];
  bitnet_block_workspace_offsets(T, H, NQ, I, off);
  int8_t* q_x = reinterpret_cast<int8_t*>(w + off[0]);
  float* s_x = reinterpret_cast<float*>(w + off[1]);
  int32_t* sum_x = reinterpret_cast<int32_t*>(w + off[2]);
  int8_t* q_a = reinterpret_cast<int8_t*>(w + off[3]);
  float* s_a = reinterpret_cast<float*>(w + off[4]);
  int32_t* sum_a = reinterpret_cast<int32_t*>(w + off[5]);
  uint8_t* wf = w + off[6];
  const uint8_t* pqkv[3] = {p_q, p_k, p_v};
  const int64_t nqkv[3] = {NQ, NKV, NKV};
  void* oqkv[3] = {out_q, out_k, out_v};
  const int64_t nH[1] = {H};
  void* oo[1] = {out_o};
  if (T > ENG_MAX_T || !eng_quant_ok(H) || !eng_quant_ok(NQ) || !eng_quant_ok(I)) {
    bitnet_status st = enqueue_quant(x, xt, g_attn_norm, eps, T, H, q_x, s_x, sum_x, s);
    if (st == BITNET_OK) st = enqueue_gemv(q_x, s_x, sum_x, 3, pqkv, nqkv, oqkv, nullptr, T, H, ot, false, act, nullptr, s);
    if (st == BITNET_OK) st = enqueue_quant(attn_out, xt, g_attn_sub_norm, eps, T, NQ, q_a, s_a, sum_a, s);
    if (st == BITNET_OK) st = enqueue_gemv(q_a, s_a, sum_a, 1, &p_o, nH, oo, nullptr, T, NQ, ot, false, act, nullptr, s);
    if (st == BITNET_OK)
      st = enqueue_ffn_launches(out_o, ot, g_ffn_norm, p_gate, p_up, g_ffn_sub_norm, p_down, T, H, I, act, eps,
                                out_ffn, ot, wf, s);
    return st;
  }
  // One engine launch: o first (the FFN depends on it), then q/k/v while o's barrier
  // completes, then the FFN.
  size_t offf[FFN_WS_SLOTS];
  bitnet_ffn_workspace_offsets(T, H, I, offf);
  EngArgs ea;
  memset(&ea, 0, sizeof(ea));
  ea.T = (int)T;
  ea.eps = eps;
  ea.counters = reinterpret_cast<unsigned*>(wf + offf[7]);
  int bar = 0;
  const int xf = xt == BITNET_F32;
  EngPhase po = eng_gemv((int)NQ, false, 1, &p_o, nH, oo, nullptr, ot, act, nullptr);
  EngPhase pqkvp = eng_gemv((int)H, false, 3, pqkv, nqkv, oqkv, nullptr, ot, act, nullptr);
  int qa_bar = -1, qx_bar = -1;
  if (!eng_local_ok(T, NQ)) {
    EngPhase qp = eng_quant(attn_out, xf, (int)NQ, g_attn_sub_norm, q_a, s_a, sum_a);
    qp.arrive_barrier = qa_bar = bar++;
    ea.ph[ea.n_phases++] = qp;
  }
  if (!eng_local_ok(T, H)) {
    EngPhase qp = eng_quant(x, xf, (int)H, g_attn_norm, q_x, s_x, sum_x);
    qp.arrive_barrier = qx_bar = bar++;
    ea.ph[ea.n_phases++] = qp;
  }
  if (qa_bar >= 0) {
    eng_src_global(po, q_a, s_a, sum_a);
    po.wait_barrier = qa_bar;
  } else {
    eng_src_local(po, attn_out, xf, g_attn_sub_norm, q_a, s_a, sum_a);
  }
  po.arrive_barrier = bar++;
  ea.ph[ea.n_phases++] = po;
  if (qx_bar >= 0) {
    eng_src_global(pqkvp, q_x, s_x, sum_x);
    pqkvp.wait_barrier = qx_bar;
  } else {
    eng_src_local(pqkvp, x, xf, g_attn_norm, q_x, s_x, sum_x);
  }
  ea.ph[ea.n_phases++] = pqkvp;
  plan_ffn(ea, bar, po.arrive_barrier, out_o, ot == BITNET_F32, g_ffn_norm, p_gate, p_up, g_ffn_sub_norm, p_down, T,
           H, I, act, out_ffn, ot, wf);
  return enqueue_engine(ea, s);
}

bitnet_status bitnet_debug_set_wait_limit(long long cycles) {
  if (cycles <= 0) cycles = kDefaultWaitLimitCycles;
  BN_CUDA(cudaDeviceSynchronize(), "wait limit (synchronize)");
  BN_CUDA(cudaMemcpyToSymbol(c_wait_limit, &cycles, sizeof(cycles)), "wait limit (copy)");
  BN_CUDA(cudaDeviceSynchronize(), "wait limit (synchronize)");
  return BITNET_OK;
}

bitnet_status bitnet_get_device_status(bitnet_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  const int zero = 0;
  BN_CUDA(cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s), "status read");
  BN_CUDA(cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s), "status clear");
  BN_CUDA(cudaStreamSynchronize(s), "status sync");
  return v == 0 ? BITNET_OK : (bitnet_status)v;
}

const char* bitnet_status_string(bitnet_status st) {
  switch (st) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_NULL: return "null pointer";
    case BITNET_ERR_SHAPE: return "invalid shape";
    case BITNET_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BITNET_ERR_DTYPE: return "invalid dtype or activation";
    case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
    case BITNET_ERR_CUDA: return "CUDA error";
    case BITNET_ERR_TIMEOUT: return "kernel wait timed out";
  }
  return "unknown status";
}

const char* bitnet_last_error(void) { return t_last_error.c_str(); }

}  // extern "C"

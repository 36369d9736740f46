// Shared device helpers of the sm_100a kernels: exact fp32/fp64 steps, block
// reductions, programmatic-dependent-launch control, bulk L2 prefetch.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/bitnet_b200.h"

#define BN_DEV __device__ __forceinline__
#define BN_HOST_DEV __host__ __device__

namespace bitnet {

// Device status word (bounded waits that gave up set BITNET_ERR_TIMEOUT here).  The
// library is one translation unit (bitnet_b200.cu includes every kernel header).
__device__ int g_device_status = 0;

// ---------------------------------------------------------------- launch control
// Programmatic dependent launch: let the next kernel on the stream start its
// prologue now; wait for the previous kernel's memory before reading activations.
BN_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
BN_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bulk prefetch of a contiguous global range into L2 (address and size 16-byte multiples).
BN_DEV void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

BN_DEV uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16-byte shared-memory load at a shared-space address.
BN_DEV uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// The same, only where `pred` holds; elsewhere `v` keeps its value.
BN_DEV void lds128_if(uint4& v, uint32_t addr, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "@p ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "r"(addr), "r"((uint32_t)pred));
}

// ---------------------------------------------------------------- mbarriers, bulk copies
BN_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

BN_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Make barrier initialisation visible to the async proxy (bulk copies, tensor cores).
BN_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
BN_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

BN_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
BN_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
BN_DEV void mbar_arrive_count(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
BN_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Limit of every bounded wait, in SM clock cycles (about a second by default).  A wait that
// runs past it gives up: the device status word is set to BITNET_ERR_TIMEOUT and the kernel
// leaves its loops.  bitnet_debug_set_wait_limit() changes it between launches (tests use a
// short limit to make waits run out on purpose).
constexpr long long kDefaultWaitLimitCycles = 2000000000ll;
__constant__ long long c_wait_limit = kDefaultWaitLimitCycles;
// After a wait has given up, the copies a CTA issued into its own shared memory are still
// awaited before it exits, with this fixed limit (not the settable one): they are plain reads
// of global memory and always land.
constexpr long long kDrainLimitCycles = 2000000000ll;

// Wait for phase `parity` of a barrier, giving up after c_wait_limit clock cycles: then the
// device status word is set to BITNET_ERR_TIMEOUT and false returned.
BN_DEV bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64(), lim = c_wait_limit;
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > lim) {
      atomicExch(&g_device_status, (int)BITNET_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Wait, with the fixed drain limit, for phase `parity` of a barrier that a copy into this
// CTA's shared memory completes (used on the way out after another wait gave up).
BN_DEV void mbar_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 <= kDrainLimitCycles) {
  }
}

// Bulk copy global -> this CTA's shared memory, completing `bytes` on barrier `bar`
// (no multicast).  Addresses 16-byte aligned, size a multiple of 16.
BN_DEV void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// The same with an L2 cache policy (createpolicy), e.g. evict-first for bytes read once.
BN_DEV void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}
BN_DEV uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 2-D TMA load of one box of `map` at (x, y) into this CTA's shared memory, completing on
// barrier `bar` (no multicast).  x * element size must be a multiple of 16 bytes.
BN_DEV void tma_load_2d(uint32_t dst, const void* map, int x, int y, uint32_t bar) {
  asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
               ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar)
               : "memory");
}
BN_DEV void tma_load_2d_hint(uint32_t dst, const void* map, int x, int y, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;"
      ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// 16-byte asynchronous copy global -> shared (both 16-byte aligned), completed by
// cp_async_wait_all in the issuing thread.
BN_DEV void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
BN_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
BN_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Named barrier over `count` threads (a multiple of 32).
BN_DEV void named_sync(int id, int count) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory"); }
// Named barrier that also returns whether `pred` was true in any of the threads.
BN_DEV bool named_sync_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------- exact helpers
// 2**e as an fp64 (exact for -1022 <= e <= 1023).
BN_DEV double pow2_f64(int e) { return __longlong_as_double((long long)(1023 + e) << 52); }

// E with M = m * 2**E, 0.5 <= m < 1, for a normal positive fp64 M.
BN_DEV int frexp_exponent(double M) { return (int)((__double_as_longlong(M) >> 52) & 0x7FF) - 1022; }

// Smallest L with 2**L >= n (n >= 1).
BN_DEV int ceil_log2_i64(long long n) { return n <= 1 ? 0 : 64 - __clzll(n - 1); }

// Fixed-point grid exponent e = 62 - E(M) - ceil_log2(n) of an order-free sum of n
// non-negative terms whose maximum is M > 0.
BN_DEV int fixed_point_exponent(double M, long long n) { return 62 - frexp_exponent(M) - ceil_log2_i64(n); }

// fp32( (fp64(S) * 2**-e) / n ): the mean of a fixed-point sum.
BN_DEV float fixed_point_mean(long long S, int e, long long n) {
  if (S == 0) return 0.0f;
  double v = __dmul_rn(__ll2double_rn(S), pow2_f64(-e));
  return __double2float_rn(__ddiv_rn(v, __ll2double_rn(n)));
}

BN_DEV float bf16_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// The terms of the exact fixed-point sums on the grid 2^-e (p2e = 2^e): rint(v^2 2^e) and
// rint(|v| 2^e) for an fp32 v, in fp64, where v^2 and the scaling are exact; then rounded
// half to even to an integer.  Valid while the result is below 2^62, which the choice of e
// guarantees.
BN_DEV long long fixed_sq_term(float v, double p2e) {
  const double d = (double)v;
  return __double2ll_rn(__dmul_rn(__dmul_rn(d, d), p2e));
}
BN_DEV long long fixed_abs_term(float v, double p2e) { return __double2ll_rn(__dmul_rn((double)fabsf(v), p2e)); }

// Rounding to an integer without a conversion instruction (conversions issue at a quarter of
// the fp64 add rate): adding 1.5 * 2^52 to a double x with |x| < 2^51 leaves rint(x) -- the
// addition rounds to the nearest integer, ties to even -- in the low bits of the significand.
BN_DEV long long rint_i64_small(double x) {
  return __double_as_longlong(__dadd_rn(x, 6755399441055744.0)) - 0x4338000000000000ll;
}
// The sums' n terms are each below 2^(62 - ceil_log2(n)), hence below 2^51 once n > 1024.
constexpr long long kFixedSmallMinN = 1025;
template <bool SMALL>
BN_DEV long long fixed_sq_term_t(float v, double p2e) {
  if (!SMALL) return fixed_sq_term(v, p2e);
  const double d = (double)v;
  return rint_i64_small(__dmul_rn(__dmul_rn(d, d), p2e));
}

// int8 code of an activation: clamp(rint(p), -128, 127), ties to even, for the fp32 product
// p = y * s (NaN gives 0, as the conversion instruction does).  Clamping first keeps |p| below
// 2^22, where adding 1.5 * 2^23 rounds p to an integer in the low significand bits.
BN_DEV int quant_code(float p) {
  const float c = fminf(fmaxf(p, -128.0f), 127.0f);
  const int q = __float_as_int(__fadd_rn(c, 12582912.0f)) - 0x4B400000;
  return p == p ? q : 0;
}

// ---------------------------------------------------------------- reductions
BN_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
BN_DEV long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
BN_DEV int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide reductions through a small shared scratch of >= 32 entries; every thread
// gets the result.  max over non-negative floats and integer sums are exact, so the
// result does not depend on the order.
template <typename T, typename Op>
BN_DEV T block_reduce(T v, T* scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();  // scratch may still be read by a previous reduction
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  // every warp reduces the (at most 32) warp results with shuffles: one shared load per thread
  T r = lane < nw ? scratch[lane] : Op::identity();
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r = op(r, __shfl_xor_sync(0xffffffffu, r, o));
  return r;
}

// The same with one barrier instead of two: consecutive calls alternate between two scratch
// areas, so a call's area is rewritten only after the following call's barrier, which every
// thread reaches after it has read that area.
template <typename T, typename Op>
BN_DEV T block_reduce_alt(T v, T* scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = lane < nw ? scratch[lane] : Op::identity();
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r = op(r, __shfl_xor_sync(0xffffffffu, r, o));
  return r;
}

struct MaxOp {
  BN_DEV float operator()(float a, float b) const { return fmaxf(a, b); }
  BN_DEV static float identity() { return -INFINITY; }
};
struct AddOpLL {
  BN_DEV long long operator()(long long a, long long b) const { return a + b; }
  BN_DEV static long long identity() { return 0; }
};
struct AddOpI {
  BN_DEV int operator()(int a, int b) const { return a + b; }
  BN_DEV static int identity() { return 0; }
};

}  // namespace bitnet

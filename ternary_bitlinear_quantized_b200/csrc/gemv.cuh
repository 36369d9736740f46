// Shared pieces of the BitLinear product: the register-fed int8 tensor-core step
// (mma.sync m16n8k32, u8 weights x s8 activations -> s32), the epilogue arithmetic
// (dequantisation, bf16 / fp32 store, the FFN activation with its fp64 exp) and the
// host-side description of a product launch.
//
// "fix: I2_S ARM kernel layout + squared-ReLU FFN - passes the gate on the official
// 2B4T GGUF", bullet "ggml-cpu: I2_S NEON kernel for the canonical layout": codes
// c = w + 1 in the interleaved 128/32 layout, and the caller subtracts the activation
// sum, so acc = sum q*c - sum q.  Field g of a 32-bit packed word (bits 7-2g:6-2g of each
// byte) holds the codes of 4 consecutive in-features, so masking the word with
// 0x03030303 << (6 - 2g) gives an mma A register directly -- the codes scaled by
// 4^(3-g), which stays in u8 range; each field accumulates separately and the sums are
// combined exactly (acc = D0/64 + D1/16 + D2/4 + D3).  The pairing of mma k-slots with
// in-features only has to agree between A and B (the dot product is order-free).
#pragma once
#include "common.cuh"

namespace bitnet {

constexpr int GEMV_ROWS = 16;  // weight rows of one mma tile

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

}  // namespace bitnet

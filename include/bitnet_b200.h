/*
 * bitnet_b200.h -- C ABI of the BitNet b1.58 BitLinear forward on NVIDIA B200 (sm_100a).
 *
 * The forward of one BitLinear: an RMSNorm on the activations (optional), per-token
 * absmax int8 quantisation of the activations, the integer product with absmean-ternary
 * weights stored as 2-bit I2_S codes, and the dequantising rescale.  On top of it, the
 * BitNet FFN block: gate/up -> relu2 or SiLU -> ffn_sub_norm -> down.
 *
 * Sources (web pages, by title):
 *   [RMS]  "Add optional RMSNorm support to BitNet quantization (config + layers)"
 *          (transformers pull request 38087): use_rms_norm (default off) and
 *          rms_norm_eps (default 1e-6); BitLinear applies BitNetRMSNorm to the
 *          activations before quantisation; BitNetMLP.forward (review thread).
 *   [I2S]  "fix: I2_S ARM kernel layout + squared-ReLU FFN - passes the gate on the
 *          official 2B4T GGUF" (cpp-bitnet pull request 7): description bullets
 *          "I2_S NEON kernel for the canonical layout" (interleaved 128-weight / 32-byte
 *          blocks, codes c = w + 1, the callers subtract the activation sum),
 *          "llama-quantize I2_S emits the canonical layout" (one scale per tensor after
 *          the packed data, 28 zeroed trailer bytes), "squared-ReLU FFN" (relu2 vs
 *          SiLU chosen from config) and "Known gaps" (rows divisible by 128).
 *   [IQ1]  "More BitNet-like IQ1_S quantizations" (llama.cpp discussion 8722):
 *          BitNet b1.58 keeps 8-bit activations and ternary weights.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless stated otherwise, 16-byte aligned, to
 *     contiguous row-major tensors.  The caller allocates and owns every buffer; the
 *     library allocates no device memory.
 *   - Calls are asynchronous on stream `s` (a cudaStream_t; NULL = legacy default
 *     stream).  Kernels are launched with programmatic dependent launch: a kernel may
 *     start, and read its WEIGHTS (`packed`) and norm GAINS, while the previous kernel
 *     on `s` is still running; it reads activations only after that kernel has
 *     finished.  So weights and gains must not be written by the kernel that directly
 *     precedes the call on `s` unless that kernel finishes before this one is enqueued
 *     (any torch kernel or copy satisfies this; so does bitnet_pack_i2s).
 *   - Argument errors are returned before anything is launched.  A launch failure
 *     returns BITNET_ERR_CUDA; bitnet_last_error() gives the CUDA message (per thread).
 *   - T = 0 (no tokens) is valid and launches nothing.
 *   - Entry points are reentrant; the only global state is the device status word read
 *     by bitnet_get_device_status().
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bitnet_stream; /* the same handle as cudaStream_t */

typedef enum {
  BITNET_OK = 0,
  BITNET_ERR_NULL = 1,      /* a required pointer is NULL                               */
  BITNET_ERR_SHAPE = 2,     /* a size is negative/zero where it must be positive, K % 128 != 0 for
                               packed weights, or a size is beyond the supported maximum   */
  BITNET_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned                          */
  BITNET_ERR_DTYPE = 4,     /* unknown bitnet_dtype / bitnet_act value                    */
  BITNET_ERR_WORKSPACE = 5, /* workspace missing or smaller than the *_workspace_bytes() */
  BITNET_ERR_CUDA = 6,      /* a CUDA call failed; see bitnet_last_error()               */
  BITNET_ERR_TIMEOUT = 7    /* a kernel gave up a bounded wait (device status word)      */
} bitnet_status;

typedef enum { BITNET_BF16 = 0, BITNET_F32 = 1 } bitnet_dtype;
typedef enum { BITNET_RELU2 = 0, BITNET_SILU = 1 } bitnet_act;

/* Largest in-feature count K the norm/quant kernels accept (a whole row is staged in
 * shared memory as fp32). */
#define BITNET_MAX_K 49152

/* Size of an I2_S tensor of N rows and K in-features: N*K/4 bytes of codes followed by
 * a 32-byte trailer (fp32 scale, then 28 zero bytes).  [I2S] "llama-quantize I2_S emits
 * the canonical layout".  Returns 0 if N <= 0, K <= 0 or K % 128 != 0. */
size_t bitnet_i2s_packed_bytes(int64_t N, int64_t K);

/* Ternarise and pack latent fp32 weights W [N, K] into I2_S (`packed`, which must hold
 * bitnet_i2s_packed_bytes(N, K) bytes).
 *   beta = max(mean|W|, 1e-5)   (the mean is an exact fixed-point sum rounded once to fp32)
 *   s_w  = 1 / beta;  c = clamp(round_half_even(W * s_w), -1, 1) + 1  in {0, 1, 2}
 *   element k of row n (block b = (n*K + k) / 128, g = (k % 128) / 32, i = k % 32) goes to
 *   byte 32 b + i, bits (7 - 2g):(6 - 2g); fp32 beta (little endian) at byte N*K/4, then
 *   28 zero bytes.
 * [I2S] "I2_S NEON kernel for the canonical layout", "llama-quantize I2_S emits the
 * canonical layout"; rows divisible by 128 per "Known gaps".  The trailer is used as
 * scratch during the call.  Errors: NULL, SHAPE (K % 128 != 0, N or K <= 0), ALIGN. */
bitnet_status bitnet_pack_i2s(const float* W, int64_t N, int64_t K, uint8_t* packed,
                              bitnet_stream s);

/* The same packing for weights that are already ternary x scale, with the scale taken the
 * BitNet way: beta = |w| of the first non-zero weight in row-major order (1e-5 if all are
 * zero, when every code is the zero weight anyway), then s_w, codes and trailer as above;
 * exactly ternary x scale inputs get their ternary values back as codes.
 * [I2S] "Known gaps": quantize_i2_s keeps the BitNet convention (scale = first non-zero
 * |w|), so inputs must already be ternary x scale.  Errors as bitnet_pack_i2s. */
bitnet_status bitnet_pack_i2s_prescaled(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                        bitnet_stream s);

/* Validate an I2_S tensor of N x K weights (N*K/4 code bytes + 32-byte trailer) on the
 * device.  counts: DEVICE int64[3], 8-byte aligned, overwritten asynchronously with
 *   counts[0]  2-bit fields holding 3 (no ternary weight maps to it),
 *   counts[1]  non-zero bytes among the 28 trailer bytes after the scale,
 *   counts[2]  1 if the stored fp32 scale is not finite and positive, else 0.
 * A tensor written by bitnet_pack_i2s(_prescaled) gives {0, 0, 0}.
 * [I2S] "llama-quantize I2_S emits the canonical layout": ggml_validate_row_data accepts
 * I2_S.  Errors: NULL, SHAPE (as bitnet_pack_i2s), ALIGN (packed 16 bytes, counts 8). */
bitnet_status bitnet_validate_i2s(const uint8_t* packed, int64_t N, int64_t K, int64_t* counts, bitnet_stream s);

/* BitNetRMSNorm + per-token absmax int8 quantisation of x [T, K] (bf16 or fp32).
 *   with gain:  ms = mean(x^2) (exact fixed-point sum, rounded once to fp32),
 *               inv = 1 / sqrt(ms + eps),  y = (x * inv) * gain      (fp32, no FMA)
 *   gain NULL:  y = x   (use_rms_norm off)
 *   s_x[t] = 127 / max(max|y|, 1e-5);  q = clamp(round_half_even(y * s_x), -128, 127);
 *   sum_q[t] = sum_k q[t, k]  (the activation sum the I2_S product subtracts)
 * [RMS] use_rms_norm / rms_norm_eps; [IQ1] 8-bit activations.
 * Outputs: q int8 [T, K], s_x fp32 [T], sum_q int32 [T].  1 <= K <= BITNET_MAX_K.
 * Errors: NULL, SHAPE, ALIGN, DTYPE. */
bitnet_status bitnet_rmsnorm_quant_act(const void* x, bitnet_dtype xt, const float* gain,
                                       float eps, int64_t T, int64_t K, int8_t* q,
                                       float* s_x, int32_t* sum_q, bitnet_stream s);

/* One BitLinear product after bitnet_rmsnorm_quant_act:
 *   acc[t, n] = sum_k q[t, k] * c[n, k] - sum_q[t]        (int32, = sum_k q * w exactly)
 *   out[t, n] = fp32(acc) * (beta / s_x[t])               (beta from the packed trailer)
 * written as bf16 (round to nearest even) or fp32 into out [T, N].  If acc_debug is not
 * NULL the int32 accumulators are also written there ([T, N]).  [I2S] "I2_S NEON kernel
 * for the canonical layout" (codes c = w + 1, activation-sum correction).
 * Requires K % 128 == 0.  Errors: NULL, SHAPE, ALIGN, DTYPE. */
bitnet_status bitnet_bitlinear(const int8_t* q, const float* s_x, const int32_t* sum_q,
                               const uint8_t* packed, int64_t T, int64_t N, int64_t K,
                               void* out, bitnet_dtype ot, int32_t* acc_debug,
                               bitnet_stream s);

/* Several BitLinears that share one quantised input (the q, k, v projections of a
 * decoder block) in one launch.  `packed`, `N` and `out` are HOST arrays of n_tensors
 * (1..4) entries; each tensor keeps its own scale.  Same arithmetic and errors as
 * bitnet_bitlinear. */
bitnet_status bitnet_bitlinear_group(const int8_t* q, const float* s_x, const int32_t* sum_q,
                                     int n_tensors, const uint8_t* const* packed,
                                     const int64_t* N, int64_t T, int64_t K,
                                     void* const* out, bitnet_dtype ot, bitnet_stream s);

/* The gate/up half of the BitNet FFN with its activation fused into the epilogue:
 *   g = BitLinear(p_gate), u = BitLinear(p_up) on the same quantised input (fp32, internal)
 *   h[t, i] = act(g) * u   (relu2 or SiLU exactly as in bitnet_ffn_block)
 * p_gate, p_up: I2_S [I, K]; h: fp32 [T, I].  [RMS] BitNetMLP.forward (act_fn(gate_proj(x))
 * * up_proj(x)); [I2S] "bitnet-b1.58: squared-ReLU FFN".  Errors as bitnet_bitlinear. */
bitnet_status bitnet_bitlinear_gate_up_act(const int8_t* q, const float* s_x, const int32_t* sum_q,
                                           const uint8_t* p_gate, const uint8_t* p_up, int64_t T,
                                           int64_t I, int64_t K, bitnet_act act, float* h,
                                           bitnet_stream s);

/* The integer part of bitnet_bitlinear only: acc[t, n] = sum_k q[t, k] * c[n, k] - sum_q[t]
 * (int32 [T, N]); no scale is read and no float output is written.  With the activation
 * sum of a slice of the in-features (sum_q of that slice) and an I2_S tensor holding only
 * those in-features, acc is that slice's share of the product, and the shares of disjoint
 * slices add up exactly to the full product (tensor parallelism over K).  [I2S] "I2_S NEON
 * kernel for the canonical layout".  Errors: NULL, SHAPE, ALIGN. */
bitnet_status bitnet_bitlinear_acc(const int8_t* q, const int32_t* sum_q, const uint8_t* packed, int64_t T,
                                   int64_t N, int64_t K, int32_t* acc, bitnet_stream s);

/* out[t, n] = fp32(acc[t, n]) * (beta / s_x[t]) with beta from the trailer of `packed` (an I2_S
 * tensor of N x K weights): the dequantising epilogue of bitnet_bitlinear applied to int32
 * accumulators that were summed over ranks.  out: bf16 (nearest even) or fp32 [T, N].
 * Errors: NULL, SHAPE, ALIGN (packed), DTYPE. */
bitnet_status bitnet_dequant_acc(const int32_t* acc, const float* s_x, const uint8_t* packed, int64_t T,
                                 int64_t N, int64_t K, void* out, bitnet_dtype ot, bitnet_stream s);

/* ffn_sub_norm + absmax int8 of h [T, K_total] when each rank holds Ks of its columns (h [T, Ks]
 * fp32 here, the rank's gate/up shard; gain: the matching Ks entries of ffn_sub_norm or NULL).
 * Every reduction of the norm is exact (maxima and an integer fixed-point sum), so it is
 * finished over the ranks by all-reduces, and the result is bit-identical to the unsharded
 * bitnet_rmsnorm_quant_act of the whole row:
 *   shard_amax    amax[t] = max |h[t, :]| over this shard          -> all-reduce MAX over ranks
 *   shard_sumsq   S[t] = sum rint(h^2 2^e) over this shard, on the grid e of the whole row
 *                 (from the GLOBAL amax and K_total)                -> all-reduce SUM (int64)
 *   shard_ymax    inv[t] = 1/sqrt(mean + eps) (mean = fp32(S 2^-e / K_total)), and
 *                 ymax[t] = max |(h inv) gain| over this shard      -> all-reduce MAX
 *                 (gain NULL: inv = 1, ymax = the global amax; S is not read)
 *   shard_quant   s_x[t] = 127 / max(ymax, 1e-5) (global ymax), q = clamp(rint(y s_x)) [T, Ks],
 *                 sum_q[t] = this shard's sum of q (the shard's activation sum)
 * [RMS] BitNetMLP.forward (ffn_sub_norm over the whole intermediate row).  Per-token
 * arrays (amax, inv, ymax, s_x: fp32 [T]; S: int64 [T], 8-byte aligned; sum_q: int32 [T]) are
 * device memory.  Ks % 4 == 0; h, gain, q 16-byte aligned.  Errors: NULL, SHAPE, ALIGN. */
bitnet_status bitnet_subnorm_shard_amax(const float* h, int64_t T, int64_t Ks, float* amax, bitnet_stream s);
bitnet_status bitnet_subnorm_shard_sumsq(const float* h, int64_t T, int64_t Ks, const float* amax, int64_t K_total,
                                         int64_t* S, bitnet_stream s);
bitnet_status bitnet_subnorm_shard_ymax(const float* h, const float* gain, int64_t T, int64_t Ks, const float* amax,
                                        const int64_t* S, int64_t K_total, float eps, float* inv, float* ymax,
                                        bitnet_stream s);
bitnet_status bitnet_subnorm_shard_quant(const float* h, const float* gain, int64_t T, int64_t Ks, const float* inv,
                                         const float* ymax, int8_t* q, float* s_x, int32_t* sum_q, bitnet_stream s);

/* Workspace of bitnet_ffn_block, in bytes (0 if a size is invalid). */
size_t bitnet_ffn_workspace_bytes(int64_t T, int64_t H, int64_t I);

/* Byte offsets inside that workspace, so that a caller can read the intermediates after
 * a call: off[0] q_x int8 [T,H], off[1] s_x fp32 [T], off[2] sum_x int32 [T],
 * off[3] h fp32 [T,I], off[4] q_h int8 [T,I], off[5] s_h fp32 [T], off[6] sum_h int32 [T],
 * off[7] 256 bytes of grid-barrier counters, followed by the decode engine's per-CTA
 * partial reductions (no layout promised).  `off` is a HOST array of 8 entries.
 * Returns BITNET_ERR_SHAPE on invalid sizes. */
bitnet_status bitnet_ffn_workspace_offsets(int64_t T, int64_t H, int64_t I, size_t* off);

/* The BitNet FFN block on x [T, H]:
 *   (q_x, s_x, sum_x) = rmsnorm_quant(x, g_ffn)                 (ffn_norm; NULL = off)
 *   g = BitLinear(gate), u = BitLinear(up)                       (fp32 [T, I], internal)
 *   h = act(g) * u:  relu2: r = max(g, 0), h = (r*r)*u;
 *                    SiLU:  h = fp32(g / (1 + exp(-g))) * u, exp taken in fp64
 *   (q_h, s_h, sum_h) = rmsnorm_quant(h, g_sub)                  (ffn_sub_norm)
 *   out = BitLinear(down)                                        (bf16 or fp32 [T, H])
 * [RMS] BitNetMLP.forward = down(ffn_sub_norm(act(gate(x)) * up(x)));
 * [I2S] "bitnet-b1.58: squared-ReLU FFN" (relu2 vs SiLU from config).
 * p_gate, p_up: I2_S [I, H]; p_down: I2_S [H, I]; H % 128 == 0 and I % 128 == 0.
 * ws: device workspace of at least bitnet_ffn_workspace_bytes(T, H, I) bytes (16-byte
 * aligned).  Its barrier counters (off[7]) must be ZERO before the first call (allocate it
 * zeroed once); every call leaves them zero, except a call that ends in
 * BITNET_ERR_TIMEOUT, after which they must be zeroed again.  Up to 16 tokens the whole
 * block is one launch (grid barriers between the dependent steps); more tokens run as
 * separate launches on the tensor-core path.  Two calls that share a workspace must not
 * run concurrently.  Errors: NULL, SHAPE, ALIGN, DTYPE, WORKSPACE. */
bitnet_status bitnet_ffn_block(const void* x, bitnet_dtype xt, const float* g_ffn,
                               const uint8_t* p_gate, const uint8_t* p_up,
                               const float* g_sub, const uint8_t* p_down,
                               int64_t T, int64_t H, int64_t I, bitnet_act act, float eps,
                               void* out, bitnet_dtype ot, void* ws, size_t ws_bytes,
                               bitnet_stream s);

/* The same FFN block for callers that cannot allocate device memory themselves -- for
 * example a plugin running inside a host framework that owns all device memory and forbids
 * allocation while it serves, or a process under a hard memory cap.  (The BitNet pages
 * have no counterpart: this is an interface convenience, not part of the method.)
 *   - The workspace is a file-scope device array of bitnet_ffn_block_noalloc_max_bytes()
 *     bytes (4 MiB) inside the library; every GPU that loads the library holds it until
 *     the process exits.  Sizes whose workspace (bitnet_ffn_workspace_bytes) exceeds it
 *     are rejected with BITNET_ERR_WORKSPACE (bitnet_last_error() says why).
 *   - The call allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *     The first call on a device looks up the array's device address on that device
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Every call clears the grid-barrier counters of the array with cudaMemsetAsync on `s`
 *     before it launches; the rest of the array keeps the previous call's contents.
 *   - All calls share the one array per device, so calls that overlap on the GPU (other
 *     streams, other threads) race: serialise them.
 * Arguments, arithmetic and other errors as bitnet_ffn_block (without ws / ws_bytes). */
size_t bitnet_ffn_block_noalloc_max_bytes(void);
bitnet_status bitnet_ffn_block_noalloc(const void* x, bitnet_dtype xt, const float* g_ffn,
                                       const uint8_t* p_gate, const uint8_t* p_up,
                                       const float* g_sub, const uint8_t* p_down, int64_t T,
                                       int64_t H, int64_t I, bitnet_act act, float eps, void* out,
                                       bitnet_dtype ot, bitnet_stream s);

/* Workspace of bitnet_decoder_block, in bytes (0 if a size is invalid).  NQ = the q (and
 * o-input) width, usually H. */
size_t bitnet_block_workspace_bytes(int64_t T, int64_t H, int64_t NQ, int64_t I);

/* Byte offsets inside that workspace: off[0..2] q, s, sum of x (attn_norm) [T,H];
 * off[3..5] the same for the attention output (attn_sub_norm) [T,NQ]; off[6] the FFN's
 * workspace (layout of bitnet_ffn_workspace_offsets).  `off`: HOST array of 7 entries. */
bitnet_status bitnet_block_workspace_offsets(int64_t T, int64_t H, int64_t NQ, int64_t I, size_t* off);

/* The BitLinear projections of one BitNet decoder block, in dependency order:
 *   q, k, v = BitLinear_{p_q, p_k, p_v}(rmsnorm_quant(x, g_attn_norm))      -> out_q/k/v
 *   o       = BitLinear_{p_o}(rmsnorm_quant(attn_out, g_attn_sub_norm))       -> out_o [T,H]
 *   ffn     = bitnet_ffn_block(o; g_ffn_norm, gate, up, g_ffn_sub_norm, down) -> out_ffn [T,H]
 * x [T,H] and attn_out [T,NQ] are the block input and the attention output (the
 * attention itself, rotary embedding and residual adds are not part of this call).
 * Shapes: p_q [NQ,H], p_k / p_v [NKV,H], p_o [H,NQ], p_gate / p_up [I,H], p_down [H,I].
 * [RMS] BitLinear with BitNetRMSNorm on its input, BitNetMLP.forward with ffn_sub_norm;
 * [IQ1] the per-block norm weights attn_norm, attn_sub_norm, ffn_norm, ffn_sub_norm.
 * Outputs are bf16 or fp32 (ot).  Up to 16 tokens the block is ONE launch; the workspace
 * (bitnet_block_workspace_bytes) follows the rules of bitnet_ffn_block (zero it once).
 * Errors: NULL, SHAPE, ALIGN, DTYPE, WORKSPACE. */
bitnet_status bitnet_decoder_block(const void* x, const void* attn_out, bitnet_dtype xt,
                                   const float* g_attn_norm, const float* g_attn_sub_norm,
                                   const float* g_ffn_norm, const float* g_ffn_sub_norm,
                                   const uint8_t* p_q, const uint8_t* p_k, const uint8_t* p_v,
                                   const uint8_t* p_o, const uint8_t* p_gate, const uint8_t* p_up,
                                   const uint8_t* p_down, int64_t T, int64_t H, int64_t NQ,
                                   int64_t NKV, int64_t I, bitnet_act act, float eps, void* out_q,
                                   void* out_k, void* out_v, void* out_o, void* out_ffn,
                                   bitnet_dtype ot, void* ws, size_t ws_bytes, bitnet_stream s);

/* The attention between a block's q/k/v and o projections at decode (the rest of the
 * decoder block).  The BitNet pages keep the transformer's attention and only replace its
 * linear layers ("Add BitNet" in flash-linear-attention: transformer code with nn.Linear
 * swapped for BitLinear; [IQ1] the per-block attn_q/k/v/output tensors), so these compute the
 * textbook form.  Head size d must be 128.
 *
 * bitnet_rope_kv_append: rotary embedding of q [T, Hq, d] and k [T, Hkv, d] (bf16 or fp32,
 * the projections' outputs) at positions pos0 + t: for i < d/2 the pair (x_i, x_{i+d/2})
 * turns by a = p theta^(-2i/d) (angle, sine and cosine in fp64, the rotation in fp32).  The
 * rotated q goes to q_rot (fp32 [T, Hq, d]); the rotated k and the unchanged v are appended
 * to the KV cache k_cache / v_cache (bf16 [Hkv][L_max][d], rows pos0 .. pos0 + T - 1, rounded
 * to nearest even).  Errors: NULL, SHAPE (d != 128, Hq % Hkv, pos0 + T > L_max, theta <= 0),
 * DTYPE. */
bitnet_status bitnet_rope_kv_append(const void* q, const void* k, const void* v, bitnet_dtype xt, int64_t T,
                                    int64_t Hq, int64_t Hkv, int64_t d, int64_t pos0, double theta, float* q_rot,
                                    void* k_cache, void* v_cache, int64_t L_max, bitnet_stream s);

/* Workspace of bitnet_attention_decode for L cache rows in use, in bytes (0 if invalid). */
size_t bitnet_attention_workspace_bytes(int64_t T, int64_t Hq, int64_t Hkv, int64_t L);

/* Causal grouped-query attention of T new tokens (positions pos0 .. pos0 + T - 1, already in
 * the cache) against cache rows 0 .. pos0 + t: out[t, h] = softmax(q_rot[t, h] . k / sqrt(d)) v
 * with key/value head h / (Hq / Hkv), in fp32 (split over 64-row chunks of the cache, merged
 * exactly as running maxima and sums), written as bf16 or fp32 [T, Hq, d].  T * Hq / Hkv <= 128,
 * pos0 + T <= 65536 (SHAPE otherwise).
 * ws: bitnet_attention_workspace_bytes(T, Hq, Hkv, pos0 + T) bytes, 16-byte aligned.
 * Errors: NULL, SHAPE, ALIGN, DTYPE, WORKSPACE. */
bitnet_status bitnet_attention_decode(const float* q_rot, const void* k_cache, const void* v_cache, int64_t T,
                                      int64_t Hq, int64_t Hkv, int64_t d, int64_t pos0, int64_t L_max, void* out,
                                      bitnet_dtype ot, void* ws, size_t ws_bytes, bitnet_stream s);

/* Synchronises `s`, then reads and clears the device status word of the current
 * device: BITNET_OK, or BITNET_ERR_TIMEOUT if a kernel gave up a bounded wait since
 * the last read. */
bitnet_status bitnet_get_device_status(bitnet_stream s);

/* Test and debugging aid (no counterpart on the pages): sets the limit of every bounded wait
 * in the kernels on the CURRENT device, in SM clock cycles (<= 0 restores the default of
 * 2e9, about a second).  A wait that runs past the limit gives up, sets BITNET_ERR_TIMEOUT in
 * the device status word and the kernel returns early with its outputs incomplete (it still
 * lets its own in-flight copies land, with a fixed limit).  Tests use a short limit to make
 * waits run out on purpose.  Synchronises the device before and after; call it only while no
 * kernel of this library runs.  Errors: CUDA. */
bitnet_status bitnet_debug_set_wait_limit(long long cycles);

/* Static English text of a status code. */
const char* bitnet_status_string(bitnet_status st);

/* The CUDA error text of the last BITNET_ERR_CUDA on this thread ("" if none). */
const char* bitnet_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* BITNET_B200_H */

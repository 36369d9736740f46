"""CPU oracle of the BitNet b1.58 BitLinear forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline``
leg and its ``--impl reference`` arm) may import this module.  The product path
(``ternary_bitlinear_quantized_b200``) never imports, calls or links it, and this
module imports nothing from the product path.

Plain numpy, written for reading, not speed.  Every quantity that decides an integer
(a weight code, an int8 activation) is taken in fp32, the precision the CUDA kernels
take it in; the exact sums that feed those decisions are integer (fixed-point) sums,
so their result does not depend on the order of summation.  A library matmul serves
as the integer dot product: it runs in fp64 on integer operands whose every partial
sum stays below 2**53, so its result is exact.

What each function follows (pages by title):

* "Add optional RMSNorm support to BitNet quantization (config + layers)"
  (transformers pull request): ``use_rms_norm`` / ``rms_norm_eps`` (default 1e-6);
  BitLinear applies BitNetRMSNorm to the activations before quantising them;
  ``BitNetMLP.forward`` = down(ffn_sub_norm(act(gate(x)) * up(x))).
* "fix: I2_S ARM kernel layout + squared-ReLU FFN - passes the gate on the official
  2B4T GGUF" (cpp-bitnet pull request), description bullets "I2_S NEON kernel for the
  canonical layout" and "llama-quantize I2_S emits the canonical layout": 2-bit codes
  c = w + 1 whose dot product is corrected by the activation sum; the interleaved
  128-weight / 32-byte block layout; one scale per tensor stored after the packed data;
  the zeroed trailer; rows divisible by 128; relu2 vs SiLU chosen from config.
* BitNet b1.58 quantisers (absmean ternary weights, per-token absmax int8 activations),
  as named by both pages above and by "More BitNet-like IQ1_S quantizations"
  (llama.cpp discussion: 8-bit activations, ternary weights).

Readings where the pages are silent:

* bit order inside an I2_S block: element 128 b + 32 g + i is byte 32 b + i, bits
  (7 - 2g):(6 - 2g) -- the interleaved layout, as opposed to the "sequential (byte
  i/4, field i%4)" order the cpp-bitnet page calls wrong;
* trailer: fp32 scale beta (little endian) then 28 zero bytes (32 bytes in all);
* round() is round-half-to-even;
* mean(x^2) and mean|W| are exact fixed-point sums (``fixed_point_mean_f32``) rounded
  once to fp32; everything after them is a sequence of single IEEE fp32 operations;
* the dequantisation factor is beta / s_x (= 1 / (s_x * s_w)) rounded to fp32, then
  out = fp32(acc) * factor;
* SiLU's exp is the fp64 ``pinned_exp`` below.

Parity status: every function here is pinned by ``tests/test_oracle.py`` (golden bytes,
closed forms, invariants, brute force).  No function is "parity unpinned".
"""
from __future__ import annotations

import decimal
import math

import numpy as np

F32 = np.float32
F64 = np.float64
QBLOCK = 128          # weights per I2_S block
QBLOCK_BYTES = 32     # bytes per I2_S block
TRAILER_BYTES = 32    # fp32 scale + 28 zero bytes
ABS_FLOOR = F32(1e-5)  # the 1e-5 floor of both absmax and absmean


# ----------------------------------------------------------------------------- sums

def fixed_point_grid(M: float, n: int) -> int:
    """Grid exponent e of an order-free sum of n non-negative terms whose largest is M > 0:
    with M = m 2**E (0.5 <= m < 1) and 2**L >= n, e = 62 - E - L, so that every scaled term
    is below 2**(62 - L) and n of them sum below 2**62 in int64."""
    _, E = math.frexp(float(M))
    L = (int(n) - 1).bit_length()
    return 62 - E - L


def fixed_point_sum_on_grid(terms: np.ndarray, e: int) -> int:
    """Sum of rint(term * 2**e) over ``terms`` (each scaled exactly, rounded half-to-even to
    an integer); the integer sum is the same in any order and over any split of the terms."""
    terms = np.asarray(terms, dtype=F64).ravel()
    if terms.size == 0:
        return 0
    return int(np.rint(np.ldexp(terms, e)).astype(np.int64).sum(dtype=np.int64))


def fixed_point_sum(terms: np.ndarray) -> tuple[int, int]:
    """Order-free sum of non-negative fp64 ``terms`` on the fixed-point grid of
    ``fixed_point_grid(max(terms), n)``.  Returns (S, e)."""
    terms = np.asarray(terms, dtype=F64).ravel()
    n = terms.size
    if n == 0:
        return 0, 0
    M = float(terms.max())
    if M == 0.0:
        return 0, 0
    e = fixed_point_grid(M, n)
    return fixed_point_sum_on_grid(terms, e), e


def fixed_point_mean_f32(terms: np.ndarray) -> np.float32:
    """fp32( (fp64(S) * 2**-e) / n ): the mean of ``terms`` from ``fixed_point_sum``."""
    terms = np.asarray(terms, dtype=F64).ravel()
    S, e = fixed_point_sum(terms)
    if S == 0:
        return F32(0.0)
    return F32(math.ldexp(float(S), -e) / float(terms.size))


# ----------------------------------------------------------------------------- bf16

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 exactly."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(F32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# ----------------------------------------------------------------------------- a1: pack

def i2s_packed_bytes(N: int, K: int) -> int:
    """N*K/4 bytes of 2-bit codes, then the 32-byte trailer."""
    return N * K // 4 + TRAILER_BYTES


def absmean_scale(W: np.ndarray) -> np.float32:
    """beta = max(mean|W|, 1e-5): the per-tensor weight scale (s_w = 1 / beta)."""
    return np.maximum(fixed_point_mean_f32(np.abs(np.asarray(W, dtype=F32)).astype(F64)), ABS_FLOOR)


def ternary_codes(W: np.ndarray, beta: np.float32) -> np.ndarray:
    """c = clamp(round(W * s_w), -1, 1) + 1 with s_w = 1 / beta, in fp32."""
    s_w = F32(1.0) / F32(beta)
    w = np.asarray(W, dtype=F32) * s_w
    return (np.clip(np.rint(w), -1, 1) + 1).astype(np.uint8)


def interleave_i2s(codes: np.ndarray) -> np.ndarray:
    """Codes [N, K] (values 0..2) -> N*K/4 bytes in the interleaved 128/32 layout."""
    N, K = codes.shape
    blk = codes.reshape(N * K // QBLOCK, 4, QBLOCK_BYTES).astype(np.uint8)  # [b, g, i]
    out = (blk[:, 0, :] << 6) | (blk[:, 1, :] << 4) | (blk[:, 2, :] << 2) | blk[:, 3, :]
    return out.reshape(-1).astype(np.uint8)


def pack_i2s(W: np.ndarray) -> np.ndarray:
    """Latent fp32 weights [N, K] -> I2_S bytes [N*K/4 + 32] (codes, fp32 beta, 28 zeros)."""
    W = np.asarray(W, dtype=F32)
    N, K = W.shape
    if K % QBLOCK != 0:
        raise ValueError("I2_S needs rows divisible by 128")
    beta = absmean_scale(W)
    body = interleave_i2s(ternary_codes(W, beta))
    trailer = np.zeros(TRAILER_BYTES, dtype=np.uint8)
    trailer[:4] = np.frombuffer(np.asarray([beta], dtype="<f4").tobytes(), dtype=np.uint8)
    return np.concatenate([body, trailer])


def first_nonzero_scale(W: np.ndarray) -> np.float32:
    """beta = |w| of the first non-zero weight in row-major order: the BitNet convention that
    quantize_i2_s keeps for inputs that are already ternary x scale ("fix: I2_S ARM kernel
    layout + squared-ReLU FFN", "Known gaps").  An all-zero tensor has no such weight; its
    codes are all zero weights whatever the scale, and 1e-5 (the absmean floor) is stored."""
    flat = np.asarray(W, dtype=F32).reshape(-1)
    nz = np.flatnonzero(flat != 0)
    return F32(abs(flat[nz[0]])) if nz.size else ABS_FLOOR


def pack_i2s_prescaled(W: np.ndarray) -> np.ndarray:
    """Ternary x scale fp32 weights [N, K] -> I2_S bytes, with beta = first_nonzero_scale(W)
    and the codes of ternary_codes (for exactly ternary x scale inputs, w * (1 / beta) rounds
    to -1, 0 or 1, the ternary value itself)."""
    W = np.asarray(W, dtype=F32)
    N, K = W.shape
    if K % QBLOCK != 0:
        raise ValueError("I2_S needs rows divisible by 128")
    beta = first_nonzero_scale(W)
    body = interleave_i2s(ternary_codes(W, beta))
    trailer = np.zeros(TRAILER_BYTES, dtype=np.uint8)
    trailer[:4] = np.frombuffer(np.asarray([beta], dtype="<f4").tobytes(), dtype=np.uint8)
    return np.concatenate([body, trailer])


def validate_i2s(packed: np.ndarray, N: int, K: int) -> tuple[int, int, int]:
    """Checks of an I2_S tensor, the row-data validation that llama.cpp's
    ggml_validate_row_data gains for I2_S in the same pull request (bullet "llama-quantize
    I2_S emits the canonical layout"): (2-bit fields holding 3, which no ternary weight
    maps to; non-zero bytes among the 28 trailer bytes after the scale; 1 if the stored
    scale is not a finite positive fp32, else 0)."""
    packed = np.asarray(packed, dtype=np.uint8)
    nb = N * K // 4
    body = packed[:nb]
    bad_codes = int(sum(int(np.count_nonzero(((body >> (2 * g)) & 3) == 3)) for g in range(4)))
    trailer = packed[nb:nb + TRAILER_BYTES]
    bad_trailer = int(np.count_nonzero(trailer[4:]))
    beta = np.frombuffer(trailer[:4].tobytes(), dtype="<f4")[0]
    bad_scale = 0 if (np.isfinite(beta) and beta > 0) else 1
    return bad_codes, bad_trailer, bad_scale


def unpack_i2s(packed: np.ndarray, N: int, K: int) -> tuple[np.ndarray, np.float32]:
    """I2_S bytes -> (codes uint8 [N, K], beta)."""
    packed = np.asarray(packed, dtype=np.uint8)
    body = packed[: N * K // 4].reshape(N * K // QBLOCK, QBLOCK_BYTES)
    codes = np.empty((N * K // QBLOCK, 4, QBLOCK_BYTES), dtype=np.uint8)
    for g in range(4):
        codes[:, g, :] = (body >> (6 - 2 * g)) & 0x3
    beta = np.frombuffer(packed[N * K // 4: N * K // 4 + 4].tobytes(), dtype="<f4")[0]
    return codes.reshape(N, K), F32(beta)


# ----------------------------------------------------------------------------- a2: norm + quant

def rmsnorm_quant_act(x: np.ndarray, gain: np.ndarray | None, eps: float):
    """x fp32 [T, K] (bf16 values widened, or fp32 h) -> (q int8 [T,K], s_x fp32 [T], sum_q int32 [T]).

    With a gain: ms = mean(x^2) (fixed point), inv = 1 / sqrt(ms + eps), y = (x * inv) * g.
    Without one (use_rms_norm off): y = x.  Then s_x = 127 / max(max|y|, 1e-5),
    q = clamp(round(y * s_x), -128, 127) and sum_q = sum(q).
    """
    x = np.atleast_2d(np.asarray(x, dtype=F32))
    T, K = x.shape
    q = np.zeros((T, K), dtype=np.int8)
    s_x = np.zeros(T, dtype=F32)
    for t in range(T):
        row = x[t]
        if gain is not None:
            ms = fixed_point_mean_f32(row.astype(F64) * row.astype(F64))
            inv = F32(1.0) / np.sqrt(ms + F32(eps))
            y = (row * inv) * np.asarray(gain, dtype=F32)
        else:
            y = row
        a = np.max(np.abs(y)) if K else F32(0.0)
        s = F32(127.0) / np.maximum(F32(a), ABS_FLOOR)
        q[t] = np.clip(np.rint(y * s), -128, 127).astype(np.int8)
        s_x[t] = s
    sum_q = q.astype(np.int64).sum(axis=1).astype(np.int32)
    return q, s_x, sum_q


# ----------------------------------------------------------------------------- a6 split over ranks

# ffn_sub_norm when each rank holds some columns of h (tensor parallelism over the FFN's
# intermediate dimension, the split the gate/up projections produce).  The same arithmetic
# as rmsnorm_quant_act, taken in stages whose partial results are combined over the ranks
# by maxima and integer sums; the combination is exact, so the result equals
# rmsnorm_quant_act of the whole row.

def shard_amax(h: np.ndarray) -> np.ndarray:
    """max |h| of each row of this shard (combined over ranks by a maximum)."""
    h = np.atleast_2d(np.asarray(h, dtype=F32))
    return np.max(np.abs(h), axis=1) if h.shape[1] else np.zeros(h.shape[0], F32)


def shard_sumsq(h: np.ndarray, amax: np.ndarray, n_total: int) -> np.ndarray:
    """This shard's part of the fixed-point sum of h^2 on the grid of the whole row (from
    the global max |h| and the global row length); combined over ranks by a sum."""
    h = np.atleast_2d(np.asarray(h, dtype=F32))
    out = np.zeros(h.shape[0], dtype=np.int64)
    for t in range(h.shape[0]):
        a = float(amax[t])
        if a > 0.0:
            e = fixed_point_grid(a * a, n_total)
            out[t] = fixed_point_sum_on_grid(h[t].astype(F64) * h[t].astype(F64), e)
    return out


def shard_ymax(h, gain, amax, S, n_total: int, eps: float):
    """inv = 1 / sqrt(mean(h^2) + eps) of the whole row (from the combined sum) and this
    shard's max |y|, y = (h * inv) * g (no gain: inv = 1 and y = h).  Returns (inv, ymax)."""
    h = np.atleast_2d(np.asarray(h, dtype=F32))
    T = h.shape[0]
    inv = np.ones(T, dtype=F32)
    ymax = np.zeros(T, dtype=F32)
    for t in range(T):
        if gain is None:
            ymax[t] = amax[t]
            continue
        a = float(amax[t])
        ms = F32(0.0)
        if a > 0.0 and S[t] != 0:
            e = fixed_point_grid(a * a, n_total)
            ms = F32(math.ldexp(float(S[t]), -e) / float(n_total))
        inv[t] = F32(1.0) / np.sqrt(ms + F32(eps))
        y = (h[t] * inv[t]) * np.asarray(gain, dtype=F32)
        ymax[t] = np.max(np.abs(y)) if y.size else F32(0.0)
    return inv, ymax


def shard_quant(h, gain, inv, ymax):
    """s_x = 127 / max(global max |y|, 1e-5); this shard's q and its partial sum of q."""
    h = np.atleast_2d(np.asarray(h, dtype=F32))
    T, Ks = h.shape
    q = np.zeros((T, Ks), dtype=np.int8)
    s = np.zeros(T, dtype=F32)
    for t in range(T):
        y = h[t] if gain is None else (h[t] * F32(inv[t])) * np.asarray(gain, dtype=F32)
        s[t] = F32(127.0) / np.maximum(F32(ymax[t]), ABS_FLOOR)
        q[t] = np.clip(np.rint(y * s[t]), -128, 127).astype(np.int8)
    return q, s, q.astype(np.int64).sum(axis=1).astype(np.int32)


# ----------------------------------------------------------------------------- a3/a4: dot + dequant

def bitlinear_acc(q: np.ndarray, sum_q: np.ndarray, packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """acc[t, n] = sum_k q[t,k] c[n,k] - sum_q[t]  (= sum_k q[t,k] w[n,k], w = c - 1), int32."""
    codes, _ = unpack_i2s(packed, N, K)
    qf = np.asarray(q, dtype=F64)
    acc_c = qf @ codes.astype(F64).T
    acc = acc_c - np.asarray(sum_q, dtype=F64)[:, None]
    acc_w = qf @ (codes.astype(F64) - 1.0).T
    assert np.array_equal(acc, acc_w), "sum q*c - sum q must equal sum q*w"
    assert np.all(np.abs(acc) < 2 ** 31)
    return acc.astype(np.int32)


def dequant(acc: np.ndarray, s_x: np.ndarray, beta: np.float32) -> np.ndarray:
    """out = fp32(acc) * (beta / s_x), both fp32 operations."""
    f = F32(beta) / np.asarray(s_x, dtype=F32)
    return np.asarray(acc, dtype=np.int32).astype(F32) * f[:, None]


def bitlinear(q, s_x, sum_q, packed, N, K, out_dtype="f32", return_acc=False):
    """One BitLinear after activation quantisation; out fp32 [T, N] (bf16-rounded if asked)."""
    acc = bitlinear_acc(q, sum_q, packed, N, K)
    _, beta = unpack_i2s(packed, N, K)
    out = dequant(acc, s_x, beta)
    if out_dtype == "bf16":
        out = round_to_bf16(out)
    return (out, acc) if return_acc else out


# ----------------------------------------------------------------------------- a5: activation

_LN2_DEC = decimal.Context(prec=60).ln(decimal.Decimal(2))  # ln 2 to 60 digits
_LN2 = float(_LN2_DEC)
# ln 2 split so that k * _LN2_HI is exact for |k| < 2**11 (Cody and Waite's reduction):
# _LN2_HI keeps the top 32 significant bits of ln 2, _LN2_LO is the rest, rounded to fp64.
_LN2_HI = float(np.frombuffer((np.frombuffer(np.float64(_LN2).tobytes(), np.uint64)
                               & np.uint64(0xFFFFFFFFFFE00000)).tobytes(), np.float64)[0])
_LN2_LO = float(decimal.Context(prec=60).subtract(_LN2_DEC, decimal.Decimal(_LN2_HI)))
_EXP_TAYLOR = [1.0 / math.factorial(n) for n in range(18)]  # degree-17 Taylor series of exp


def pinned_exp(x: np.ndarray) -> np.ndarray:
    """exp in fp64 with a fixed operation sequence (so that any IEEE fp64 machine agrees):
    k = rint(x / ln2); r = (x - k ln2_hi) - k ln2_lo; p = Taylor(r) in Horner form;
    exp = p * 2**k.  Below -700 the result is 0, above 709 it is +inf."""
    x = np.asarray(x, dtype=F64)
    k = np.rint(x / _LN2)
    r = (x - k * _LN2_HI) - k * _LN2_LO
    p = np.full_like(r, _EXP_TAYLOR[17])
    for n in range(16, -1, -1):
        p = p * r + _EXP_TAYLOR[n]
    small = x < -700.0
    big = x > 709.0
    kk = np.where(small | big, 0, k).astype(np.int64)
    out = np.ldexp(p, kk)
    out = np.where(small, 0.0, out)
    return np.where(big, np.inf, out)


def ffn_act(g: np.ndarray, u: np.ndarray, act: str) -> np.ndarray:
    """h = act(g) * u in fp32.  relu2: r = max(g, 0), h = (r*r)*u.
    SiLU: s = fp32(g / (1 + exp(-g))) in fp64 with ``pinned_exp``, h = s*u."""
    g = np.asarray(g, dtype=F32)
    u = np.asarray(u, dtype=F32)
    if act == "relu2":
        r = np.maximum(g, F32(0.0))
        return (r * r) * u
    if act == "silu":
        gd = g.astype(F64)
        s = (gd / (1.0 + pinned_exp(-gd))).astype(F32)
        return s * u
    raise ValueError(act)


# ----------------------------------------------------------------------------- composed paths

def bitlinear_from_x(x, gain, eps, packed, N, K, out_dtype="f32"):
    q, s, sq = rmsnorm_quant_act(x, gain, eps)
    return bitlinear(q, s, sq, packed, N, K, out_dtype)


def ffn_block(x, g_ffn, p_gate, p_up, g_sub, p_down, H, I, act, eps, out_dtype="bf16",
              return_intermediates=False):
    """BitNetMLP: down(ffn_sub_norm(act(gate(x)) * up(x))), each projection a BitLinear;
    gate and up share the quantised input (ffn_norm)."""
    q, s, sq = rmsnorm_quant_act(x, g_ffn, eps)
    g = bitlinear(q, s, sq, p_gate, I, H, "f32")
    u = bitlinear(q, s, sq, p_up, I, H, "f32")
    h = ffn_act(g, u, act)
    q2, s2, sq2 = rmsnorm_quant_act(h, g_sub, eps)
    out = bitlinear(q2, s2, sq2, p_down, H, I, out_dtype)
    if return_intermediates:
        return out, dict(q=q, s_x=s, sum_q=sq, g=g, u=u, h=h, q_h=q2, s_h=s2, sum_h=sq2)
    return out


def decoder_block(x, attn_out, gains: dict, packed: dict, shape: dict, act, eps, out_dtype="bf16"):
    """The BitLinear projections of one decoder block: q,k,v from x through attn_norm;
    o from the (synthetic) attention output through attn_sub_norm; the FFN from o's
    output.  ``shape`` maps tensor name -> (N, K).  Returns a dict of outputs."""
    out = {}
    q, s, sq = rmsnorm_quant_act(x, gains["attn_norm"], eps)
    for nm in ("q", "k", "v"):
        N, K = shape[nm]
        out[nm] = bitlinear(q, s, sq, packed[nm], N, K, out_dtype)
    N, K = shape["o"]
    out["o"] = bitlinear_from_x(attn_out, gains["attn_sub_norm"], eps, packed["o"], N, K, out_dtype)
    I, H = shape["gate"]
    out["ffn"] = ffn_block(out["o"], gains["ffn_norm"], packed["gate"], packed["up"],
                           gains["ffn_sub_norm"], packed["down"], H, I, act, eps, out_dtype)
    return out


# ----------------------------------------------------------------------------- the rest of the block

# The attention between the q/k/v and o projections of a decoder block.  The pages keep the
# transformer's attention and only swap its linear layers for BitLinear ("Add BitNet" in
# flash-linear-attention: the transformer code with nn.Linear replaced; "More BitNet-like
# IQ1_S quantizations": per-block attn_q/k/v/output and attn_norm/attn_sub_norm tensors).
# They do not print it, so it is written here in its textbook form, in fp64: rotary position
# embedding on q and k (the rotate-half pairing of dimensions i and i + d/2, frequency
# theta^(-2i/d)), then causal scaled dot-product attention with grouped key/value heads.

def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """theta^(-2i/d) for i < d/2, in fp64."""
    return np.power(float(theta), -2.0 * np.arange(d // 2, dtype=F64) / float(d))


def apply_rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """x [T, H, d] at token positions [T] -> rotated copy (fp64): for i < d/2,
    (x_i, x_{i+d/2}) -> (x_i cos a - x_{i+d/2} sin a, x_{i+d/2} cos a + x_i sin a), a = p theta^(-2i/d)."""
    x = np.asarray(x, dtype=F64)
    T, H, d = x.shape
    ang = np.asarray(positions, dtype=F64)[:, None] * rope_inv_freq(d, theta)[None, :]  # [T, d/2]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: np.ndarray) -> np.ndarray:
    """Causal grouped-query attention in fp64.  q [T, Hq, d] (already rotated) at positions
    q_pos [T]; k, v [L, Hkv, d] (keys already rotated) at positions 0..L-1.  Query head h uses
    key/value head h // (Hq / Hkv); a query at position p sees keys 0..p.  Returns [T, Hq, d]:
    softmax(q . k / sqrt(d)) v."""
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    T, Hq, d = q.shape
    L, Hkv, _ = k.shape
    group = Hq // Hkv
    out = np.zeros((T, Hq, d), dtype=F64)
    for t in range(T):
        n = int(q_pos[t]) + 1
        for h in range(Hq):
            kh = h // group
            s = (k[:n, kh, :] @ q[t, h, :]) / math.sqrt(d)
            w = np.exp(s - s.max())
            out[t, h] = (w / w.sum()) @ v[:n, kh, :]
    return out

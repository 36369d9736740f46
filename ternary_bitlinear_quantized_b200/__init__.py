"""Python binding of libbitnet_b200.so: the BitNet b1.58 BitLinear forward on B200.

Argument marshalling only -- every step of the arithmetic runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (the library allocates no device memory:
outputs and workspaces are allocated here with torch and passed down); calls are
enqueued on torch's current stream.  The library must have been built
(``python -m ternary_bitlinear_quantized_b200.build``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "lib", "i2s_packed_bytes", "pack_i2s", "rmsnorm_quant_act", "bitlinear", "bitlinear_group", "bitlinear_gate_up_act",
    "ffn_workspace_bytes", "ffn_workspace_offsets", "ffn_block", "ffn_block_noalloc", "block_workspace_bytes", "block_workspace_offsets",
    "decoder_block", "device_status", "BitnetError",
    "BF16", "F32", "RELU2", "SILU",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet_b200.so")

BF16, F32 = 0, 1
RELU2, SILU = 0, 1
_STATUS = {0: "ok", 1: "null pointer", 2: "invalid shape", 3: "pointer not 16-byte aligned",
           4: "invalid dtype or activation", 5: "workspace missing or too small", 6: "CUDA error",
           7: "kernel wait timed out"}

EXPORTS = [
    "bitnet_i2s_packed_bytes", "bitnet_pack_i2s", "bitnet_rmsnorm_quant_act", "bitnet_bitlinear",
    "bitnet_bitlinear_group", "bitnet_bitlinear_gate_up_act", "bitnet_ffn_workspace_bytes", "bitnet_ffn_workspace_offsets",
    "bitnet_ffn_block", "bitnet_ffn_block_noalloc_max_bytes", "bitnet_ffn_block_noalloc",
    "bitnet_block_workspace_bytes", "bitnet_block_workspace_offsets", "bitnet_decoder_block",
    "bitnet_get_device_status", "bitnet_status_string", "bitnet_last_error",
]


class BitnetError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {_STATUS.get(status, status)}"
        if status == 6:
            msg += f" ({_lib.bitnet_last_error().decode()})"
        super().__init__(msg)
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m ternary_bitlinear_quantized_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    c_p, c_i64, c_i, c_f, c_sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "bitnet_i2s_packed_bytes": (c_sz, [c_i64, c_i64]),
        "bitnet_pack_i2s": (c_i, [c_p, c_i64, c_i64, c_p, c_p]),
        "bitnet_pack_i2s_prescaled": (c_i, [c_p, c_i64, c_i64, c_p, c_p]),
        "bitnet_validate_i2s": (c_i, [c_p, c_i64, c_i64, c_p, c_p]),
        "bitnet_rmsnorm_quant_act": (c_i, [c_p, c_i, c_p, c_f, c_i64, c_i64, c_p, c_p, c_p, c_p]),
        "bitnet_bitlinear": (c_i, [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_i, c_p, c_p]),
        "bitnet_bitlinear_group": (c_i, [c_p, c_p, c_p, c_i, c_p, c_p, c_i64, c_i64, c_p, c_i, c_p]),
        "bitnet_bitlinear_gate_up_act": (c_i, [c_p, c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_i, c_p, c_p]),
        "bitnet_bitlinear_acc": (c_i, [c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_p]),
        "bitnet_dequant_acc": (c_i, [c_p, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_i, c_p]),
        "bitnet_subnorm_shard_amax": (c_i, [c_p, c_i64, c_i64, c_p, c_p]),
        "bitnet_subnorm_shard_sumsq": (c_i, [c_p, c_i64, c_i64, c_p, c_i64, c_p, c_p]),
        "bitnet_subnorm_shard_ymax": (c_i, [c_p, c_p, c_i64, c_i64, c_p, c_p, c_i64, c_f, c_p, c_p, c_p]),
        "bitnet_subnorm_shard_quant": (c_i, [c_p, c_p, c_i64, c_i64, c_p, c_p, c_p, c_p, c_p, c_p]),
        "bitnet_ffn_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64]),
        "bitnet_ffn_workspace_offsets": (c_i, [c_i64, c_i64, c_i64, c_p]),
        "bitnet_ffn_block": (c_i, [c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_i, c_f, c_p, c_i,
                                   c_p, c_sz, c_p]),
        "bitnet_ffn_block_noalloc_max_bytes": (c_sz, []),
        "bitnet_ffn_block_noalloc": (c_i, [c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_i, c_f, c_p, c_i,
                                           c_p]),
        "bitnet_block_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64, c_i64]),
        "bitnet_block_workspace_offsets": (c_i, [c_i64, c_i64, c_i64, c_i64, c_p]),
        "bitnet_decoder_block": (c_i, [c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p,
                                       c_i64, c_i64, c_i64, c_i64, c_i64, c_i, c_f, c_p, c_p, c_p, c_p, c_p, c_i,
                                       c_p, c_sz, c_p]),
        "bitnet_rope_kv_append": (c_i, [c_p, c_p, c_p, c_i, c_i64, c_i64, c_i64, c_i64, c_i64, ctypes.c_double, c_p,
                                        c_p, c_p, c_i64, c_p]),
        "bitnet_attention_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64, c_i64]),
        "bitnet_attention_decode": (c_i, [c_p, c_p, c_p, c_i64, c_i64, c_i64, c_i64, c_i64, c_i64, c_p, c_i, c_p, c_sz,
                                          c_p]),
        "bitnet_get_device_status": (c_i, [c_p]),
        "bitnet_debug_set_wait_limit": (c_i, [ctypes.c_longlong]),
        "bitnet_status_string": (ctypes.c_char_p, [c_i]),
        "bitnet_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != 0:
        raise BitnetError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {dt}")


def _torch_dtype(code: int) -> torch.dtype:
    return torch.bfloat16 if code == BF16 else torch.float32


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


# ----------------------------------------------------------------------------- API

def i2s_packed_bytes(N: int, K: int) -> int:
    return int(lib().bitnet_i2s_packed_bytes(N, K))


def pack_i2s(W: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Latent fp32 weights [N, K] -> I2_S bytes (uint8 [N*K/4 + 32])."""
    _need(W, "W")
    N, K = W.shape
    nbytes = i2s_packed_bytes(N, K)
    if nbytes == 0:
        raise BitnetError(2, "pack_i2s")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _check(lib().bitnet_pack_i2s(_ptr(W), N, K, _ptr(out), _stream(stream)), "pack_i2s")
    return out


def pack_i2s_prescaled(W: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Ternary x scale fp32 weights [N, K] -> I2_S bytes, scale = first non-zero |w|."""
    _need(W, "W")
    N, K = W.shape
    nbytes = i2s_packed_bytes(N, K)
    if nbytes == 0:
        raise BitnetError(2, "pack_i2s_prescaled")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _check(lib().bitnet_pack_i2s_prescaled(_ptr(W), N, K, _ptr(out), _stream(stream)), "pack_i2s_prescaled")
    return out


def validate_i2s(packed: torch.Tensor, N: int, K: int, counts: torch.Tensor | None = None, stream=None):
    """Device-side I2_S checks -> int64 [3] device tensor: (fields holding 3, non-zero
    trailer bytes after the scale, 1 if the scale is not finite and positive)."""
    _need(packed, "packed")
    if counts is None:
        counts = torch.empty(3, dtype=torch.int64, device=packed.device)
    _check(lib().bitnet_validate_i2s(_ptr(packed), N, K, _ptr(counts), _stream(stream)), "validate_i2s")
    return counts


def rmsnorm_quant_act(x: torch.Tensor, gain: torch.Tensor | None, eps: float = 1e-6, out=None, stream=None):
    """x bf16/fp32 [T, K] -> (q int8 [T, K], s_x fp32 [T], sum_q int32 [T])."""
    _need(x, "x")
    T, K = x.shape
    if out is None:
        out = (torch.empty(T, K, dtype=torch.int8, device=x.device),
               torch.empty(T, dtype=torch.float32, device=x.device),
               torch.empty(T, dtype=torch.int32, device=x.device))
    q, s, sq = out
    _check(lib().bitnet_rmsnorm_quant_act(_ptr(x), _dtype_code(x.dtype), _ptr(gain), eps, T, K, _ptr(q), _ptr(s),
                                          _ptr(sq), _stream(stream)), "rmsnorm_quant_act")
    return q, s, sq


def bitlinear(q, s_x, sum_q, packed, N: int, out_dtype=torch.bfloat16, out=None, acc_debug=None, stream=None):
    """acc = sum q*c - sum_q; out = fp32(acc) * (beta / s_x) as out_dtype [T, N]."""
    T, K = q.shape
    if out is None:
        out = torch.empty(T, N, dtype=out_dtype, device=q.device)
    _check(lib().bitnet_bitlinear(_ptr(q), _ptr(s_x), _ptr(sum_q), _ptr(packed), T, N, K, _ptr(out),
                                  _dtype_code(out.dtype), _ptr(acc_debug), _stream(stream)), "bitlinear")
    return out


def bitlinear_acc(q, sum_q, packed, N: int, out=None, stream=None) -> torch.Tensor:
    """int32 accumulators [T, N] = q @ c^T - sum_q (no dequantisation)."""
    T, K = q.shape
    for t, nm in ((q, "q"), (sum_q, "sum_q"), (packed, "packed")):
        _need(t, nm)
    acc = out if out is not None else torch.empty(T, N, dtype=torch.int32, device=q.device)
    _check(lib().bitnet_bitlinear_acc(_ptr(q), _ptr(sum_q), _ptr(packed), T, N, K, _ptr(acc), _stream(stream)),
           "bitlinear_acc")
    return acc


def dequant_acc(acc, s_x, packed, K: int, out_dtype=torch.bfloat16, out=None, stream=None) -> torch.Tensor:
    """out = fp32(acc) * (beta / s_x), beta from the I2_S trailer of `packed` ([N, K])."""
    T, N = acc.shape
    for t, nm in ((acc, "acc"), (s_x, "s_x"), (packed, "packed")):
        _need(t, nm)
    o = out if out is not None else torch.empty(T, N, dtype=out_dtype, device=acc.device)
    _check(lib().bitnet_dequant_acc(_ptr(acc), _ptr(s_x), _ptr(packed), T, N, K, _ptr(o), _dtype_code(o.dtype),
                                    _stream(stream)), "dequant_acc")
    return o


def subnorm_shard_amax(h, out=None, stream=None):
    T, Ks = h.shape
    _need(h, "h")
    a = out if out is not None else torch.empty(T, dtype=torch.float32, device=h.device)
    _check(lib().bitnet_subnorm_shard_amax(_ptr(h), T, Ks, _ptr(a), _stream(stream)), "subnorm_shard_amax")
    return a


def subnorm_shard_sumsq(h, amax, K_total: int, out=None, stream=None):
    T, Ks = h.shape
    _need(h, "h")
    S = out if out is not None else torch.empty(T, dtype=torch.int64, device=h.device)
    _check(lib().bitnet_subnorm_shard_sumsq(_ptr(h), T, Ks, _ptr(amax), K_total, _ptr(S), _stream(stream)),
           "subnorm_shard_sumsq")
    return S


def subnorm_shard_ymax(h, gain, amax, S, K_total: int, eps: float = 1e-6, stream=None):
    T, Ks = h.shape
    _need(h, "h")
    inv = torch.empty(T, dtype=torch.float32, device=h.device)
    ymax = torch.empty(T, dtype=torch.float32, device=h.device)
    _check(lib().bitnet_subnorm_shard_ymax(_ptr(h), _ptr(gain), T, Ks, _ptr(amax), _ptr(S), K_total, eps, _ptr(inv),
                                           _ptr(ymax), _stream(stream)), "subnorm_shard_ymax")
    return inv, ymax


def subnorm_shard_quant(h, gain, inv, ymax, stream=None):
    T, Ks = h.shape
    _need(h, "h")
    q = torch.empty(T, Ks, dtype=torch.int8, device=h.device)
    s = torch.empty(T, dtype=torch.float32, device=h.device)
    sq = torch.empty(T, dtype=torch.int32, device=h.device)
    _check(lib().bitnet_subnorm_shard_quant(_ptr(h), _ptr(gain), T, Ks, _ptr(inv), _ptr(ymax), _ptr(q), _ptr(s),
                                            _ptr(sq), _stream(stream)), "subnorm_shard_quant")
    return q, s, sq


def bitlinear_group(q, s_x, sum_q, packed: list, Ns: list, out_dtype=torch.bfloat16, outs=None, stream=None):
    """Several BitLinears sharing one quantised input, in one launch."""
    T, K = q.shape
    n = len(packed)
    if outs is None:
        outs = [torch.empty(T, N, dtype=out_dtype, device=q.device) for N in Ns]
    P = (ctypes.c_void_p * n)(*[p.data_ptr() for p in packed])
    NN = (ctypes.c_int64 * n)(*Ns)
    O = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    _check(lib().bitnet_bitlinear_group(_ptr(q), _ptr(s_x), _ptr(sum_q), n, ctypes.cast(P, ctypes.c_void_p),
                                        ctypes.cast(NN, ctypes.c_void_p), T, K, ctypes.cast(O, ctypes.c_void_p),
                                        _dtype_code(outs[0].dtype), _stream(stream)), "bitlinear_group")
    return outs


def bitlinear_gate_up_act(q, s_x, sum_q, p_gate, p_up, I: int, act: int = RELU2, out=None, stream=None):
    """h = act(gate) * up, fp32 [T, I], from one quantised input (the FFN's first half)."""
    T, K = q.shape
    if out is None:
        out = torch.empty(T, I, dtype=torch.float32, device=q.device)
    _check(lib().bitnet_bitlinear_gate_up_act(_ptr(q), _ptr(s_x), _ptr(sum_q), _ptr(p_gate), _ptr(p_up), T, I, K,
                                              act, _ptr(out), _stream(stream)), "bitlinear_gate_up_act")
    return out


def ffn_workspace_bytes(T: int, H: int, I: int) -> int:
    return int(lib().bitnet_ffn_workspace_bytes(T, H, I))


def ffn_workspace_offsets(T: int, H: int, I: int) -> list[int]:
    off = (ctypes.c_size_t * 8)()
    _check(lib().bitnet_ffn_workspace_offsets(T, H, I, ctypes.cast(off, ctypes.c_void_p)), "ffn_workspace_offsets")
    return list(off)


def ffn_block(x, g_ffn, p_gate, p_up, g_sub, p_down, I: int, act: int = RELU2, eps: float = 1e-6,
              out_dtype=torch.bfloat16, out=None, ws=None, stream=None):
    """BitNet FFN: down(ffn_sub_norm(act(gate(x)) * up(x))) on x [T, H]."""
    _need(x, "x")
    T, H = x.shape
    if out is None:
        out = torch.empty(T, H, dtype=out_dtype, device=x.device)
    nws = ffn_workspace_bytes(T, H, I)
    if ws is None:
        ws = torch.zeros(max(nws, 16), dtype=torch.uint8, device=x.device)  # barrier counters start at zero
    _check(lib().bitnet_ffn_block(_ptr(x), _dtype_code(x.dtype), _ptr(g_ffn), _ptr(p_gate), _ptr(p_up), _ptr(g_sub),
                                  _ptr(p_down), T, H, I, act, eps, _ptr(out), _dtype_code(out.dtype), _ptr(ws),
                                  ws.numel(), _stream(stream)), "ffn_block")
    return out


def ffn_block_noalloc(x, g_ffn, p_gate, p_up, g_sub, p_down, I: int, act: int = RELU2, eps: float = 1e-6,
                      out_dtype=torch.bfloat16, out=None, stream=None):
    """ffn_block for callers that cannot allocate device memory: the workspace is the
    library's built-in device array (shared by all calls on a device; overlapping calls
    race).  ``out`` must be given by such callers; it is allocated here only for tests."""
    _need(x, "x")
    T, H = x.shape
    if out is None:
        out = torch.empty(T, H, dtype=out_dtype, device=x.device)
    _check(lib().bitnet_ffn_block_noalloc(_ptr(x), _dtype_code(x.dtype), _ptr(g_ffn), _ptr(p_gate), _ptr(p_up),
                                          _ptr(g_sub), _ptr(p_down), T, H, I, act, eps, _ptr(out),
                                          _dtype_code(out.dtype), _stream(stream)), "ffn_block_noalloc")
    return out


def block_workspace_bytes(T: int, H: int, NQ: int, I: int) -> int:
    return int(lib().bitnet_block_workspace_bytes(T, H, NQ, I))


def block_workspace_offsets(T: int, H: int, NQ: int, I: int) -> list[int]:
    off = (ctypes.c_size_t * 7)()
    _check(lib().bitnet_block_workspace_offsets(T, H, NQ, I, ctypes.cast(off, ctypes.c_void_p)),
           "block_workspace_offsets")
    return list(off)


def decoder_block(x, attn_out, gains: dict, packed: dict, NKV: int, I: int, act: int = RELU2, eps: float = 1e-6,
                  out_dtype=torch.bfloat16, outs=None, ws=None, stream=None):
    """The BitLinear projections of a decoder block.  gains: attn_norm, attn_sub_norm,
    ffn_norm, ffn_sub_norm (tensors or None); packed: q, k, v, o, gate, up, down.
    Returns dict q, k, v, o, ffn.  ``ws`` must start zeroed (allocated here if None)."""
    _need(x, "x")
    _need(attn_out, "attn_out")
    T, H = x.shape
    NQ = attn_out.shape[1]
    if outs is None:
        e = lambda n: torch.empty(T, n, dtype=out_dtype, device=x.device)
        outs = {"q": e(NQ), "k": e(NKV), "v": e(NKV), "o": e(H), "ffn": e(H)}
    if ws is None:
        ws = torch.zeros(block_workspace_bytes(T, H, NQ, I), dtype=torch.uint8, device=x.device)
    g = lambda k: _ptr(gains.get(k))
    _check(lib().bitnet_decoder_block(_ptr(x), _ptr(attn_out), _dtype_code(x.dtype), g("attn_norm"),
                                      g("attn_sub_norm"), g("ffn_norm"), g("ffn_sub_norm"), _ptr(packed["q"]),
                                      _ptr(packed["k"]), _ptr(packed["v"]), _ptr(packed["o"]), _ptr(packed["gate"]),
                                      _ptr(packed["up"]), _ptr(packed["down"]), T, H, NQ, NKV, I, act, eps,
                                      _ptr(outs["q"]), _ptr(outs["k"]), _ptr(outs["v"]), _ptr(outs["o"]),
                                      _ptr(outs["ffn"]), _dtype_code(outs["ffn"].dtype), _ptr(ws), ws.numel(),
                                      _stream(stream)), "decoder_block")
    return outs


def rope_kv_append(q, k, v, pos0: int, theta: float, k_cache, v_cache, q_rot=None, stream=None) -> torch.Tensor:
    """Rotate q [T, Hq, 128] and k [T, Hkv, 128] at positions pos0 + t; append k (rotated) and v
    to the bf16 caches [Hkv, L_max, 128].  Returns q_rot (fp32 [T, Hq, 128])."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, nm)
    qr = q_rot if q_rot is not None else torch.empty(T, Hq, d, dtype=torch.float32, device=q.device)
    _check(lib().bitnet_rope_kv_append(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), T, Hq, Hkv, d, pos0,
                                       float(theta), _ptr(qr), _ptr(k_cache), _ptr(v_cache), k_cache.shape[1],
                                       _stream(stream)), "rope_kv_append")
    return qr


def attention_workspace_bytes(T: int, Hq: int, Hkv: int, L: int) -> int:
    return int(lib().bitnet_attention_workspace_bytes(T, Hq, Hkv, L))


def attention_decode(q_rot, k_cache, v_cache, pos0: int, out_dtype=torch.bfloat16, out=None, ws=None,
                     stream=None) -> torch.Tensor:
    """Causal GQA attention of q_rot [T, Hq, 128] (positions pos0 + t) over cache rows 0..pos0 + t."""
    T, Hq, d = q_rot.shape
    Hkv, L_max = k_cache.shape[0], k_cache.shape[1]
    for t, nm in ((q_rot, "q_rot"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, nm)
    o = out if out is not None else torch.empty(T, Hq, d, dtype=out_dtype, device=q_rot.device)
    nws = attention_workspace_bytes(T, Hq, Hkv, pos0 + T)
    w = ws if ws is not None else torch.empty(max(nws, 16), dtype=torch.uint8, device=q_rot.device)
    _check(lib().bitnet_attention_decode(_ptr(q_rot), _ptr(k_cache), _ptr(v_cache), T, Hq, Hkv, d, pos0, L_max,
                                         _ptr(o), _dtype_code(o.dtype), _ptr(w), w.numel(), _stream(stream)),
           "attention_decode")
    return o


def debug_set_wait_limit(cycles: int) -> None:
    """Set the kernels' bounded-wait limit on the current device (cycles; <= 0 restores the
    default).  A testing aid: synchronises the device."""
    _check(lib().bitnet_debug_set_wait_limit(int(cycles)), "debug_set_wait_limit")


def device_status(stream=None) -> int:
    """Synchronise and read/clear the device status word (0 = ok, 7 = a wait timed out)."""
    return int(lib().bitnet_get_device_status(_stream(stream)))

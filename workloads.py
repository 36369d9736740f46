"""Seeded synthetic inputs for the BitNet b1.58 BitLinear forward.

This module only draws random numbers and names shapes. It holds none of the
method's arithmetic (no norm, no quantisation, no packing), so that the CPU
oracle (``oracle/``) and the CUDA path (``ternary_bitlinear_quantized_b200``)
can both be fed from it without sharing any code of the method.

Distributions (the workloads of the BitNet pages: the 2B4T model of the cpp-bitnet
pull request "fix: I2_S ARM kernel layout + squared-ReLU FFN", the Llama-2 70B
figure of the llama.cpp discussion "More BitNet-like IQ1_S quantizations", the
bitnet-r1-32b model named in the transformers pull request "Add optional RMSNorm
support to BitNet quantization"):

* latent weights  W ~ N(0, 0.02) in fp32, shape [N, K] (nn.Linear convention);
* activations     x ~ N(0, 1) in fp32, rounded to bf16 by torch (round to nearest even);
  optionally 1 % of the channels (round(0.01 K), a seeded permutation) scaled x20
  before the rounding, as outliers;
* RMSNorm gains   g ~ N(1, 0.1) in fp32;
* eps = 1e-6.

Every tensor is drawn from its own ``torch.Generator`` seeded from (seed, name), so
adding a tensor never shifts the stream of another.
"""
from __future__ import annotations

import dataclasses
import hashlib

import torch

EPS = 1e-6


def _gen(seed: int, name: str, device: str = "cpu") -> torch.Generator:
    h = hashlib.sha256(f"{seed}/{name}".encode()).digest()
    g = torch.Generator(device=device)
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def latent_weight(N: int, K: int, seed: int, name: str, device: str = "cpu") -> torch.Tensor:
    """fp32 [N, K] ~ N(0, 0.02)."""
    g = _gen(seed, "W/" + name, device)
    return torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * 0.02


def activations(T: int, K: int, seed: int, name: str, outliers: bool = False,
                device: str = "cpu") -> torch.Tensor:
    """bf16 [T, K] ~ N(0, 1); with ``outliers``, round(0.01 K) seeded channels are scaled x20."""
    g = _gen(seed, "x/" + name, device)
    x = torch.randn(T, K, generator=g, device=device, dtype=torch.float32)
    if outliers:
        n_out = int(round(0.01 * K))
        pg = _gen(seed, "outlier-channels/" + name, "cpu")
        idx = torch.randperm(K, generator=pg)[:n_out].to(device)
        x[:, idx] *= 20.0
    return x.to(torch.bfloat16)


def gain(K: int, seed: int, name: str, device: str = "cpu") -> torch.Tensor:
    """fp32 [K] ~ N(1, 0.1)."""
    g = _gen(seed, "g/" + name, device)
    return 1.0 + 0.1 * torch.randn(K, generator=g, device=device, dtype=torch.float32)


@dataclasses.dataclass(frozen=True)
class BlockShape:
    """A decoder block's BitLinear projections: q,k,v share ``attn_norm``; o takes a
    synthetic attention output through ``attn_sub_norm``; gate/up share ``ffn_norm``;
    down takes h through ``ffn_sub_norm``."""
    name: str
    hidden: int
    n_q: int
    n_kv: int
    inter: int
    act: str  # "relu2" | "silu"

    def tensors(self):
        H, I = self.hidden, self.inter
        return {
            "q": (self.n_q, H), "k": (self.n_kv, H), "v": (self.n_kv, H), "o": (H, self.n_q),
            "gate": (I, H), "up": (I, H), "down": (H, I),
        }

    def packed_bytes(self) -> int:
        return sum(n * k // 4 + 32 for (n, k) in self.tensors().values())


# bitnet-b1.58-2B-4T: hidden 2560, 20 query heads / 5 KV heads of 128, FFN 6912, relu2.
B2B4T = BlockShape("2b4t", hidden=2560, n_q=2560, n_kv=640, inter=6912, act="relu2")
# Llama-2-70B shapes: hidden 8192, GQA k/v 1024, FFN 28672, SiLU.
L70B = BlockShape("70b", hidden=8192, n_q=8192, n_kv=1024, inter=28672, act="silu")
# bitnet-r1-32b FFN: hidden 5120, intermediate 27648, relu2.
R1_32B = BlockShape("32b", hidden=5120, n_q=5120, n_kv=1024, inter=27648, act="relu2")

# The five workloads (name, shape, tokens, outliers, what runs).
WORKLOADS = {
    "bitlinear_2560_t8": dict(kind="bitlinear", N=2560, K=2560, T=8),
    "block_2b4t_decode_t1": dict(kind="block", shape=B2B4T, T=1),
    "block_2b4t_prefill_t2048": dict(kind="block", shape=B2B4T, T=2048, outliers=True),
    "proj_70b_decode_t1": dict(kind="block", shape=L70B, T=1),
    "proj_70b_decode_t16": dict(kind="block", shape=L70B, T=16),
    "ffn_32b_t1": dict(kind="ffn", shape=R1_32B, T=1),
    "ffn_32b_t64": dict(kind="ffn", shape=R1_32B, T=64),
    "ffn_32b_t512": dict(kind="ffn", shape=R1_32B, T=512),
    "ffn_32b_t4096": dict(kind="ffn", shape=R1_32B, T=4096),
}


def block_inputs(shape: BlockShape, T: int, seed: int = 0, outliers: bool = False,
                 device: str = "cpu", ffn_only: bool = False) -> dict:
    """Latent weights, gains and activations of one block (or of its FFN only)."""
    d = {}
    names = ["gate", "up", "down"] if ffn_only else list(shape.tensors())
    for nm in names:
        n, k = shape.tensors()[nm]
        d["W_" + nm] = latent_weight(n, k, seed, f"{shape.name}/{nm}", device)
    H, I = shape.hidden, shape.inter
    d["g_ffn_norm"] = gain(H, seed, f"{shape.name}/ffn_norm", device)
    d["g_ffn_sub_norm"] = gain(I, seed, f"{shape.name}/ffn_sub_norm", device)
    d["x"] = activations(T, H, seed, f"{shape.name}/x", outliers, device)
    if not ffn_only:
        d["g_attn_norm"] = gain(H, seed, f"{shape.name}/attn_norm", device)
        d["g_attn_sub_norm"] = gain(shape.n_q, seed, f"{shape.name}/attn_sub_norm", device)
        d["attn_out"] = activations(T, shape.n_q, seed, f"{shape.name}/attn_out", outliers, device)
    return d


# Attention at decode: the heads of the block shapes (2B4T: 20 query / 5 key-value heads,
# 70B: 64 / 8, head size 128) over a KV cache of synthetic earlier tokens.  The pages give no
# context length; 4096 cached positions stand in for a long prompt.
ATTN_SHAPES = {"2b4t": (20, 5), "70b": (64, 8)}
ATTN_CONTEXT = 4096


def attention_inputs(T: int, Hq: int, Hkv: int, L_max: int, pos0: int, seed: int = 0, device: str = "cpu") -> dict:
    """New tokens' q [T, Hq, 128], k and v [T, Hkv, 128] (bf16 ~ N(0, 1), the projections'
    outputs) and bf16 caches [Hkv, L_max, 128] whose first pos0 rows hold earlier tokens'
    (already rotated) keys and values ~ N(0, 1); the other rows are zero."""
    d = {}
    for nm, h in (("q", Hq), ("k", Hkv), ("v", Hkv)):
        g = _gen(seed, f"attn/{nm}", device)
        d[nm] = torch.randn(T, h, 128, generator=g, device=device).to(torch.bfloat16)
    for nm in ("k_cache", "v_cache"):
        g = _gen(seed, f"attn/{nm}", device)
        c = torch.zeros(Hkv, L_max, 128, dtype=torch.bfloat16, device=device)
        c[:, :pos0] = torch.randn(Hkv, pos0, 128, generator=g, device=device).to(torch.bfloat16)
        d[nm] = c
    return d

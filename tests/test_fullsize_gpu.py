"""Parity at the full sizes of the five workloads, in the launch configuration bench.py
times (the decode engine for T <= 16, the tensor-core path above), against the CPU oracle.

The oracle packs every tensor in full (the per-tensor scale depends on all of it) and the
GPU-packed bytes must equal it.  Outputs are compared on all tokens where the oracle is
fast enough, otherwise on sampled tokens: every step of the path is per token (the
norm, the int8 quantisation, the products and the FFN), so the oracle run on the sampled
rows of x alone gives exactly those rows of the full batch.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import ternary_bitlinear_quantized_b200 as tb
import workloads
from oracle import bitnet_oracle as O
from tests.parity_util import assert_close, bf16_to_np, out_to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"
_cache: dict = {}


def packed_pair(shape: workloads.BlockShape, names, seed=0):
    """(oracle bytes, GPU bytes) per tensor, both from the same latent weights."""
    out = {}
    for nm in names:
        key = (shape.name, nm, seed)
        if key not in _cache:
            n, k = shape.tensors()[nm]
            W = workloads.latent_weight(n, k, seed, f"{shape.name}/{nm}")
            ref = O.pack_i2s(W.numpy())
            gpu = tb.pack_i2s(W.to(DEV))
            del W
            assert np.array_equal(gpu.cpu().numpy(), ref), f"packed bytes of {nm} differ"
            _cache[key] = (ref, gpu)
        out[nm] = _cache[key]
    return out


def oracle_ffn_rows(shape, x_rows, gains, pk, act, dt):
    H, I = shape.hidden, shape.inter
    return O.ffn_block(x_rows, gains["ffn_norm"], pk["gate"][0], pk["up"][0], gains["ffn_sub_norm"], pk["down"][0],
                       H, I, act, 1e-6, dt)


def test_fullsize_bitlinear_2560_t8():
    spec = workloads.WORKLOADS["bitlinear_2560_t8"]
    N, K, T = spec["N"], spec["K"], spec["T"]
    W = workloads.latent_weight(N, K, 0, "bitlinear_2560_t8")
    x = workloads.activations(T, K, 0, "bitlinear_2560_t8/x")
    g = workloads.gain(K, 0, "bitlinear_2560_t8/g")
    ref_p = O.pack_i2s(W.numpy())
    p = tb.pack_i2s(W.to(DEV))
    assert np.array_equal(p.cpu().numpy(), ref_p)
    q, s, sq = tb.rmsnorm_quant_act(x.to(DEV), g.to(DEV))
    acc = torch.empty(T, N, dtype=torch.int32, device=DEV)
    out = tb.bitlinear(q, s, sq, p, N, torch.bfloat16, acc_debug=acc)
    rq, rs, rsq = O.rmsnorm_quant_act(bf16_to_np(x), g.numpy(), 1e-6)
    ref, racc = O.bitlinear(rq, rs, rsq, ref_p, N, K, "bf16", return_acc=True)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert_close(out_to_np(out), ref, "bf16")


def _run_block(wname, sample_tokens=None):
    spec = workloads.WORKLOADS[wname]
    sh, T = spec["shape"], spec["T"]
    d = workloads.block_inputs(sh, T, 0, spec.get("outliers", False))
    pk = packed_pair(sh, list(sh.tensors()))
    gains = {k[2:]: v for k, v in d.items() if k.startswith("g_")}
    act = tb.RELU2 if sh.act == "relu2" else tb.SILU
    outs = tb.decoder_block(d["x"].to(DEV), d["attn_out"].to(DEV), {k: v.to(DEV) for k, v in gains.items()},
                            {k: v[1] for k, v in pk.items()}, sh.n_kv, sh.inter, act, 1e-6, torch.bfloat16)
    torch.cuda.synchronize()
    assert tb.device_status() == 0
    rows = np.arange(T) if sample_tokens is None else np.asarray(sample_tokens)
    ref = O.decoder_block(bf16_to_np(d["x"])[rows], bf16_to_np(d["attn_out"])[rows],
                          {k: v.numpy() for k, v in gains.items()}, {k: v[0] for k, v in pk.items()},
                          sh.tensors(), sh.act, 1e-6, "bf16")
    for name in ("q", "k", "v", "o", "ffn"):
        got = out_to_np(outs[name])[rows]
        assert_close(got, ref[name], "bf16")
        assert np.array_equal(got.view(np.uint32), ref[name].view(np.uint32)), name


def test_fullsize_block_2b4t_decode_t1():
    _run_block("block_2b4t_decode_t1")


def test_fullsize_block_2b4t_prefill_t2048_sampled():
    _run_block("block_2b4t_prefill_t2048", sample_tokens=[0, 1, 511, 1024, 1500, 2047])


def test_fullsize_70b_decode_t1():
    _run_block("proj_70b_decode_t1")


def test_fullsize_70b_decode_t16_sampled():
    _run_block("proj_70b_decode_t16", sample_tokens=[0, 7, 8, 15])


@pytest.mark.parametrize("wname,sample", [("ffn_32b_t1", None), ("ffn_32b_t64", [0, 31, 63]),
                                          ("ffn_32b_t512", [0, 255, 511]), ("ffn_32b_t4096", [0, 2048, 4095])])
def test_fullsize_ffn_32b(wname, sample):
    spec = workloads.WORKLOADS[wname]
    sh, T = spec["shape"], spec["T"]
    d = workloads.block_inputs(sh, T, 0, ffn_only=True)
    pk = packed_pair(sh, ["gate", "up", "down"])
    out = tb.ffn_block(d["x"].to(DEV), d["g_ffn_norm"].to(DEV), pk["gate"][1], pk["up"][1],
                       d["g_ffn_sub_norm"].to(DEV), pk["down"][1], sh.inter, tb.RELU2, 1e-6, torch.bfloat16)
    torch.cuda.synchronize()
    rows = np.arange(T) if sample is None else np.asarray(sample)
    gains = {"ffn_norm": d["g_ffn_norm"].numpy(), "ffn_sub_norm": d["g_ffn_sub_norm"].numpy()}
    ref = oracle_ffn_rows(sh, bf16_to_np(d["x"])[rows], gains, pk, "relu2", "bf16")
    got = out_to_np(out)[rows]
    assert_close(got, ref, "bf16")
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))

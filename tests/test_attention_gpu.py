"""The block's attention at decode on the GPU against the fp64 oracle: the rotary embedding
and the cache append, and causal grouped-query attention over the cache.  Float results
within a stated tolerance (the GPU computes in fp32, the oracle in fp64); the appended
values (a copy) bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import ternary_bitlinear_quantized_b200 as tb
import workloads
from oracle import bitnet_oracle as O
from tests.parity_util import bf16_to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(x: torch.Tensor) -> np.ndarray:
    return bf16_to_np(x) if x.dtype == torch.bfloat16 else x.detach().cpu().numpy()


@pytest.mark.parametrize("T,Hq,Hkv,pos0,theta", [(1, 20, 5, 0, 10000.0), (3, 20, 5, 100, 10000.0),
                                                 (16, 64, 8, 4000, 500000.0), (2, 8, 8, 65000, 10000.0)])
def test_rope_kv_append(T, Hq, Hkv, pos0, theta):
    L_max = pos0 + T + 5
    d = workloads.attention_inputs(T, Hq, Hkv, L_max, 0, seed=T)
    kc = torch.zeros(Hkv, L_max, 128, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    q_rot = tb.rope_kv_append(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), pos0, theta, kc, vc)
    torch.cuda.synchronize()
    pos = np.arange(pos0, pos0 + T)
    rq = O.apply_rope(_np(d["q"]), pos, theta)
    rk = O.apply_rope(_np(d["k"]), pos, theta)
    got = q_rot.cpu().numpy().astype(np.float64)
    pair = np.sqrt(rq[..., :64] ** 2 + rq[..., 64:] ** 2)
    bound = 1e-6 * np.concatenate([pair, pair], axis=-1) + 1e-30
    assert np.all(np.abs(got - rq) <= bound)
    gk = _np(kc[:, pos0:pos0 + T]).transpose(1, 0, 2).astype(np.float64)
    # the cache holds bf16: within one bf16 rounding of the exact rotation
    pk = np.sqrt(rk[..., :64] ** 2 + rk[..., 64:] ** 2)
    assert np.all(np.abs(gk - rk) <= 2.0 ** -8 * np.abs(rk) + 1e-6 * np.concatenate([pk, pk], axis=-1))
    assert torch.equal(vc[:, pos0:pos0 + T].cpu(), d["v"].transpose(0, 1))
    assert not kc[:, :pos0].any() and not kc[:, pos0 + T:].any()


def _check_attention(got: np.ndarray, ref: np.ndarray, tol: float):
    scale = np.maximum(np.abs(ref), 1e-2 * np.max(np.abs(ref)))
    err = float(np.max(np.abs(got - ref) / scale))
    assert err <= tol, f"attention rel err {err} > {tol}"


@pytest.mark.parametrize("T,shape,pos0", [(1, "2b4t", 0), (1, "2b4t", 4095), (3, "2b4t", 1000), (1, "70b", 4095),
                                          (16, "70b", 4080), (5, "70b", 63), (8, "2b4t", 130)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_attention_decode(T, shape, pos0, out_dtype):
    Hq, Hkv = workloads.ATTN_SHAPES[shape]
    L_max = workloads.ATTN_CONTEXT + 16
    d = workloads.attention_inputs(T, Hq, Hkv, L_max, pos0 + T, seed=T + pos0)
    q = d["q"].float() * 0.3  # scores of a few units, as after a norm
    out = tb.attention_decode(q.to(DEV), d["k_cache"].to(DEV), d["v_cache"].to(DEV), pos0, out_dtype)
    torch.cuda.synchronize()
    L = pos0 + T
    ref = O.attention(q.numpy(), _np(d["k_cache"][:, :L]).transpose(1, 0, 2), _np(d["v_cache"][:, :L]).transpose(1, 0, 2),
                      np.arange(pos0, L))
    _check_attention(_np(out).astype(np.float64), ref, 1e-3 if out_dtype == torch.float32 else 1e-2)
    assert tb.device_status() == 0


def test_rope_append_then_attention_chain():
    """A decode step: rotate and append the new tokens, then attend over the cache."""
    T, (Hq, Hkv), pos0, theta = 2, workloads.ATTN_SHAPES["2b4t"], 777, 10000.0
    L_max = 1024
    d = workloads.attention_inputs(T, Hq, Hkv, L_max, pos0, seed=5)
    kc, vc = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    q_rot = tb.rope_kv_append(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), pos0, theta, kc, vc)
    out = tb.attention_decode(q_rot, kc, vc, pos0, torch.float32)
    torch.cuda.synchronize()
    pos = np.arange(pos0, pos0 + T)
    rq = O.apply_rope(_np(d["q"]), pos, theta)
    rk = O.round_to_bf16(O.apply_rope(_np(d["k"]), pos, theta).astype(np.float32))  # the cache holds bf16
    k_all = np.concatenate([_np(d["k_cache"][:, :pos0]).transpose(1, 0, 2), rk], axis=0)
    v_all = np.concatenate([_np(d["v_cache"][:, :pos0]).transpose(1, 0, 2), _np(d["v"])], axis=0)
    ref = O.attention(rq, k_all, v_all, pos)
    _check_attention(out.cpu().numpy().astype(np.float64), ref, 1e-3)

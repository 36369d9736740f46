"""Tensor parallelism of the FFN block on the GPU.  Several shards run in one process on one
GPU, their partial results are combined the way the all-reduces would combine them
(maximum, integer sum), and the output must equal the single-device oracle bit for bit;
then the real collective path with a one-rank NCCL process group."""
from __future__ import annotations

import socket

import numpy as np
import pytest
import torch

import ternary_bitlinear_quantized_b200 as tb
from ternary_bitlinear_quantized_b200 import tp
import workloads
from oracle import bitnet_oracle as O
from tests.parity_util import bf16_to_np, out_to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(T, H, I, act, seed, use_sub=True):
    sh = workloads.BlockShape("tp-gpu", hidden=H, n_q=H, n_kv=H, inter=I, act=act)
    d = workloads.block_inputs(sh, T, seed, ffn_only=True)
    pr = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in ("gate", "up", "down")}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    g_sub = d["g_ffn_sub_norm"] if use_sub else None
    ref, mid = O.ffn_block(bf16_to_np(d["x"]), d["g_ffn_norm"].numpy(), pr["gate"], pr["up"],
                           None if g_sub is None else g_sub.numpy(), pr["down"], H, I, act, 1e-6, "f32",
                           return_intermediates=True)
    return d, pg, g_sub, ref, mid


@pytest.mark.parametrize("T,H,I,act,world,use_sub", [
    (1, 256, 1024, "relu2", 2, True),
    (3, 512, 2048, "silu", 4, True),
    (16, 256, 1024, "relu2", 2, False),
    (40, 384, 1536, "silu", 2, True),      # tensor-core path for the products
    (1, 2560, 6912, "relu2", 2, True),     # 2B4T FFN shapes, two ranks (3456 = 27 blocks each)
])
def test_shards_combine_to_the_oracle(T, H, I, act, world, use_sub):
    d, pg, g_sub, ref, mid = _setup(T, H, I, act, seed=T + I, use_sub=use_sub)
    code = tb.RELU2 if act == "relu2" else tb.SILU
    x, g1 = d["x"].to(DEV), d["g_ffn_norm"].to(DEV)
    shards = [tp.make_shard(pg["gate"], pg["up"], pg["down"], None if g_sub is None else g_sub.to(DEV), H, I, r, world)
              for r in range(world)]
    runs = [tp.ShardRun(s, x, g1, code, 1e-6) for s in shards]
    amax = torch.stack([r.amax() for r in runs]).amax(0)
    S = [r.sumsq(amax) for r in runs]
    S = None if S[0] is None else torch.stack(S).sum(0)
    ymax = torch.stack([r.ymax(amax, S) for r in runs]).amax(0)
    accs = [r.down_acc(ymax) for r in runs]
    acc = torch.stack(accs).sum(0, dtype=torch.int32)
    outs = [r.finish(acc, torch.float32) for r in runs]
    # each shard's intermediates against the oracle's whole-row result
    h = torch.cat([r.h for r in runs], dim=1).cpu().numpy()
    assert np.array_equal(h.view(np.uint32), mid["h"].view(np.uint32))
    assert np.array_equal(torch.cat([r.q_h for r in runs], dim=1).cpu().numpy(), mid["q_h"])
    assert np.array_equal(sum(r.sum_h.cpu().numpy().astype(np.int64) for r in runs), mid["sum_h"].astype(np.int64))
    for r in runs:
        assert np.array_equal(r.s_h.cpu().numpy().view(np.uint32), mid["s_h"].view(np.uint32))
    for o in outs:
        assert np.array_equal(out_to_np(o).view(np.uint32), ref.view(np.uint32))
    assert tb.device_status() == 0


def test_bitlinear_acc_and_dequant_match_bitlinear():
    T, N, K = 5, 300, 1024
    W = workloads.latent_weight(N, K, 2, "acc")
    x = workloads.activations(T, K, 2, "acc")
    packed = tb.pack_i2s(W.to(DEV))
    q, s, sq = tb.rmsnorm_quant_act(x.to(DEV), None)
    acc_ref = torch.empty(T, N, dtype=torch.int32, device=DEV)
    out_ref = tb.bitlinear(q, s, sq, packed, N, torch.bfloat16, acc_debug=acc_ref)
    acc = tb.bitlinear_acc(q, sq, packed, N)
    assert torch.equal(acc, acc_ref)
    out = tb.dequant_acc(acc, s, packed, K, torch.bfloat16)
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_nccl_one_rank_equals_single_gpu_ffn_block():
    """The collective path itself (NCCL all-reduces) with one rank: the same bits as
    bitnet_ffn_block."""
    T, H, I = 2, 512, 1024
    d, pg, g_sub, ref, _ = _setup(T, H, I, "silu", seed=9)
    x, g1, g2 = d["x"].to(DEV), d["g_ffn_norm"].to(DEV), g_sub.to(DEV)
    torch.distributed.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                                         device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        shard = tp.make_shard(pg["gate"], pg["up"], pg["down"], g2, H, I, 0, 1)
        out = tp.ffn_block_tp(shard, x, g1, tb.SILU, 1e-6, torch.bfloat16)
        torch.cuda.synchronize()
    finally:
        torch.distributed.destroy_process_group()
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    single = tb.ffn_block(x, g1, pg["gate"], pg["up"], g2, pg["down"], I, tb.SILU, 1e-6, torch.bfloat16, ws=ws)
    assert torch.equal(out.view(torch.int16), single.view(torch.int16))
    assert np.array_equal(out_to_np(out).view(np.uint32), O.round_to_bf16(ref).view(np.uint32))

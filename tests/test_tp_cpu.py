"""Tensor parallelism of the FFN block on CPU: the shard cutting of the product module, and
two gloo ranks that run the oracle's staged sub-norm on their shards, combine the partial
results with all-reduces and must reproduce the single-device oracle bit for bit."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads
from oracle import bitnet_oracle as O
from ternary_bitlinear_quantized_b200 import tp


def _packed(N, K, seed, name):
    return O.pack_i2s(workloads.latent_weight(N, K, seed, name).numpy())


def test_shard_rows_and_cols_keep_codes_and_the_global_scale():
    N, K = 384, 512
    p = _packed(N, K, 1, "shard")
    codes, beta = O.unpack_i2s(p, N, K)
    pt = torch.from_numpy(p)
    r = tp.shard_rows(pt, N, K, 128, 256).numpy()
    rc, rb = O.unpack_i2s(r, 128, K)
    assert rb == beta and np.array_equal(rc, codes[128:256])
    c = tp.shard_cols(pt, N, K, 256, 512).numpy()
    cc, cb = O.unpack_i2s(c, N, 256)
    assert cb == beta and np.array_equal(cc, codes[:, 256:512])
    with pytest.raises(ValueError):
        tp.shard_cols(pt, N, K, 64, 256)  # not whole 128-weight blocks
    assert tp.shard_range(1024, 1, 4) == (256, 512)
    with pytest.raises(ValueError):
        tp.shard_range(640, 0, 4)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.numpy()


def _sum(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.numpy()


def _rank_ffn(rank, world, port, q, T, H, I, act, use_sub):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sh = workloads.BlockShape("tp", hidden=H, n_q=H, n_kv=H, inter=I, act=act)
        d = workloads.block_inputs(sh, T, seed=5, ffn_only=True)
        p = {nm: _packed(*sh.tensors()[nm], 5, nm) for nm in ("gate", "up", "down")}
        x = O.bf16_bits_to_f32(d["x"].view(torch.int16).numpy().view(np.uint16))
        g1 = d["g_ffn_norm"].numpy()
        g2 = d["g_ffn_sub_norm"].numpy() if use_sub else None
        shard = tp.make_shard(*(torch.from_numpy(p[nm]) for nm in ("gate", "up", "down")),
                              None if g2 is None else torch.from_numpy(g2), H, I, rank, world)
        Is = shard.Is
        # gate/up on this rank's rows (the oracle, on the product's shard bytes)
        qx, sx, sqx = O.rmsnorm_quant_act(x, g1, 1e-6)
        g = O.bitlinear(qx, sx, sqx, shard.p_gate.numpy(), Is, H, "f32")
        u = O.bitlinear(qx, sx, sqx, shard.p_up.numpy(), Is, H, "f32")
        h = O.ffn_act(g, u, act)
        gs = None if shard.g_sub is None else shard.g_sub.numpy()
        amax = _max(O.shard_amax(h))
        S = _sum(O.shard_sumsq(h, amax, I)) if gs is not None else None
        inv, ym = O.shard_ymax(h, gs, amax, S, I, 1e-6)
        ym = _max(ym)
        qh, sh_, sumh = O.shard_quant(h, gs, inv, ym)
        acc = O.bitlinear_acc(qh, sumh, shard.p_down.numpy(), H, Is)
        acc = _sum(acc.astype(np.int32))
        _, beta = O.unpack_i2s(shard.p_down.numpy(), H, Is)
        out = O.dequant(acc, sh_, beta)
        q.put((rank, out, qh, sh_))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("act,use_sub,world", [("relu2", True, 2), ("silu", True, 2), ("relu2", False, 2),
                                               ("silu", True, 4)])
def test_sharded_ffn_equals_single_device_oracle(act, use_sub, world):
    T, H, I = 3, 256, 128 * world * 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_ffn, args=(r, world, port, q, T, H, I, act, use_sub)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for pr in procs:
        pr.join(120)
        assert pr.exitcode == 0
    sh = workloads.BlockShape("tp", hidden=H, n_q=H, n_kv=H, inter=I, act=act)
    d = workloads.block_inputs(sh, T, seed=5, ffn_only=True)
    p = {nm: _packed(*sh.tensors()[nm], 5, nm) for nm in ("gate", "up", "down")}
    x = O.bf16_bits_to_f32(d["x"].view(torch.int16).numpy().view(np.uint16))
    ref, mid = O.ffn_block(x, d["g_ffn_norm"].numpy(), p["gate"], p["up"],
                           d["g_ffn_sub_norm"].numpy() if use_sub else None, p["down"], H, I, act, 1e-6, "f32",
                           return_intermediates=True)
    for rank, out, qh, s in res:
        assert np.array_equal(out.view(np.uint32), ref.view(np.uint32)), rank  # every rank: the same bits
        assert np.array_equal(s.view(np.uint32), mid["s_h"].view(np.uint32))
    assert np.array_equal(np.concatenate([r[2] for r in res], axis=1), mid["q_h"])

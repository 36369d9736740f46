"""The FFN block for callers that cannot allocate device memory (bitnet_ffn_block_noalloc).

Such callers -- a plugin inside a host framework that owns all device memory and forbids
allocation while serving, or a process under a hard memory cap -- get the FFN block with
its workspace in a device array built into the library.  This file checks, through the C
ABI, that two calls in a row give the same outputs as bitnet_ffn_block with a caller
workspace (bit-identical, so well within the 1e-2 / 1e-3 float tolerances of the other
tests), and that sizes beyond the built-in array are refused.  It is named so that pytest
collects it last; it also passes when run alone in a fresh process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import ternary_bitlinear_quantized_b200 as tb
import workloads
from tests.parity_util import assert_close, out_to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(T, H, I, act, seed):
    sh = workloads.BlockShape("noalloc", hidden=H, n_q=H, n_kv=H, inter=I, act=act)
    d = workloads.block_inputs(sh, T, seed, ffn_only=True)
    packs = {nm: tb.pack_i2s(d["W_" + nm].to(DEV)) for nm in ("gate", "up", "down")}
    return d["x"].to(DEV), d["g_ffn_norm"].to(DEV), d["g_ffn_sub_norm"].to(DEV), packs


@pytest.mark.parametrize("T,H,I,act", [(1, 2560, 6912, "relu2"), (3, 1024, 2048, "silu"), (40, 512, 768, "relu2")])
def test_noalloc_matches_workspace_call_twice(T, H, I, act):
    x, g1, g2, p = _inputs(T, H, I, act, seed=T + I)
    code = tb.RELU2 if act == "relu2" else tb.SILU
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    ref = tb.ffn_block(x, g1, p["gate"], p["up"], g2, p["down"], I, code, 1e-6, torch.bfloat16, ws=ws)
    for _ in range(2):
        got = tb.ffn_block_noalloc(x, g1, p["gate"], p["up"], g2, p["down"], I, code, 1e-6, torch.bfloat16)
        torch.cuda.synchronize()
        r, g = out_to_np(ref), out_to_np(got)
        assert_close(g, r, "bf16")
        assert np.array_equal(g.view(np.uint32), r.view(np.uint32))
    assert tb.device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, H, I = 256, 1024, 4096
    assert tb.ffn_workspace_bytes(T, H, I) > tb.lib().bitnet_ffn_block_noalloc_max_bytes()
    x = torch.zeros(T, H, dtype=torch.bfloat16, device=DEV)
    dummy = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(tb.BitnetError) as e:
        tb.ffn_block_noalloc(x, None, dummy, dummy, None, dummy, I)
    assert e.value.status == 5

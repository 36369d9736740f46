"""Bounded waits on the GPU: with the wait limit cut to one clock cycle, the decode engine's
grid barriers (and ring waits) give up instead of waiting; the kernel returns early, the
device status word reads BITNET_ERR_TIMEOUT, the context stays usable, and with the limit
restored the next call is correct again.  No wait is made endless: every wait in the
kernel is bounded, and after giving up a CTA still lets its own in-flight copies land."""
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
TIMEOUT = 7  # BITNET_ERR_TIMEOUT


def test_short_wait_limit_times_out_then_recovers():
    T, H, I = 1, 512, 1024
    sh = workloads.BlockShape("timeout", hidden=H, n_q=H, n_kv=H, inter=I, act="relu2")
    d = workloads.block_inputs(sh, T, 3, ffn_only=True)
    pr = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in ("gate", "up", "down")}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    args = (d["x"].to(DEV), d["g_ffn_norm"].to(DEV), pg["gate"], pg["up"], d["g_ffn_sub_norm"].to(DEV), pg["down"], I,
            tb.RELU2, 1e-6, torch.bfloat16)
    assert tb.device_status() == 0
    try:
        tb.debug_set_wait_limit(1)
        tb.ffn_block(*args, ws=ws)  # the gate/up -> down grid barrier cannot complete in one cycle
        torch.cuda.synchronize()
        assert tb.device_status() == TIMEOUT
    finally:
        tb.debug_set_wait_limit(0)  # back to the default (about a second)
    ws.zero_()  # the barrier counters must be zero again before the next call
    ref = O.ffn_block(bf16_to_np(d["x"]), d["g_ffn_norm"].numpy(), pr["gate"], pr["up"], d["g_ffn_sub_norm"].numpy(),
                      pr["down"], H, I, "relu2", 1e-6, "bf16")
    for _ in range(2):
        out = tb.ffn_block(*args, ws=ws)
        torch.cuda.synchronize()
        assert tb.device_status() == 0
        assert np.array_equal(bf16_to_np(out).view(np.uint32), ref.view(np.uint32))

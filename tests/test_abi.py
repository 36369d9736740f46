"""The C-ABI library without a GPU: it loads, exports every symbol include/bitnet_b200.h
declares, and its host-side argument checks answer before any CUDA call."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import ternary_bitlinear_quantized_b200 as tb
from ternary_bitlinear_quantized_b200 import build as tbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet_b200.h")


@pytest.fixture(scope="module")
def L():
    tbuild.build()
    return tb.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = declared_functions()
    for must in ("bitnet_pack_i2s", "bitnet_rmsnorm_quant_act", "bitnet_bitlinear", "bitnet_ffn_block"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) <= set(tb.EXPORTS) | set(declared_functions())


def test_packed_bytes(L):
    assert L.bitnet_i2s_packed_bytes(2560, 2560) == 2560 * 2560 // 4 + 32
    assert L.bitnet_i2s_packed_bytes(28672, 8192) == 28672 * 8192 // 4 + 32
    assert L.bitnet_i2s_packed_bytes(3, 200) == 0
    assert L.bitnet_i2s_packed_bytes(0, 128) == 0


def test_argument_checks_before_launch(L):
    p = ctypes.c_void_p(16)  # aligned, never dereferenced: every call below fails its checks first
    odd = ctypes.c_void_p(17)
    assert L.bitnet_pack_i2s(None, 4, 128, p, None) == 1
    assert L.bitnet_pack_i2s(p, 4, 200, p, None) == 2
    assert L.bitnet_pack_i2s(odd, 4, 128, p, None) == 3
    assert L.bitnet_rmsnorm_quant_act(p, 7, None, 1e-6, 1, 128, p, p, p, None) == 4
    assert L.bitnet_rmsnorm_quant_act(p, 0, None, 1e-6, 1, 0, p, p, p, None) == 2
    assert L.bitnet_rmsnorm_quant_act(p, 0, None, 1e-6, 1, 128, None, p, p, None) == 1
    assert L.bitnet_rmsnorm_quant_act(p, 0, None, 1e-6, 0, 128, None, None, None, None) == 0  # T = 0: no-op
    assert L.bitnet_bitlinear(p, p, p, p, 1, 16, 200, p, 0, None, None) == 2
    assert L.bitnet_bitlinear(p, p, p, p, 1, 16, 256, p, 9, None, None) == 4
    assert L.bitnet_bitlinear(p, p, p, odd, 1, 16, 256, p, 0, None, None) == 3
    assert L.bitnet_bitlinear(p, p, p, None, 1, 16, 256, p, 0, None, None) == 1
    assert L.bitnet_bitlinear(p, p, p, p, 0, 16, 256, p, 0, None, None) == 0
    assert L.bitnet_ffn_block(p, 0, None, p, p, None, p, 1, 256, 384, 0, 1e-6, p, 0, None, 0, None) == 5
    assert L.bitnet_ffn_block(p, 0, None, p, p, None, p, 1, 256, 384, 0, 1e-6, p, 0, p, 16, None) == 5
    assert L.bitnet_ffn_block(p, 0, None, p, p, None, p, 1, 256, 300, 0, 1e-6, p, 0, p, 1 << 20, None) == 2
    assert L.bitnet_ffn_block(p, 0, None, p, p, None, p, 1, 256, 384, 5, 1e-6, p, 0, p, 1 << 20, None) == 4
    assert L.bitnet_pack_i2s_prescaled(None, 4, 128, p, None) == 1
    assert L.bitnet_pack_i2s_prescaled(p, 4, 200, p, None) == 2
    assert L.bitnet_pack_i2s_prescaled(p, 4, 128, odd, None) == 3
    assert L.bitnet_validate_i2s(None, 4, 128, p, None) == 1
    assert L.bitnet_validate_i2s(p, 4, 128, None, None) == 1
    assert L.bitnet_validate_i2s(p, 0, 128, p, None) == 2
    assert L.bitnet_validate_i2s(odd, 4, 128, p, None) == 3
    assert L.bitnet_validate_i2s(p, 4, 128, ctypes.c_void_p(20), None) == 3  # counts must be 8-byte aligned


def test_noalloc_checks_arguments_like_ffn_block(L):
    """The no-alloc FFN entry answers invalid arguments with the same status as
    bitnet_ffn_block, before it touches its built-in scratch (no CUDA call is made)."""
    p = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(17)
    big = 1 << 30
    cases = [  # (x, xt, p_gate, T, H, I, act, out, ot)
        (p, 7, p, 1, 256, 384, 0, p, 0),        # bad x dtype
        (p, 0, p, 1, 256, 384, 0, p, 9),        # bad out dtype
        (p, 0, p, 1, 256, 384, 5, p, 0),        # bad activation
        (p, 0, p, 1, 200, 384, 0, p, 0),        # H % 128
        (p, 0, p, 1, 256, 300, 0, p, 0),        # I % 128
        (p, 0, p, 1, 1 << 20, 384, 0, p, 0),    # H beyond the maximum
        (p, 0, p, -1, 256, 384, 0, p, 0),       # negative T
        (None, 0, p, 1, 256, 384, 0, p, 0),     # NULL input
        (p, 0, None, 1, 256, 384, 0, p, 0),     # NULL weights
        (odd, 0, p, 1, 256, 384, 0, p, 0),      # misaligned input
    ]
    for x, xt, pg, T, H, I, act, out, ot in cases:
        want = L.bitnet_ffn_block(x, xt, None, pg, p, None, p, T, H, I, act, 1e-6, out, ot, p, big, None)
        got = L.bitnet_ffn_block_noalloc(x, xt, None, pg, p, None, p, T, H, I, act, 1e-6, out, ot, None)
        assert want != 0 and got == want, (T, H, I, want, got)
    assert L.bitnet_ffn_block_noalloc(p, 0, None, p, p, None, p, 0, 256, 384, 0, 1e-6, p, 0, None) == 0  # T = 0


def test_status_strings(L):
    for code in range(8):
        assert L.bitnet_status_string(code)
    assert L.bitnet_status_string(99) == b"unknown status"


def test_ffn_workspace_layout(L):
    off = tb.ffn_workspace_offsets(3, 256, 384)
    assert len(off) == 8 and off == sorted(off) and all(o % 256 == 0 for o in off)
    assert off[1] >= 3 * 256 and off[4] - off[3] >= 3 * 384 * 4
    assert tb.ffn_workspace_bytes(3, 256, 384) >= off[7] + 36
    boff = tb.block_workspace_offsets(3, 256, 256, 384)
    assert len(boff) == 7 and boff == sorted(boff)
    assert tb.block_workspace_bytes(3, 256, 256, 384) == boff[6] + tb.ffn_workspace_bytes(3, 256, 384)

"""CUDA path (through the C ABI) against the CPU oracle, element by element, on the same
seeded inputs.  Bytes, int8 activations, activation sums and int32 accumulators must be
bit-exact; float outputs within 1e-3 (fp32) / 1e-2 (bf16) max relative error."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import ternary_bitlinear_quantized_b200 as tb
import workloads
from oracle import bitnet_oracle as O
from tests.parity_util import act_to_np, assert_close, bf16_to_np, oracle_rows, out_to_np
from tests.tie_inputs import tie_activations, tie_weights

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tb.lib()
    yield
    assert tb.device_status() == 0


def gpu_pack(W: torch.Tensor) -> torch.Tensor:
    return tb.pack_i2s(W.to(DEV).contiguous())


# ----------------------------------------------------------------------------- a1: pack

@pytest.mark.parametrize("N,K,seed", [(1, 128, 0), (17, 384, 1), (300, 640, 2), (1000, 2560, 3), (64, 6912, 4)])
def test_pack_bytes_bitexact(N, K, seed):
    W = workloads.latent_weight(N, K, seed, "pack")
    got = gpu_pack(W).cpu().numpy()
    ref = O.pack_i2s(W.numpy())
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


def test_pack_special_cases():
    zero = torch.zeros(2, 256)
    assert np.array_equal(gpu_pack(zero).cpu().numpy(), O.pack_i2s(zero.numpy()))
    k = np.arange(128)
    hand = np.where(k % 3 == 0, 0.02, np.where(k % 3 == 1, -0.02, 0.0)).astype(np.float32).reshape(1, 128)
    assert np.array_equal(gpu_pack(torch.from_numpy(hand)).cpu().numpy(), O.pack_i2s(hand))
    rng = np.random.default_rng(5)
    tern = (rng.integers(-1, 2, size=(33, 512)) * 0.0375).astype(np.float32)
    got = gpu_pack(torch.from_numpy(tern)).cpu().numpy()
    assert np.array_equal(got, O.pack_i2s(tern))
    codes, _ = O.unpack_i2s(got, 33, 512)
    assert np.array_equal(codes.astype(int) - 1, np.rint(tern / 0.0375).astype(int))


def test_pack_repeatable_across_streams():
    W = workloads.latent_weight(257, 1024, 9, "rep").to(DEV)
    a = tb.pack_i2s(W)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = tb.pack_i2s(W)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ----------------------------------------------------------------------------- a2: quant

@pytest.mark.parametrize("N,K,case", [(1, 128, "ternary"), (17, 384, "ternary"), (300, 640, "ternary"),
                                      (64, 6912, "ternary"), (33, 256, "latent"), (5, 128, "leading_zeros"),
                                      (3, 256, "zeros")])
def test_pack_prescaled_bytes_bitexact(N, K, case):
    """Prescaled packing (scale = first non-zero |w|) against the oracle, byte for byte."""
    rng = np.random.default_rng(N * 7 + K)
    if case == "ternary":
        t = rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(N, K), p=[0.35, 0.3, 0.35])
        W = t.astype(np.float32) * np.float32(0.0213 * (1 + N % 5))
    elif case == "latent":
        W = workloads.latent_weight(N, K, 5, "prescaled").numpy()
    elif case == "leading_zeros":
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        W.reshape(-1)[: N * K // 2 + 3] = 0.0
    else:
        W = np.zeros((N, K), dtype=np.float32)
    got = tb.pack_i2s_prescaled(torch.from_numpy(W).to(DEV)).cpu().numpy()
    ref = O.pack_i2s_prescaled(W)
    assert np.array_equal(got, ref)
    if case == "ternary":
        codes, beta = O.unpack_i2s(got, N, K)
        assert np.array_equal(codes.astype(np.int16) - 1, t)


@pytest.mark.parametrize("N,K", [(4, 256), (300, 640), (2560, 2560)])
def test_validate_i2s_matches_oracle(N, K):
    W = workloads.latent_weight(N, K, 11, "validate")
    p = gpu_pack(W)
    assert tuple(tb.validate_i2s(p, N, K).cpu().tolist()) == (0, 0, 0)
    bad = p.cpu().numpy().copy()
    rng = np.random.default_rng(N + K)
    nb = N * K // 4
    idx = rng.choice(nb, size=min(50, nb), replace=False)
    bad[idx] |= 0b00110000                      # field 1 of those bytes -> 3
    bad[nb + 9] = 1                             # a trailer byte after the scale
    bad[nb:nb + 4] = np.frombuffer(np.asarray([np.nan], dtype="<f4").tobytes(), dtype=np.uint8)
    got = tuple(tb.validate_i2s(torch.from_numpy(bad).to(DEV), N, K).cpu().tolist())
    assert got == O.validate_i2s(bad, N, K) == (len(idx), 1, 1)


@pytest.mark.parametrize("T,K,dtype,use_gain,outliers", [
    (1, 2560, torch.bfloat16, True, False),
    (5, 640, torch.bfloat16, True, True),
    (3, 6912, torch.float32, True, False),
    (4, 2560, torch.bfloat16, False, False),
    (2, 100, torch.bfloat16, True, False),     # K not a multiple of 8: scalar path
    (3, 27648, torch.float32, True, False),
    (2, 28672, torch.bfloat16, True, True),
    (130, 384, torch.bfloat16, True, True),
    (300, 27648, torch.float32, True, False),   # long fp32 rows, many of them: persistent double-buffered kernel
    (301, 12288, torch.float32, False, True),
    (300, 1020, torch.float32, True, True),     # long-row kernel, rows of <= 1024 values: the general sum terms
    (297, 9000, torch.float32, True, True),     # long-row kernel, K not a multiple of 16
])
def test_quant_bitexact(T, K, dtype, use_gain, outliers):
    x = workloads.activations(T, K, 11, "quant", outliers)
    if dtype == torch.float32:
        x = x.float() * 3.0 + 0.25 * torch.randn(T, K, generator=torch.Generator().manual_seed(1))
    x[T // 2] = 0  # a zero token
    g = workloads.gain(K, 11, "quant") if use_gain else None
    q, s, sq = tb.rmsnorm_quant_act(x.to(DEV), None if g is None else g.to(DEV), 1e-6)
    rq, rs, rsq = O.rmsnorm_quant_act(act_to_np(x), None if g is None else g.numpy(), 1e-6)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(sq.cpu().numpy(), rsq)


# ----------------------------------------------------------------------------- rounding ties

def test_pack_ties_bitexact():
    """Weights at exactly +-0.5 and +-1.5 times beta (beta = 2**-6): the codes take the
    half-to-even decision, so a kernel that rounds half away from zero differs here."""
    W = tie_weights(N=160, K=256)
    got = gpu_pack(torch.from_numpy(W)).cpu().numpy()
    ref = O.pack_i2s(W)
    assert np.array_equal(got, ref)
    codes, beta = O.unpack_i2s(got, 160, 256)
    assert beta == np.float32(2.0 ** -6)
    assert np.array_equal(codes.astype(np.int16) - 1, np.where(np.abs(W) < 2.0 ** -6, 0, np.sign(W)).astype(np.int16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quant_ties_bitexact(dtype):
    """Activations (n + 1/2)/64 with absmax 127/64 (s_x = 64): every entry is a .5 tie."""
    x = tie_activations()
    xt = torch.from_numpy(x).to(dtype)
    assert np.array_equal(act_to_np(xt), x)  # exact in bf16
    q, s, sq = tb.rmsnorm_quant_act(xt.to(DEV), None, 1e-6)
    rq, rs, rsq = O.rmsnorm_quant_act(x, None, 1e-6)
    assert np.all(rs == np.float32(64.0))
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(sq.cpu().numpy(), rsq)


@pytest.mark.parametrize("reps", [1, 14])  # 3 tokens (decode engine) and 42 (tensor-core path)
def test_bitlinear_ties_bitexact(reps):
    """Tie activations through the product with tie weights: q, codes, int32 accumulators and
    outputs against the oracle, bit for bit."""
    x = np.tile(tie_activations(), (reps, 1))
    T, K = x.shape
    W = tie_weights(N=160, K=K)
    packed_ref = O.pack_i2s(W)
    packed = gpu_pack(torch.from_numpy(W))
    assert np.array_equal(packed.cpu().numpy(), packed_ref)
    q, s, sq = tb.rmsnorm_quant_act(torch.from_numpy(x).to(torch.bfloat16).to(DEV), None, 1e-6)
    acc = torch.empty(T, 160, dtype=torch.int32, device=DEV)
    out = tb.bitlinear(q, s, sq, packed, 160, torch.float32, acc_debug=acc)
    rq, rs, rsq = O.rmsnorm_quant_act(x, None, 1e-6)
    ref, racc = O.bitlinear(rq, rs, rsq, packed_ref, 160, K, "f32", return_acc=True)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(out_to_np(out).view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------------------------- a3/a4: product

def run_bitlinear(T, N, K, seed, out_dtype, outliers=False):
    W = workloads.latent_weight(N, K, seed, "bl")
    x = workloads.activations(T, K, seed, "bl", outliers)
    g = workloads.gain(K, seed, "bl")
    packed_ref = O.pack_i2s(W.numpy())
    packed = torch.from_numpy(packed_ref).to(DEV)  # oracle bytes: this test isolates the product
    q, s, sq = tb.rmsnorm_quant_act(x.to(DEV), g.to(DEV), 1e-6)
    acc = torch.empty(T, N, dtype=torch.int32, device=DEV)
    out = tb.bitlinear(q, s, sq, packed, N, out_dtype, acc_debug=acc)
    rq, rs, rsq = O.rmsnorm_quant_act(bf16_to_np(x), g.numpy(), 1e-6)
    dt = "bf16" if out_dtype == torch.bfloat16 else "f32"
    ref, racc = O.bitlinear(rq, rs, rsq, packed_ref, N, K, dt, return_acc=True)
    return out, acc, ref, racc, dt


@pytest.mark.parametrize("T,N,K", [(1, 1, 128), (1, 300, 640), (3, 17, 384), (8, 2560, 2560), (9, 100, 1024),
                                   (16, 64, 2560), (17, 48, 256), (33, 40, 640), (1, 640, 6912), (2, 48, 8192),
                                   (4, 33, 28672), (1, 28672, 128), (12, 150, 1152),
                                   (64, 300, 640), (200, 130, 1280), (300, 256, 256), (513, 384, 2560)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_bitlinear_parity(T, N, K, out_dtype):
    out, acc, ref, racc, dt = run_bitlinear(T, N, K, T * 1000 + N, out_dtype)
    assert np.array_equal(acc.cpu().numpy(), racc)
    got = out_to_np(out)
    assert_close(got, ref, dt)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))  # same op sequence: bit-identical


@pytest.mark.parametrize("T", [2, 100])
def test_bitlinear_group_matches_singles(T):
    K = 2560
    Ns = [2560, 640, 640]
    x = workloads.activations(T, K, 3, "grp")
    g = workloads.gain(K, 3, "grp")
    Ws = [workloads.latent_weight(n, K, 3, f"grp{i}") for i, n in enumerate(Ns)]
    packs_ref = [O.pack_i2s(W.numpy()) for W in Ws]
    packs = [torch.from_numpy(p).to(DEV) for p in packs_ref]
    q, s, sq = tb.rmsnorm_quant_act(x.to(DEV), g.to(DEV), 1e-6)
    outs = tb.bitlinear_group(q, s, sq, packs, Ns, torch.bfloat16)
    rq, rs, rsq = O.rmsnorm_quant_act(bf16_to_np(x), g.numpy(), 1e-6)
    for o, p, n in zip(outs, packs_ref, Ns):
        ref = O.bitlinear(rq, rs, rsq, p, n, K, "bf16")
        assert np.array_equal(out_to_np(o), ref)


# ----------------------------------------------------------------------------- a5-a7: FFN block

def run_ffn(T, H, I, act, seed, out_dtype=torch.bfloat16, x_dtype=torch.bfloat16):
    sh = workloads.BlockShape("ffn-test", hidden=H, n_q=H, n_kv=H, inter=I, act=act)
    d = workloads.block_inputs(sh, T, seed, ffn_only=True)
    x = d["x"] if x_dtype == torch.bfloat16 else d["x"].float()
    pr = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in ("gate", "up", "down")}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    code = tb.RELU2 if act == "relu2" else tb.SILU
    out = tb.ffn_block(x.to(DEV), d["g_ffn_norm"].to(DEV), pg["gate"], pg["up"], d["g_ffn_sub_norm"].to(DEV),
                       pg["down"], I, code, 1e-6, out_dtype, ws=ws)
    dt = "bf16" if out_dtype == torch.bfloat16 else "f32"
    ref, mid = O.ffn_block(act_to_np(x), d["g_ffn_norm"].numpy(), pr["gate"], pr["up"], d["g_ffn_sub_norm"].numpy(),
                           pr["down"], H, I, act, 1e-6, dt, return_intermediates=True)
    return out, ws, ref, mid, dt


@pytest.mark.parametrize("act", ["relu2", "silu"])
@pytest.mark.parametrize("T,H,I", [(1, 256, 384), (3, 640, 1280), (17, 256, 640), (2, 8192, 512), (10, 1152, 2304),
                                   (64, 512, 768), (130, 384, 1280), (3, 8192, 512), (1, 256, 16512),
                                   (16, 2048, 1024), (300, 256, 9216)])
def test_ffn_block_parity(act, T, H, I):
    out, ws, ref, mid, dt = run_ffn(T, H, I, act, seed=T + H)
    off = tb.ffn_workspace_offsets(T, H, I)
    wsn = ws.cpu().numpy()
    q_x = wsn[off[0]:off[0] + T * H].view(np.int8).reshape(T, H)
    h = wsn[off[3]:off[3] + T * I * 4].view(np.float32).reshape(T, I)
    q_h = wsn[off[4]:off[4] + T * I].view(np.int8).reshape(T, I)
    sum_h = wsn[off[6]:off[6] + T * 4].view(np.int32)
    assert np.array_equal(q_x, mid["q"])
    assert np.array_equal(h.view(np.uint32), mid["h"].view(np.uint32))
    assert np.array_equal(q_h, mid["q_h"])
    assert np.array_equal(sum_h, mid["sum_h"])
    got = out_to_np(out)
    assert_close(got, ref, dt)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("T,H,I", [(1, 512, 9216), (4, 256, 8320)])
def test_ffn_block_distributed_sub_norm_without_gain_twice(T, H, I):
    """The decode path spreads ffn_sub_norm over all CTAs when h is too long to quantise in
    every CTA; here with ffn_sub_norm switched off (y = h) and the workspace reused."""
    sh = workloads.BlockShape("ffn-nog", hidden=H, n_q=H, n_kv=H, inter=I, act="relu2")
    d = workloads.block_inputs(sh, T, T + I, ffn_only=True)
    pr = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in ("gate", "up", "down")}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    ref, mid = O.ffn_block(bf16_to_np(d["x"]), d["g_ffn_norm"].numpy(), pr["gate"], pr["up"], None, pr["down"], H, I,
                           "relu2", 1e-6, "bf16", return_intermediates=True)
    off = tb.ffn_workspace_offsets(T, H, I)
    for _ in range(2):
        out = tb.ffn_block(d["x"].to(DEV), d["g_ffn_norm"].to(DEV), pg["gate"], pg["up"], None, pg["down"], I,
                           tb.RELU2, 1e-6, torch.bfloat16, ws=ws)
        torch.cuda.synchronize()
        wsn = ws.cpu().numpy()
        assert np.array_equal(wsn[off[4]:off[4] + T * I].view(np.int8).reshape(T, I), mid["q_h"])
        assert np.array_equal(wsn[off[6]:off[6] + T * 4].view(np.int32), mid["sum_h"])
        assert np.array_equal(out_to_np(out).view(np.uint32), ref.view(np.uint32))
    assert tb.device_status() == 0


@pytest.mark.parametrize("T", [1, 3])
def test_ffn_block_distributed_sub_norm_fallback(T):
    """The grid-wide ffn_sub_norm takes the exact sum from each CTA's candidate grids unless a
    CTA's max |h| is far below the row's (its candidates then miss the row's grid) -- here
    the second half of the gate rows has a single non-zero weight each, so the h of those
    rows is about 2^-6 of the rest and the fallback round runs; bit-exact either way."""
    H, I = 512, 16512
    sh = workloads.BlockShape("ffn-fb", hidden=H, n_q=H, n_kv=H, inter=I, act="relu2")
    d = workloads.block_inputs(sh, T, 77, ffn_only=True)
    Wg = d["W_gate"].clone()
    Wg[I // 2:] = 0.0
    Wg[I // 2:, int(torch.argmax(d["x"][0].float()))] = 0.05  # token 0's largest input: g > 0, relu2(g) > 0
    pr = {"gate": O.pack_i2s(Wg.numpy()), "up": O.pack_i2s(d["W_up"].numpy()), "down": O.pack_i2s(d["W_down"].numpy())}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    ref, mid = O.ffn_block(bf16_to_np(d["x"]), d["g_ffn_norm"].numpy(), pr["gate"], pr["up"],
                           d["g_ffn_sub_norm"].numpy(), pr["down"], H, I, "relu2", 1e-6, "bf16",
                           return_intermediates=True)
    nz = np.abs(mid["h"][0, I // 2:])
    assert np.max(nz) > 0 and np.max(nz) < np.max(np.abs(mid["h"][0])) * 2.0 ** -4  # far below the row's max
    off = tb.ffn_workspace_offsets(T, H, I)
    for _ in range(2):
        out = tb.ffn_block(d["x"].to(DEV), d["g_ffn_norm"].to(DEV), pg["gate"], pg["up"], d["g_ffn_sub_norm"].to(DEV),
                           pg["down"], I, tb.RELU2, 1e-6, torch.bfloat16, ws=ws)
        torch.cuda.synchronize()
        wsn = ws.cpu().numpy()
        assert np.array_equal(wsn[off[4]:off[4] + T * I].view(np.int8).reshape(T, I), mid["q_h"])
        assert np.array_equal(wsn[off[6]:off[6] + T * 4].view(np.int32), mid["sum_h"])
        assert np.array_equal(out_to_np(out).view(np.uint32), ref.view(np.uint32))
    assert tb.device_status() == 0


@pytest.mark.parametrize("T,mode", [(1, "all"), (3, "all"), (300, "all"), (300, "tile0")])
def test_ffn_block_distributed_sub_norm_ymax_ties(T, mode):
    """max |y| of the decode engine's grid-wide ffn_sub_norm comes from each CTA's (h, g)
    candidate near its largest |h g| unless a CTA has several; here every gate row and every up
    row is the same and the sub-norm gain is constant ("all": |h g| ties everywhere), or only the
    first 128 rows of gate and up and the first 128 gain values are ("tile0"), so the grid-barrier
    path runs.  T = 300 takes the prefill path (long-row quantisation of h) on the same ties.
    Bit-exact either way."""
    H, I = 512, 16512
    sh = workloads.BlockShape("ffn-ties", hidden=H, n_q=H, n_kv=H, inter=I, act="relu2")
    d = workloads.block_inputs(sh, T, 78, ffn_only=True)
    if mode == "all":
        Wg = d["W_gate"][:1].repeat(I, 1).contiguous()
        Wu = d["W_up"][:1].repeat(I, 1).contiguous()
        g_sub = torch.full_like(d["g_ffn_sub_norm"], 1.5)
    else:
        Wg, Wu, g_sub = d["W_gate"].clone(), d["W_up"].clone(), d["g_ffn_sub_norm"].clone()
        Wg[:128] = Wg[:1]
        Wu[:128] = Wu[:1]
        g_sub[:128] = 1.5
    pr = {"gate": O.pack_i2s(Wg.numpy()), "up": O.pack_i2s(Wu.numpy()), "down": O.pack_i2s(d["W_down"].numpy())}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    ws = torch.zeros(tb.ffn_workspace_bytes(T, H, I), dtype=torch.uint8, device=DEV)
    ref, mid = O.ffn_block(bf16_to_np(d["x"]), d["g_ffn_norm"].numpy(), pr["gate"], pr["up"], g_sub.numpy(),
                           pr["down"], H, I, "relu2", 1e-6, "bf16", return_intermediates=True)
    if mode == "all":
        assert np.all(mid["h"] == mid["h"][:, :1])  # every row of h the same
    else:
        assert np.all(mid["h"][:, :128] == mid["h"][:, :1])
    off = tb.ffn_workspace_offsets(T, H, I)
    for _ in range(2):
        out = tb.ffn_block(d["x"].to(DEV), d["g_ffn_norm"].to(DEV), pg["gate"], pg["up"], g_sub.to(DEV),
                           pg["down"], I, tb.RELU2, 1e-6, torch.bfloat16, ws=ws)
        torch.cuda.synchronize()
        wsn = ws.cpu().numpy()
        assert np.array_equal(wsn[off[4]:off[4] + T * I].view(np.int8).reshape(T, I), mid["q_h"])
        assert np.array_equal(wsn[off[6]:off[6] + T * 4].view(np.int32), mid["sum_h"])
        assert np.array_equal(out_to_np(out).view(np.uint32), ref.view(np.uint32))
    assert tb.device_status() == 0


def test_ffn_block_fp32_io():
    out, _, ref, _, dt = run_ffn(2, 384, 512, "silu", seed=5, out_dtype=torch.float32, x_dtype=torch.float32)
    assert np.array_equal(out_to_np(out).view(np.uint32), ref.view(np.uint32))


def test_empty_token_batch_is_noop():
    q = torch.empty(0, 256, dtype=torch.int8, device=DEV)
    s = torch.empty(0, dtype=torch.float32, device=DEV)
    sq = torch.empty(0, dtype=torch.int32, device=DEV)
    packed = gpu_pack(workloads.latent_weight(32, 256, 0, "e"))
    out = tb.bitlinear(q, s, sq, packed, 32, torch.bfloat16)
    assert out.shape == (0, 32)
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    qq, _, _ = tb.rmsnorm_quant_act(x, None)
    assert qq.shape == (0, 256)


# ----------------------------------------------------------------------------- decoder block

def run_block(T, H, NQ, NKV, I, act, seed, out_dtype=torch.bfloat16, calls=1):
    sh = workloads.BlockShape("blk-test", hidden=H, n_q=NQ, n_kv=NKV, inter=I, act=act)
    d = workloads.block_inputs(sh, T, seed)
    pr = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in sh.tensors()}
    pg = {nm: torch.from_numpy(v).to(DEV) for nm, v in pr.items()}
    gains = {k[2:]: v.to(DEV) for k, v in d.items() if k.startswith("g_")}
    code = tb.RELU2 if act == "relu2" else tb.SILU
    ws = torch.zeros(tb.block_workspace_bytes(T, H, NQ, I), dtype=torch.uint8, device=DEV)
    outs = [tb.decoder_block(d["x"].to(DEV), d["attn_out"].to(DEV), gains, pg, NKV, I, code, 1e-6, out_dtype, ws=ws)
            for _ in range(calls)]
    dt = "bf16" if out_dtype == torch.bfloat16 else "f32"
    ref = O.decoder_block(bf16_to_np(d["x"]), bf16_to_np(d["attn_out"]), {k: v.numpy() for k, v in
                          {k[2:]: v for k, v in d.items() if k.startswith("g_")}.items()}, pr, sh.tensors(), act,
                          1e-6, dt)
    return outs, ref, dt, ws


@pytest.mark.parametrize("T,H,NQ,NKV,I,act", [
    (1, 256, 256, 128, 384, "relu2"),
    (1, 2560, 2560, 640, 6912, "relu2"),     # the 2B4T shapes at decode
    (5, 512, 512, 256, 1024, "silu"),
    (16, 1024, 1024, 256, 2048, "relu2"),    # T * K above the per-CTA quantisation limit
    (3, 8192, 1024, 128, 640, "silu"),       # large hidden: QUANT phases
    (40, 384, 384, 128, 640, "relu2"),       # tensor-core path
])
def test_decoder_block_parity(T, H, NQ, NKV, I, act):
    outs, ref, dt, ws = run_block(T, H, NQ, NKV, I, act, seed=T + H, calls=2)
    for name in ("q", "k", "v", "o", "ffn"):
        for o in outs:  # the second call reuses the workspace (its barrier counters were reset)
            got = out_to_np(o[name])
            assert_close(got, ref[name], dt)
            assert np.array_equal(got.view(np.uint32), ref[name].view(np.uint32)), name
    off = tb.block_workspace_offsets(T, H, NQ, I)
    offf = tb.ffn_workspace_offsets(T, H, I)
    counters = ws[off[6] + offf[7]: off[6] + offf[7] + 64].cpu().numpy()
    assert not counters.any()

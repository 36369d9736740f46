"""Pins of the CPU oracle to things other than itself (no GPU).

Each test checks the oracle against what the BitNet pages and the mathematics fix:
hand-worked golden bytes (tests/golden/), exact rational arithmetic, closed forms,
invariants, special cases that reduce to a library routine, and brute force on tiny
inputs written independently of the oracle's vectorised code.  The last group plants
plausible mistakes in the oracle and checks that a pin catches each one.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import bitnet_oracle as O
import workloads
from tests.tie_inputs import tie_activations, tie_weights

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


# ----------------------------------------------------------------------------- helpers

def fraction_to_f32(fr: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of an exact rational."""
    c = F32(float(fr))
    best = None
    for cand in (np.nextafter(c, F32(-np.inf)), c, np.nextafter(c, F32(np.inf))):
        d = abs(Fraction(float(cand)) - fr)
        key = (d, int(np.asarray(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return F32(best[1])


def ulp_f32(x) -> float:
    x = F32(abs(x))
    return float(np.nextafter(x, F32(np.inf)) - x)


def brute_unpack(packed: np.ndarray, N: int, K: int):
    """Pure-Python decode of the interleaved 128/32 layout, element by element."""
    data = bytes(np.asarray(packed, dtype=np.uint8)[: N * K // 4])
    codes = [[None] * K for _ in range(N)]
    for b in range(N * K // 128):
        for i in range(32):
            byte = data[32 * b + i]
            for g in range(4):
                flat = 128 * b + 32 * g + i
                codes[flat // K][flat % K] = (byte >> (6 - 2 * g)) & 3
    beta = np.frombuffer(bytes(packed[N * K // 4: N * K // 4 + 4]), dtype="<f4")[0]
    return codes, F32(beta)


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def bf16_inputs(T, K, seed=0, outliers=False):
    x = workloads.activations(T, K, seed, "oracle-test", outliers)
    return O.bf16_bits_to_f32(x.view(torch.int16).numpy().view(np.uint16))


# ----------------------------------------------------------------------------- a1: pack

def handworked_weights():
    k = np.arange(128)
    w = np.where(k % 3 == 0, F32(0.02), np.where(k % 3 == 1, F32(-0.02), F32(0.0)))
    return w.astype(F32).reshape(1, 128)


def test_pack_handworked_block_golden():
    g = read_golden("i2s_block_k128.txt")
    W = handworked_weights()
    packed = O.pack_i2s(W)
    assert packed.size == 32 + 32
    assert [f"{b:02x}" for b in packed[:32]] == g["bytes"]
    beta_exact = fraction_to_f32(Fraction(int(g["nonzeros"][0])) * Fraction(float(F32(0.02))) / 128)
    beta = np.frombuffer(packed[32:36].tobytes(), dtype="<f4")[0]
    assert beta == beta_exact
    assert not packed[36:].any() and packed[36:].size == int(g["trailer_zero_bytes"][0])


def test_pack_zero_tensor_golden():
    g = read_golden("i2s_zero_tensor.txt")
    packed = O.pack_i2s(np.zeros((2, 256), F32))
    assert np.all(packed[: int(g["count"][0])] == int(g["byte"][0], 16))
    assert np.frombuffer(packed[128:132].tobytes(), "<f4")[0] == F32(float(g["beta_f32"][0]))
    assert not packed[132:].any()


def test_pack_rejects_ragged_rows():
    with pytest.raises(ValueError):
        O.pack_i2s(np.zeros((4, 200), F32))


def test_packed_size_and_3b_tensor_sizes():
    g = read_golden("tensor_sizes_3b.txt")
    for name, (r, c, size, unit) in g.items():
        nbytes = int(r) * int(c) * 4
        printed = float(size)
        got = nbytes / 2 ** 20
        assert abs(got - printed) <= 0.006 * max(printed, 1), (name, got, printed)
        if int(c) % 128 == 0 and int(c) > 1:
            assert O.i2s_packed_bytes(int(r), int(c)) == int(r) * int(c) // 4 + 32
    # I2_S is 2 bits per weight: 16x below fp32 and 8x below bf16, up to the trailer.
    assert O.i2s_packed_bytes(3200, 8640) == 6_912_032
    assert abs(2 * 3200 * 8640 / O.i2s_packed_bytes(3200, 8640) - 8.0) < 1e-4


@pytest.mark.parametrize("N,K,seed", [(3, 128, 0), (5, 256, 1), (17, 384, 2), (64, 1024, 3)])
def test_pack_matches_bruteforce_decode(N, K, seed):
    W = workloads.latent_weight(N, K, seed, "pin").numpy()
    packed = O.pack_i2s(W)
    assert packed.size == N * K // 4 + 32
    codes, beta = brute_unpack(packed, N, K)
    # Independent codes: round-half-even of W / beta in exact arithmetic for the same fp32 s_w.
    s_w = F32(1.0) / beta
    for n in range(N):
        for k in range(K):
            prod = Fraction(float(W[n, k])) * Fraction(float(s_w))
            v = float(F32(float(prod)))  # fp32 product, correctly rounded
            want = max(-1, min(1, round(fraction_to_f32(Fraction(v)).item()))) + 1
            assert codes[n][k] == want, (n, k)
    vc, vb = O.unpack_i2s(packed, N, K)
    assert vb == beta and np.array_equal(vc, np.array(codes, dtype=np.uint8))


@pytest.mark.parametrize("N,K,seed", [(8, 256, 0), (33, 512, 1), (100, 1280, 2)])
def test_beta_is_exact_mean_rounded(N, K, seed):
    W = workloads.latent_weight(N, K, seed, "beta").numpy()
    exact = sum(Fraction(float(abs(v))) for v in W.ravel()) / (N * K)
    beta = O.absmean_scale(W)
    want = fraction_to_f32(exact)
    assert abs(float(beta) - float(want)) <= ulp_f32(want), (beta, want)


@pytest.mark.parametrize("alpha", [1e-4, 3e-3, 0.0123, 0.5, 1.0, 7.25, 300.0])
def test_scale_invariance_of_ternary_inputs(alpha):
    rng = np.random.default_rng(int(alpha * 1e4) % 2**31)
    T = rng.integers(-1, 2, size=(6, 256)).astype(F32)
    T[0, :] = 0.0
    T[0, 5] = 1.0  # a row with a single non-zero
    packed = O.pack_i2s(F32(alpha) * T)
    codes, beta = brute_unpack(packed, 6, 256)
    assert np.array_equal(np.array(codes) - 1, T.astype(int))
    # Re-packing the dequantised tensor keeps the codes (ternary x scale is a fixed point).
    W2 = (np.array(codes, dtype=F32) - 1) * beta
    assert np.array_equal(O.pack_i2s(W2)[: 6 * 256 // 4], packed[: 6 * 256 // 4])


# ----------------------------------------------------------------------------- a2: norm + quant

@pytest.mark.parametrize("K,seed", [(128, 0), (2560, 1), (6912, 2)])
def test_mean_square_is_exact_mean_rounded(K, seed):
    x = bf16_inputs(3, K, seed)
    for t in range(3):
        exact = sum(Fraction(float(v)) ** 2 for v in x[t]) / K
        ms = O.fixed_point_mean_f32(x[t].astype(np.float64) ** 2)
        want = fraction_to_f32(exact)
        assert abs(float(ms) - float(want)) <= ulp_f32(want)


def test_fixed_point_sum_is_order_free_and_bounded():
    rng = np.random.default_rng(0)
    v = np.abs(rng.standard_normal(10_000)) ** 3
    S1, e1 = O.fixed_point_sum(v)
    S2, e2 = O.fixed_point_sum(v[::-1].copy())
    S3, e3 = O.fixed_point_sum(rng.permutation(v))
    assert S1 == S2 == S3 and e1 == e2 == e3
    assert 0 < S1 < 2 ** 62
    assert abs(math.ldexp(S1, -e1) - math.fsum(v)) <= 10_000 * math.ldexp(1.0, -e1)


@pytest.mark.parametrize("use_norm", [True, False])
def test_quant_invariants(use_norm):
    T, K = 7, 640
    x = bf16_inputs(T, K, 4)
    x[3] = 0.0  # a zero token
    g = workloads.gain(K, 0, "pin").numpy() if use_norm else None
    q, s, sq = O.rmsnorm_quant_act(x, g, 1e-6)
    assert q.dtype == np.int8 and s.dtype == F32 and sq.dtype == np.int32
    for t in range(T):
        if t == 3:
            assert not q[t].any() and s[t] == F32(127.0) / F32(1e-5) and sq[t] == 0
            continue
        xd = x[t].astype(np.float64)
        y = xd / math.sqrt(np.mean(xd * xd) + 1e-6) * g.astype(np.float64) if use_norm else xd
        a = np.max(np.abs(y))
        assert abs(float(s[t]) - 127.0 / a) <= 1e-6 * 127.0 / a
        assert np.max(np.abs(q[t])) == 127
        assert np.abs(q[t][np.argmax(np.abs(y))]) == 127
        assert np.all(np.abs(q[t] - y * 127.0 / a) <= 0.5 + 1e-4)
        assert sq[t] == int(q[t].astype(np.int64).sum())


def test_quant_without_gain_is_plain_absmax():
    x = bf16_inputs(2, 256, 9)
    q, s, _ = O.rmsnorm_quant_act(x, None, 1e-6)
    for t in range(2):
        a = max(abs(float(v)) for v in x[t])
        assert s[t] == fraction_to_f32(Fraction(127) / Fraction(float(F32(a))))
        for k in range(256):
            exact = Fraction(float(x[t, k])) * Fraction(float(s[t]))
            v = float(F32(float(exact)))  # the fp32 product, correctly rounded
            assert q[t, k] == max(-128, min(127, round(v)))


def test_quant_ties_round_half_even():
    # amax = 127/64 makes s_x = 64 exactly, so x = (n + 0.5)/64 lands on a tie.
    x = np.zeros((1, 128), F32)
    x[0, 0] = F32(127.0 / 64.0)
    halves = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 100.5]
    for i, h in enumerate(halves):
        x[0, 1 + i] = F32(h / 64.0)
    q, s, _ = O.rmsnorm_quant_act(x, None, 1e-6)
    assert s[0] == F32(64.0)
    assert list(q[0, 1:1 + len(halves)]) == [0, 2, 2, 4, 0, -2, -2, 100]


def test_ties_of_codes_and_activations_round_half_even():
    """The tie fixtures land on exact .5 ties and round half to even: weights +-0.5 beta -> 0,
    +-1.5 beta -> +-1 (after the clamp); activations (n + 1/2)/64 with s_x = 64 -> the even
    neighbour."""
    W = tie_weights()
    assert O.absmean_scale(W) == F32(2.0 ** -6)
    codes, _ = O.unpack_i2s(O.pack_i2s(W), *W.shape)
    want = np.where(np.abs(W) < 2.0 ** -6, 0, np.sign(W)).astype(np.int16)
    assert np.array_equal(codes.astype(np.int16) - 1, want)
    x = tie_activations()
    q, s, _ = O.rmsnorm_quant_act(x, None, 1e-6)
    assert np.all(s == F32(64.0))
    for t in range(x.shape[0]):
        for k in range(x.shape[1]):
            v = Fraction(float(x[t, k])) * 64
            lo = math.floor(v)
            want_q = lo if (v - lo != Fraction(1, 2) or lo % 2 == 0) else lo + 1
            assert q[t, k] == max(-128, min(127, want_q))


def test_rmsnorm_matches_textbook():
    x = bf16_inputs(4, 2560, 5)
    g = workloads.gain(2560, 0, "pin").numpy()
    # y is not returned; check through s_x, which is 127 / max|y|.
    _, s, _ = O.rmsnorm_quant_act(x, g, 1e-6)
    for t in range(4):
        xd = x[t].astype(np.float64)
        y = xd / math.sqrt(float(np.mean(xd * xd)) + 1e-6) * g.astype(np.float64)
        assert abs(float(s[t]) * np.max(np.abs(y)) - 127.0) <= 127.0 * 4e-7


# ----------------------------------------------------------------------------- a3/a4: dot + dequant

@pytest.mark.parametrize("T,N,K,seed", [(1, 1, 128, 0), (2, 3, 128, 1), (3, 4, 256, 2), (4, 2, 384, 3)])
def test_dot_bruteforce(T, N, K, seed):
    W = workloads.latent_weight(N, K, seed, "dot").numpy()
    packed = O.pack_i2s(W)
    x = bf16_inputs(T, K, seed)
    q, s, sq = O.rmsnorm_quant_act(x, None, 1e-6)
    acc = O.bitlinear_acc(q, sq, packed, N, K)
    codes, beta = brute_unpack(packed, N, K)
    out = O.bitlinear(q, s, sq, packed, N, K, "f32")
    for t in range(T):
        for n in range(N):
            want = sum(int(q[t, k]) * (codes[n][k] - 1) for k in range(K))
            assert acc[t, n] == want
            # Dequantised value in exact arithmetic: acc * beta / s_x.
            exact = Fraction(want) * Fraction(float(beta)) / Fraction(float(s[t]))
            if want == 0:
                assert out[t, n] == 0
            else:
                assert abs(Fraction(float(out[t, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 22)


@pytest.mark.parametrize("T", [1, 3, 16])
def test_bitlinear_matches_textbook_gemv(T):
    N, K = 96, 1024
    W = workloads.latent_weight(N, K, T, "gemv").numpy()
    packed = O.pack_i2s(W)
    x = bf16_inputs(T, K, T)
    g = workloads.gain(K, T, "gemv").numpy()
    q, s, sq = O.rmsnorm_quant_act(x, g, 1e-6)
    codes, beta = O.unpack_i2s(packed, N, K)
    # Textbook: dequantise both operands in fp64 and take the plain matrix product.
    xq = q.astype(np.float64) / s.astype(np.float64)[:, None]
    wq = (codes.astype(np.float64) - 1.0) * float(beta)
    ref = xq @ wq.T
    # fp64 rounding of the textbook sum: a few ulp of the sum of |terms|.
    slack = 1e-14 * (np.abs(xq) @ np.abs(wq).T)
    for dt, tol in (("f32", 1e-6), ("bf16", 2.0 ** -8)):
        out = O.bitlinear(q, s, sq, packed, N, K, dt).astype(np.float64)
        assert np.all(np.abs(out - ref) <= tol * np.abs(ref) + slack)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(100_000).astype(F32) * 10.0 ** rng.integers(-30, 30, 100_000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38], F32)]).astype(F32)
    got = O.f32_to_bf16_bits(v)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert np.array_equal(O.bf16_bits_to_f32(got), torch.from_numpy(v).to(torch.bfloat16).float().numpy())


# ----------------------------------------------------------------------------- a5: activation

def test_pinned_exp_against_libm():
    xs = np.concatenate([np.linspace(-700, 709, 200_001), np.array([0.0, 1.0, -1.0, math.log(2.0), 1e-300])])
    got = O.pinned_exp(xs)
    want = np.array([math.exp(v) for v in xs])
    rel = np.abs(got - want) / want
    assert np.max(rel) <= 4e-15
    assert O.pinned_exp(np.array([0.0]))[0] == 1.0
    assert O.pinned_exp(np.array([-800.0]))[0] == 0.0 and np.isinf(O.pinned_exp(np.array([710.0]))[0])


def test_silu_matches_torch():
    g = (np.random.default_rng(1).standard_normal(50_000) * 8).astype(F32)
    h = O.ffn_act(g, np.ones_like(g), "silu")
    ref = torch.nn.functional.silu(torch.from_numpy(g).double()).numpy()
    err = np.abs(h.astype(np.float64) - ref)
    assert np.all(err <= np.array([ulp_f32(v) for v in ref]) * 0.5 + 1e-45)


def test_relu2_closed_form():
    rng = np.random.default_rng(2)
    g = rng.standard_normal(20_000).astype(F32)
    u = rng.standard_normal(20_000).astype(F32)
    h = O.ffn_act(g, u, "relu2").astype(np.float64)
    ref = np.where(g > 0, g.astype(np.float64) ** 2 * u, 0.0)
    assert np.all(h[g <= 0] == 0)
    assert np.max(np.abs(h - ref) / np.maximum(np.abs(ref), 1e-30)) <= 2.5e-7


# ----------------------------------------------------------------------------- composed: FFN

def textbook_ffn(x, g_ffn, W_gate, W_up, g_sub, W_down, act, eps=1e-6):
    """BitNetMLP in fp64 from the plain formulas: RMSNorm, absmax int8, absmean ternary."""
    def norm_quant(v, gain):
        v = v.astype(np.float64)
        y = v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + eps) * gain.astype(np.float64)
        s = 127.0 / np.maximum(np.max(np.abs(y), axis=1, keepdims=True), 1e-5)
        return np.clip(np.round(y * s), -128, 127) / s

    def ternary(W):
        W = W.astype(np.float64)
        beta = max(np.mean(np.abs(W)), 1e-5)
        return np.clip(np.round(W / beta), -1, 1) * beta

    xq = norm_quant(x, g_ffn)
    gt, up = xq @ ternary(W_gate).T, xq @ ternary(W_up).T
    a = np.maximum(gt, 0.0) ** 2 if act == "relu2" else gt / (1.0 + np.exp(-gt))
    hq = norm_quant(a * up, g_sub)
    return hq @ ternary(W_down).T


@pytest.mark.parametrize("act", ["relu2", "silu"])
def test_ffn_block_matches_textbook(act):
    H, I, T = 256, 640, 3
    d = {nm: workloads.latent_weight(n, k, 7, "ffn/" + nm).numpy()
         for nm, (n, k) in {"gate": (I, H), "up": (I, H), "down": (H, I)}.items()}
    x = bf16_inputs(T, H, 7)
    g1 = workloads.gain(H, 7, "ffn1").numpy()
    g2 = workloads.gain(I, 7, "ffn2").numpy()
    p = {nm: O.pack_i2s(W) for nm, W in d.items()}
    out = O.ffn_block(x, g1, p["gate"], p["up"], g2, p["down"], H, I, act, 1e-6, "f32")
    ref = textbook_ffn(x, g1, d["gate"], d["up"], g2, d["down"], act)
    assert np.linalg.norm(out - ref) / np.linalg.norm(ref) <= 2e-3


def textbook_block(x, attn_out, gains, W, act, eps=1e-6):
    """The decoder block's projections in fp64 from the plain formulas: q, k, v from x
    through attn_norm; o from the attention output through attn_sub_norm; the FFN (its own
    textbook) from o's output through ffn_norm and ffn_sub_norm."""
    def norm_quant(v, gain):
        v = v.astype(np.float64)
        y = v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + eps) * gain.astype(np.float64)
        s = 127.0 / np.maximum(np.max(np.abs(y), axis=1, keepdims=True), 1e-5)
        return np.clip(np.round(y * s), -128, 127) / s

    def ternary(Wm):
        Wm = Wm.astype(np.float64)
        beta = max(np.mean(np.abs(Wm)), 1e-5)
        return np.clip(np.round(Wm / beta), -1, 1) * beta

    xq = norm_quant(x, gains["attn_norm"])
    out = {nm: xq @ ternary(W[nm]).T for nm in ("q", "k", "v")}
    out["o"] = norm_quant(attn_out, gains["attn_sub_norm"]) @ ternary(W["o"]).T
    out["ffn"] = textbook_ffn(out["o"], gains["ffn_norm"], W["gate"], W["up"], gains["ffn_sub_norm"], W["down"], act,
                              eps)
    return out


def _tiny_block(seed=3, T=2):
    # n_q == hidden, so attn_norm and attn_sub_norm have the same length and a swap of the
    # two would not fail on shapes alone.
    sh = workloads.BlockShape("tiny", hidden=256, n_q=256, n_kv=128, inter=384, act="relu2")
    d = workloads.block_inputs(sh, T=T, seed=seed)
    W = {nm: d["W_" + nm].numpy() for nm in sh.tensors()}
    packed = {nm: O.pack_i2s(W[nm]) for nm in sh.tensors()}
    gains = {k[2:]: v.numpy() for k, v in d.items() if k.startswith("g_")}
    xb = O.bf16_bits_to_f32(d["x"].view(torch.int16).numpy().view(np.uint16))
    ab = O.bf16_bits_to_f32(d["attn_out"].view(torch.int16).numpy().view(np.uint16))
    return sh, W, packed, gains, xb, ab


def test_decoder_block_matches_textbook(block_fn=None):
    """Each projection of the oracle's block against an fp64 textbook computation that takes
    its own gain and its own input ("Add optional RMSNorm support to BitNet quantization": a
    BitLinear normalises its own input; the per-block norms attn_norm, attn_sub_norm,
    ffn_norm, ffn_sub_norm of "More BitNet-like IQ1_S quantizations")."""
    block_fn = block_fn or O.decoder_block
    sh, W, packed, gains, xb, ab = _tiny_block()
    out = block_fn(xb, ab, gains, packed, sh.tensors(), "relu2", 1e-6, "f32")
    ref = textbook_block(xb, ab, gains, W, "relu2")
    for nm in ("q", "k", "v", "o", "ffn"):
        err = np.linalg.norm(out[nm] - ref[nm]) / np.linalg.norm(ref[nm])
        assert err <= 2e-3, f"{nm}: relative error {err}"


def _block_mutant(kind):
    """A copy of the oracle's decoder_block with one plausible routing mistake."""
    def block(x, attn_out, gains, packed, shape, act, eps, out_dtype="bf16"):
        g = dict(gains)
        if kind == "norms_swapped":
            g["attn_norm"], g["attn_sub_norm"] = gains["attn_sub_norm"], gains["attn_norm"]
        qkv_in = attn_out if kind == "qkv_from_attn_out" else x
        out = {}
        q, s, sq = O.rmsnorm_quant_act(qkv_in, g["attn_norm"], eps)
        for nm in ("q", "k", "v"):
            N, K = shape[nm]
            out[nm] = O.bitlinear(q, s, sq, packed[nm], N, K, out_dtype)
        N, K = shape["o"]
        out["o"] = O.bitlinear_from_x(attn_out, g["attn_sub_norm"], eps, packed["o"], N, K, out_dtype)
        I, H = shape["gate"]
        ffn_in = x if kind == "ffn_from_block_input" else out["o"]
        ffn_norm = g["ffn_sub_norm"][:H] if kind == "ffn_norms_swapped" else g["ffn_norm"]
        out["ffn"] = O.ffn_block(ffn_in, ffn_norm, packed["gate"], packed["up"], g["ffn_sub_norm"], packed["down"],
                                 H, I, act, eps, out_dtype)
        return out
    return block


@pytest.mark.parametrize("kind", ["norms_swapped", "qkv_from_attn_out", "ffn_from_block_input",
                                  "ffn_norms_swapped"])
def test_decoder_block_pin_catches_routing_mistakes(kind):
    with pytest.raises(AssertionError):
        test_decoder_block_matches_textbook(_block_mutant(kind))


def test_decoder_block_runs_and_chains():
    sh = workloads.BlockShape("tiny", hidden=256, n_q=256, n_kv=128, inter=384, act="relu2")
    d = workloads.block_inputs(sh, T=2, seed=3)
    packed = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in sh.tensors()}
    gains = {k[2:]: v.numpy() for k, v in d.items() if k.startswith("g_")}
    xb = O.bf16_bits_to_f32(d["x"].view(torch.int16).numpy().view(np.uint16))
    ab = O.bf16_bits_to_f32(d["attn_out"].view(torch.int16).numpy().view(np.uint16))
    out = O.decoder_block(xb, ab, gains, packed, sh.tensors(), "relu2", 1e-6, "bf16")
    assert out["q"].shape == (2, 256) and out["k"].shape == (2, 128) and out["ffn"].shape == (2, 256)
    ffn = O.ffn_block(out["o"], gains["ffn_norm"], packed["gate"], packed["up"], gains["ffn_sub_norm"],
                      packed["down"], 256, 384, "relu2", 1e-6, "bf16")
    assert np.array_equal(ffn, out["ffn"])


# ----------------------------------------------------------------------------- planted mistakes

def _sequential_interleave(codes):
    N, K = codes.shape
    c = codes.reshape(-1, 4).astype(np.uint8)  # byte i/4, field i%4
    return ((c[:, 0] << 6) | (c[:, 1] << 4) | (c[:, 2] << 2) | c[:, 3]).astype(np.uint8)


@pytest.mark.parametrize("mutant", ["sequential_layout", "codes_minus_one", "no_half_even", "half_away_from_zero",
                                    "mean_without_divide", "transposed_dot", "gate_up_swapped"])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    if mutant == "sequential_layout":
        monkeypatch.setattr(O, "interleave_i2s", _sequential_interleave)
        check = test_pack_handworked_block_golden
    elif mutant == "codes_minus_one":
        orig = O.ternary_codes
        monkeypatch.setattr(O, "ternary_codes", lambda W, b: (orig(W, b).astype(np.int16) - 1).astype(np.uint8) & 3)
        check = test_pack_handworked_block_golden
    elif mutant == "no_half_even":
        monkeypatch.setattr(O.np, "rint", lambda v: np.floor(np.asarray(v) + 0.5))
        check = test_quant_ties_round_half_even
    elif mutant == "half_away_from_zero":
        monkeypatch.setattr(O.np, "rint", lambda v: np.sign(v) * np.floor(np.abs(np.asarray(v)) + 0.5))
        check = test_ties_of_codes_and_activations_round_half_even
    elif mutant == "mean_without_divide":
        monkeypatch.setattr(O, "fixed_point_mean_f32",
                            lambda t: F32(math.ldexp(float(O.fixed_point_sum(t)[0]), -O.fixed_point_sum(t)[1])))
        check = lambda: test_mean_square_is_exact_mean_rounded(128, 0)
    elif mutant == "transposed_dot":
        orig_unpack = O.unpack_i2s
        def bad(packed, N, K):
            c, b = orig_unpack(packed, N, K)
            return c[:, ::-1].copy(), b
        monkeypatch.setattr(O, "unpack_i2s", bad)
        check = lambda: test_dot_bruteforce(2, 3, 128, 1)
    else:
        orig_ffn_act = O.ffn_act
        monkeypatch.setattr(O, "ffn_act", lambda g, u, act: orig_ffn_act(u, g, act))
        check = lambda: test_ffn_block_matches_textbook("relu2")
    with pytest.raises(AssertionError):
        check()


# ----------------------------------------------------------------------------- prescaled pack, validator

def _ternary_times_scale(N, K, scale, seed, density=0.7):
    rng = np.random.default_rng(seed)
    t = rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(N, K), p=[density / 2, 1 - density, density / 2])
    return t, (t.astype(F32) * F32(scale))


def test_prescaled_pack_recovers_scale_and_ternary_values():
    """quantize_i2_s's convention: inputs are ternary x scale and the scale is the first
    non-zero |w|; so the stored scale is that scale exactly and the codes are t + 1."""
    t, W = _ternary_times_scale(3, 256, 0.0374, 1)
    p = O.pack_i2s_prescaled(W)
    codes, beta = O.unpack_i2s(p, 3, 256)
    assert beta == F32(0.0374)
    assert np.array_equal(codes.astype(np.int16) - 1, t)
    # the same code bytes as the absmean pack (whose scale is smaller: scale x density)
    pa = O.pack_i2s(W)
    assert np.array_equal(p[:3 * 256 // 4], pa[:3 * 256 // 4])
    assert O.unpack_i2s(pa, 3, 256)[1] < beta


def test_prescaled_pack_first_nonzero_in_row_major_order():
    W = np.zeros((2, 128), dtype=F32)
    W[1, 5] = F32(0.25)      # later in row-major order
    W[0, 100] = F32(-0.7)    # first non-zero: row 0 comes first
    W[0, 120] = F32(0.7)
    p = O.pack_i2s_prescaled(W)
    codes, beta = O.unpack_i2s(p, 2, 128)
    assert beta == F32(0.7)
    assert codes[0, 100] == 0 and codes[0, 120] == 2 and codes[1, 5] == 1  # 0.25 / 0.7 rounds to 0
    z = O.pack_i2s_prescaled(np.zeros((1, 128), dtype=F32))
    zc, zb = O.unpack_i2s(z, 1, 128)
    assert zb == F32(1e-5) and np.all(zc == 1)


def test_validate_i2s_counts_planted_faults():
    W = workloads.latent_weight(4, 256, 3, "validate").numpy()
    p = O.pack_i2s(W)
    assert O.validate_i2s(p, 4, 256) == (0, 0, 0)
    bad = p.copy()
    bad[5] |= 0b11000000           # field 0 of byte 5 -> 3
    bad[77] |= 0b00001111          # fields 2 and 3 of byte 77 -> 3
    assert O.validate_i2s(bad, 4, 256) == (3, 0, 0)
    nb = 4 * 256 // 4
    tr = p.copy()
    tr[nb + 10] = 7                # a trailer byte after the scale
    tr[nb + 31] = 1
    assert O.validate_i2s(tr, 4, 256) == (0, 2, 0)
    for val in (np.nan, np.inf, -1.0, 0.0):
        sc = p.copy()
        sc[nb:nb + 4] = np.frombuffer(np.asarray([val], dtype="<f4").tobytes(), dtype=np.uint8)
        assert O.validate_i2s(sc, 4, 256) == (0, 0, 1), val


# ----------------------------------------------------------------------------- rotary embedding, attention

def test_rope_is_identity_at_position_zero_and_preserves_pair_norms():
    x = np.random.default_rng(1).standard_normal((3, 4, 128))
    assert np.array_equal(O.apply_rope(x, np.zeros(3), 10000.0), x)
    y = O.apply_rope(x, np.array([1, 17, 4095]), 10000.0)
    n_x = x[..., :64] ** 2 + x[..., 64:] ** 2
    n_y = y[..., :64] ** 2 + y[..., 64:] ** 2
    assert np.allclose(n_x, n_y, rtol=1e-13, atol=0)


def test_rope_equals_complex_rotation():
    """(x_i + j x_{i+d/2}) e^{j p theta^(-2i/d)}: the rotation written with complex numbers."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 2, 64))
    pos = np.array([0, 3, 100, 1000, 65535])
    for theta in (10000.0, 500000.0):
        z = x[..., :32] + 1j * x[..., 32:]
        i = np.arange(32)
        rot = np.exp(1j * pos[:, None, None] * np.power(theta, -2.0 * i / 64.0)[None, None, :])
        want = np.concatenate([(z * rot).real, (z * rot).imag], axis=-1)
        assert np.allclose(O.apply_rope(x, pos, theta), want, rtol=0, atol=1e-12)


def test_rope_dot_products_depend_on_relative_position_only():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((1, 1, 128)), rng.standard_normal((1, 1, 128))
    d0 = float(np.sum(O.apply_rope(q, np.array([7]), 1e4) * O.apply_rope(k, np.array([3]), 1e4)))
    for shift in (1, 50, 1000):
        d1 = float(np.sum(O.apply_rope(q, np.array([7 + shift]), 1e4) * O.apply_rope(k, np.array([3 + shift]), 1e4)))
        assert abs(d1 - d0) <= 1e-9 * (1 + abs(d0))


def _sdpa_reference(q, k, v, q_pos):
    """torch's scaled_dot_product_attention in fp64, with the key/value heads repeated for
    their query groups and an explicit causal mask."""
    T, Hq, d = q.shape
    L, Hkv, _ = k.shape
    kk = torch.from_numpy(k).double().repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)  # [Hq, L, d]
    vv = torch.from_numpy(v).double().repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
    qq = torch.from_numpy(q).double().permute(1, 0, 2)  # [Hq, T, d]
    mask = torch.from_numpy(np.arange(L)[None, :] <= np.asarray(q_pos)[:, None])  # [T, L]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("T,Hq,Hkv,L", [(1, 4, 1, 37), (3, 20, 5, 130), (16, 8, 2, 64)])
def test_attention_matches_torch_sdpa(T, Hq, Hkv, L, attn_fn=None):
    attn_fn = attn_fn or O.attention
    rng = np.random.default_rng(T + L)
    q, k, v = rng.standard_normal((T, Hq, 128)), rng.standard_normal((L, Hkv, 128)), rng.standard_normal((L, Hkv, 128))
    q_pos = np.arange(L - T, L)
    assert np.allclose(attn_fn(q, k, v, q_pos), _sdpa_reference(q, k, v, q_pos), rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(4)
    q, k, v = rng.standard_normal((1, 2, 128)), rng.standard_normal((5, 1, 128)), rng.standard_normal((5, 1, 128))
    # a query at position 0 sees only key 0: the output is v_0
    assert np.allclose(O.attention(q, k, v, np.array([0]))[0, :, :], np.repeat(v[0], 2, axis=0), rtol=0, atol=1e-15)
    # identical keys: uniform weights, the mean of the visible values
    kk = np.repeat(k[:1], 5, axis=0)
    assert np.allclose(O.attention(q, kk, v, np.array([4]))[0, 0], v[:, 0].mean(axis=0), rtol=1e-13, atol=1e-15)


def _attention_mutant(kind):
    def attn(q, k, v, q_pos):
        T, Hq, d = q.shape
        L, Hkv, _ = k.shape
        out = np.zeros((T, Hq, d))
        for t in range(T):
            n = L if kind == "not_causal" else int(q_pos[t]) + 1
            for h in range(Hq):
                kh = h % Hkv if kind == "heads_interleaved" else h // (Hq // Hkv)
                s = (k[:n, kh] @ q[t, h]) / (d if kind == "scale_by_d" else math.sqrt(d))
                w = np.exp(s - s.max())
                out[t, h] = (w / w.sum()) @ v[:n, kh]
        return out
    return attn


@pytest.mark.parametrize("kind", ["not_causal", "heads_interleaved", "scale_by_d"])
def test_attention_pin_catches_planted_mistakes(kind):
    with pytest.raises(AssertionError):
        test_attention_matches_torch_sdpa(3, 20, 5, 130, attn_fn=_attention_mutant(kind))


def test_rope_pin_catches_a_sign_flip(monkeypatch):
    orig = O.apply_rope
    monkeypatch.setattr(O, "apply_rope", lambda x, p, th: orig(x, -np.asarray(p, dtype=np.float64), th))
    with pytest.raises(AssertionError):
        test_rope_equals_complex_rotation()

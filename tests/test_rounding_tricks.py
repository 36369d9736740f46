"""Rounding steps the quantisation kernels use in place of conversion instructions, checked on
the CPU against their plain definitions (exact rationals, round half to even):

- a fixed-point term rint(v^2 2^e) as the bits of one fused multiply-add v (v 2^e) + 1.5 * 2^52
  (fp64), valid while the term is below 2^51, and the sum of such bits taken modulo 2^64 with
  the offset removed once;
- an int8 activation code as the low byte of the fp32 bits of clamp(p, -128, 127) + 1.5 * 2^23,
  and the sum of codes from the sum of those bits modulo 2^32."""
from fractions import Fraction

import numpy as np

MAGIC64 = 6755399441055744.0  # 1.5 * 2^52
OFF64 = 0x4338000000000000
MAGIC32 = np.float32(12582912.0)  # 1.5 * 2^23
OFF32 = 0x4B400000


def rint_half_even(x: Fraction) -> int:
    f = x.numerator // x.denominator
    r = x - f
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return f


def fma_term_bits(v: np.float32, e: int) -> int:
    """Bits of RN(v * (v * 2^e) + 1.5 * 2^52): the product v 2^e is exact (a power-of-two
    scaling in range), and float() of a Fraction rounds once, to nearest even."""
    d = Fraction(float(v))
    dp = d * Fraction(2) ** e
    r = float(d * dp + Fraction(MAGIC64))
    return int(np.array([r], dtype=np.float64).view(np.int64)[0])


def test_fixed_point_terms_by_one_rounding():
    rng = np.random.default_rng(5)
    for _ in range(3000):
        v = np.float32(rng.standard_normal() * 10.0 ** rng.uniform(-4, 4))
        # the grid of a row whose max is M >= |v| with n > 1024 terms: e = 62 - E(M) - ceil_log2(n)
        M = float(v) ** 2 * 2.0 ** rng.uniform(0, 30)
        E = int(np.frexp(M)[1])
        n = int(rng.integers(1025, 60000))
        e = 62 - E - int(np.ceil(np.log2(n)))
        exact = Fraction(float(v)) ** 2 * Fraction(2) ** e
        want = rint_half_even(exact)
        assert want < 2 ** 51
        assert fma_term_bits(v, e) - OFF64 == want


def test_term_sums_modulo_2_64():
    rng = np.random.default_rng(6)
    for _ in range(200):
        k = int(rng.integers(1, 29))
        terms = [int(t) for t in rng.integers(0, 2 ** 51, size=k)]
        bits = sum(OFF64 + t for t in terms) % 2 ** 64
        assert (bits - k * OFF64) % 2 ** 64 == sum(terms)


def code_of(p: np.float32) -> int:
    """The oracle's definition: clamp(rint(p), -128, 127), ties to even."""
    return int(np.clip(np.rint(np.float64(p)), -128, 127))


def test_code_byte_from_offset_bits():
    rng = np.random.default_rng(8)
    ps = np.concatenate([rng.uniform(-300, 300, 20000), np.arange(-260, 260) / 2.0]).astype(np.float32)
    c = np.minimum(np.maximum(ps, np.float32(-128)), np.float32(127))
    b = (c + MAGIC32).astype(np.float32).view(np.uint32).astype(np.int64)
    codes = np.array([code_of(p) for p in ps])
    assert np.array_equal(b - OFF32, codes)
    assert np.array_equal(b & 0xFF, codes & 0xFF)  # the stored byte
    total = int(b.sum()) % 2 ** 32
    assert ((total - len(ps) * OFF32) % 2 ** 32) == int(codes.sum()) % 2 ** 32


def test_fixed_point_term_ties():
    """v = (2a + 1) 2^-j on the grid e = 2j - 1: v^2 2^e = (2a + 1)^2 / 2 is a .5 tie, rounded
    to the even neighbour (a half-away rounding fails here)."""
    for a in range(0, 300, 7):
        for j in (0, 3, 10, 40):
            v = np.float32((2 * a + 1) * 2.0 ** -j)
            e = 2 * j - 1
            exact = Fraction(float(v)) ** 2 * Fraction(2) ** e
            assert exact.denominator == 2
            want = rint_half_even(exact)
            assert want % 2 == 0
            assert fma_term_bits(v, e) - OFF64 == want

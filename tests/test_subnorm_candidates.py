"""The decode engine's grid-wide ffn_sub_norm takes max |y| (y = fl(fl(h inv) g), fp32) from
candidates: in every CTA, the (h, g) pairs whose exact |h g| is within a relative 2^-20 of that
CTA's largest.  This rests on a rounding bound -- the element holding max |y| has an exact |h g|
within a relative 2^-22 of the row's largest -- checked here on the CPU with IEEE fp32 products
(numpy rounds each float32 multiply to nearest), on random rows and on rows built to sit on the
edge of a tie."""
import numpy as np

F = np.float32


def y_of(h, inv, g):
    return (h * F(inv)).astype(F) * g  # two fp32 roundings, as in the kernels


def check_row(h, g, inv):
    y = np.abs(y_of(h, inv, g)).astype(np.float64)
    p = np.abs(h.astype(np.float64) * g.astype(np.float64))  # exact: 24 x 24 bits
    ymax = y.max()
    if ymax < 1e-5:  # below the scale's clamp the choice of element does not matter
        return
    holders = np.nonzero(y == ymax)[0]
    assert np.all(p[holders] >= p.max() * (1.0 - 2.0 ** -22)), (p[holders], p.max())


def test_random_rows():
    rng = np.random.default_rng(7)
    for _ in range(300):
        n = int(rng.integers(2, 4000))
        h = (rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 3)).astype(F)
        g = rng.uniform(0.25, 4.0, n).astype(F)
        inv = F(10.0 ** rng.uniform(-3, 3))
        check_row(h, g, inv)


def test_near_ties():
    """Pairs whose exact products differ by a few ulps, so the roundings of y can reorder them."""
    rng = np.random.default_rng(11)
    for _ in range(2000):
        base = F(rng.uniform(1.0, 2.0))
        k = rng.integers(-8, 9, size=64)
        h = (base * (1.0 + k * 2.0 ** -23)).astype(F)
        g = (F(rng.uniform(0.5, 2.0)) * (1.0 + rng.integers(-8, 9, size=64) * 2.0 ** -23)).astype(F)
        inv = F(rng.uniform(0.5, 2.0)) * F(2.0) ** F(rng.integers(-20, 20))
        check_row(h, g, F(inv))


def test_candidate_set_holds_the_max():
    """Split rows over 'CTAs'; max |y| over each CTA's candidates (exact |h g| within 2^-20 of
    the CTA's largest) equals max |y| over the row."""
    rng = np.random.default_rng(3)
    for _ in range(300):
        n = int(rng.integers(64, 3000))
        h = (rng.standard_normal(n) * 3.0).astype(F)
        h[rng.integers(0, n, size=8)] = h[0]  # some repeated values
        g = rng.uniform(0.5, 2.0, n).astype(F)
        g[rng.integers(0, n, size=8)] = g[0]
        inv = F(rng.uniform(0.1, 10.0))
        y = np.abs(y_of(h, inv, g))
        p = np.abs(h.astype(np.float64) * g.astype(np.float64))
        best = F(0.0)
        for part in np.array_split(np.arange(n), int(rng.integers(1, 40))):
            if part.size == 0:
                continue
            pc = p[part].max()
            cand = part[p[part] >= pc - pc * 2.0 ** -20]
            best = max(best, y[cand].max())
        assert best == y.max()

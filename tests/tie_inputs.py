"""Inputs that land on exact rounding ties (x.5) of both quantisers, for the oracle pins and
the GPU parity tests: the pages fix round() only as "round"; the reading taken is round half
to even, and these inputs are where a kernel that rounds half away from zero would differ.
Plain data construction, no arithmetic of the method."""
from __future__ import annotations

import numpy as np

F32 = np.float32


def tie_activations():
    """Rows whose absmax is 127/64, so that s_x = 64 exactly (no norm) and every other entry
    (n + 1/2)/64 is an exact .5 tie of y * s_x; all values are exact in bf16."""
    halves = np.array([0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 10.5, 63.5, 100.5, 125.5], dtype=np.float64)
    rng = np.random.default_rng(0)
    x = np.zeros((3, 256), dtype=F32)
    for t in range(3):
        v = rng.choice(np.concatenate([halves, -halves]), size=256) / 64.0
        v[rng.integers(0, 256)] = 127.0 / 64.0 * (1 if t != 1 else -1)
        x[t] = v.astype(F32)
    return x


def tie_weights(N=8, K=256, seed=0):
    """Weights with mean|W| = 2**-6 exactly (so s_w = 64 and W * s_w is exact): half of each
    row at +-0.5 beta (a tie that rounds to 0) and half at +-1.5 beta (a tie that rounds to
    +-2, clamped to +-1)."""
    rng = np.random.default_rng(seed)
    W = np.zeros((N, K), dtype=F32)
    for n in range(N):
        mag = np.concatenate([np.full(K // 2, 0.5), np.full(K // 2, 1.5)]) * 2.0 ** -6
        W[n] = (rng.permutation(mag) * rng.choice([-1.0, 1.0], size=K)).astype(F32)
    return W

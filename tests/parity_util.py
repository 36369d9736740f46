"""Helpers of the GPU parity tests: feed the same seeded inputs to the CUDA path (through
the C ABI binding) and to the CPU oracle, and compare."""
from __future__ import annotations

import numpy as np
import torch

from oracle import bitnet_oracle as O

# Float tolerances (max relative error, elementwise): 1e-3 for fp32 output, 1e-2 for bf16.
TOL = {"f32": 1e-3, "bf16": 1e-2}


def bf16_to_np(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> exact fp32 numpy values (via the bit patterns)."""
    return O.bf16_bits_to_f32(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def act_to_np(x: torch.Tensor) -> np.ndarray:
    return bf16_to_np(x) if x.dtype == torch.bfloat16 else x.detach().cpu().numpy().astype(np.float32)


def out_to_np(x: torch.Tensor) -> np.ndarray:
    return act_to_np(x)


def max_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    zero = ref == 0
    if np.any(got[zero] != 0):
        return float("inf")
    if not np.any(~zero):
        return 0.0
    return float(np.max(np.abs(got[~zero] - ref[~zero]) / np.abs(ref[~zero])))


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str):
    err = max_rel_err(got, ref)
    assert err <= TOL[dtype], f"max rel err {err} > {TOL[dtype]}"
    return err


def oracle_rows(packed: np.ndarray, N: int, K: int, rows: np.ndarray) -> np.ndarray:
    """An I2_S tensor made of the given rows of an oracle-packed tensor (same trailer)."""
    rb = K // 4
    body = np.concatenate([packed[r * rb:(r + 1) * rb] for r in rows])
    return np.concatenate([body, packed[N * rb: N * rb + 32]])

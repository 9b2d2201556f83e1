"""Shared helpers for the tests: comparison metrics and host<->device moves.

The tolerances are the ones the parity bar fixes:
  * bf16 attention: max |O - O_ref| <= 2e-2 and relative L1 <= 5e-3
  * 8-bit attention: cosine similarity >= 0.999 and relative L1 <= 2e-2
  * first-block cache: relative error of rel <= 1e-5, identical decisions
"""
from __future__ import annotations

import numpy as np

BF16_MAX_ABS = 2e-2
BF16_REL_L1 = 5e-3
Q8_COSINE = 0.999
Q8_REL_L1 = 2e-2
FBC_REL_ERR = 1e-5


def rel_l1(out: np.ndarray, ref: np.ndarray) -> float:
    """sum |out - ref| / sum |ref| over all elements."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(out - ref).sum() / np.abs(ref).sum())


def max_abs(out: np.ndarray, ref: np.ndarray) -> float:
    return float(np.abs(np.asarray(out, dtype=np.float64) - np.asarray(ref, dtype=np.float64)).max())


def cosine(out: np.ndarray, ref: np.ndarray) -> float:
    a = np.asarray(out, dtype=np.float64).reshape(-1)
    b = np.asarray(ref, dtype=np.float64).reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def to_device_bf16(bits: np.ndarray, device="cuda"):
    """uint16 bf16 bit patterns -> a bf16 CUDA tensor with identical bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def from_device_bf16(t) -> np.ndarray:
    """bf16 tensor -> fp64 numpy array (exact widening)."""
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def assert_bf16_parity(out, ref, what=""):
    ma, rl = max_abs(out, ref), rel_l1(out, ref)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    assert ma <= BF16_MAX_ABS and rl <= BF16_REL_L1, f"{what}: max|dO|={ma:.3e} relL1={rl:.3e}"
    return ma, rl

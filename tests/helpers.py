"""Small host-side helpers for the tests (no step arithmetic lives here)."""
from __future__ import annotations

import numpy as np
import torch


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round a float array to bf16 (torch's conversion) and return the raw bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bits -> float64 through torch's own bf16 widening."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.double().numpy()


def as_f64(a: np.ndarray) -> np.ndarray:
    return bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def rand_tier(rng, B, Hkv, cap, D, dtype="f32", length=None, std=1.0):
    """K, V [B, Hkv, cap, D] and per-unit lengths (default: full)."""
    k = rng.standard_normal((B, Hkv, cap, D)).astype(np.float32) * std
    v = rng.standard_normal((B, Hkv, cap, D)).astype(np.float32)
    if dtype == "bf16":
        k, v = bf16_bits(k), bf16_bits(v)
    if length is None:
        length = np.full(B * Hkv, cap, np.int32)
    return k, v, np.asarray(length, np.int32)


def rand_q(rng, B, Hq, D, dtype="f32"):
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    return bf16_bits(q) if dtype == "bf16" else q


def order_desc(z: np.ndarray) -> np.ndarray:
    """Token order by score descending, lower index first on ties (numpy lexsort)."""
    n = len(z)
    zz = z.astype(np.float64) + 0.0  # -0 -> +0
    return np.lexsort((np.arange(n), -zz))

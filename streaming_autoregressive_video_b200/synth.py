"""Seeded synthetic inputs for the tests, the bench and the oracle checks.

This module draws numbers and nothing else: N(0,1) values from a seeded torch
CPU generator, optionally scaled, rounded once to the storage dtype.  It holds
no arithmetic of the attention method, so both the CUDA path and the CPU oracle
can be fed the very same bytes from it.
"""
from __future__ import annotations

import numpy as np
import torch


def seed_of(*parts: int) -> int:
    """Deterministic 63-bit seed from a tuple of small integers (FNV-1a)."""
    h = 0xCBF29CE484222325
    for p in parts:
        for b in int(p).to_bytes(8, "little", signed=True):
            h ^= b
            h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h & 0x7FFFFFFFFFFFFFFF


def normal(seed: int, shape, dtype: str = "bf16", scale: float = 1.0) -> np.ndarray:
    """N(0,1)*scale drawn on the CPU, returned in storage form.

    bf16 -> uint16 numpy array of bfloat16 bit patterns (round to nearest even);
    f32  -> float32 numpy array.
    """
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * float(scale)
    if dtype == "bf16":
        return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "f32":
        return x.numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


def normal_device(seed: int, shape, dtype: str, device, scale: float = 1.0) -> torch.Tensor:
    """Large inputs drawn directly on a CUDA device (bench sizes).

    The device generator is seeded; the exact bytes of any call that is checked
    against the oracle are copied back to the host from the tensor itself.
    """
    g = torch.Generator(device=device).manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if scale != 1.0:
        x.mul_(float(scale))
    return x.to(torch.bfloat16) if dtype == "bf16" else x


def ragged_fill(seed: int, rollouts: int, lo: int, hi: int) -> np.ndarray:
    """Per-rollout committed window frames, uniform on [lo, hi]."""
    rng = np.random.default_rng(int(seed))
    return rng.integers(lo, hi + 1, size=rollouts).astype(np.int32)

"""Seeded synthetic inputs for the hybrid attention core.

This module holds no arithmetic of the method: it only draws random numbers
with the distributions of the workload and rounds them to the storage type.
Both the CUDA path and the fp64 oracle are fed from it.

Recipe (per batch element b, its own PCG64 stream seeded ``seed * 1000 + b``):

* q, k, v ~ N(0, 1), [T, N, H, d]; q and k are L2-normalised over d per
  (token, head);
* beta = sigmoid(N(0, 1)) per (token, head); alpha = sigmoid(N(2, 0.5)) per
  (frame, head);
* gate_sm, gate_lin ~ N(0, 1), elementwise [T, N, H, d_v];
* text_k, text_v, text_beta drawn the same way for L text tokens.

In bf16 mode every bf16-stored tensor is rounded to bf16 (round to nearest
even) here, and the *rounded* values are what both paths see.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BF16_TENSORS = ("q", "k", "v", "gate_sm", "gate_lin", "text_k", "text_v")


@dataclass(frozen=True)
class Shape:
    B: int
    T: int
    N: int
    H: int
    d_k: int
    d_v: int
    L: int = 0


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest-even bf16, returned as uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _l2n(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def _sig(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _one_batch(rng: np.random.Generator, s: Shape) -> dict:
    f32 = np.float32
    T, N, H = s.T, s.N, s.H
    out = {
        "q": _l2n(rng.standard_normal((T, N, H, s.d_k), dtype=f32)),
        "k": _l2n(rng.standard_normal((T, N, H, s.d_k), dtype=f32)),
        "v": rng.standard_normal((T, N, H, s.d_v), dtype=f32),
        "beta": _sig(rng.standard_normal((T, N, H), dtype=f32)),
        "alpha": _sig(2.0 + 0.5 * rng.standard_normal((T, H), dtype=f32)),
        "gate_sm": rng.standard_normal((T, N, H, s.d_v), dtype=f32),
        "gate_lin": rng.standard_normal((T, N, H, s.d_v), dtype=f32),
    }
    if s.L > 0:
        out["text_k"] = _l2n(rng.standard_normal((s.L, H, s.d_k), dtype=f32))
        out["text_v"] = rng.standard_normal((s.L, H, s.d_v), dtype=f32)
        out["text_beta"] = _sig(rng.standard_normal((s.L, H), dtype=f32))
    return out


def make_inputs(shape: Shape, seed: int, dtype: str = "f32") -> dict:
    """Return a dict of float32 arrays (the values both paths see) with a
    leading batch axis.  For dtype="bf16" the bf16-stored tensors are already
    rounded, and their bit patterns are under key ``<name>_bits``."""
    parts = [_one_batch(np.random.Generator(np.random.PCG64(seed * 1000 + b)), shape)
             for b in range(shape.B)]
    inp = {key: np.stack([p[key] for p in parts]) for key in parts[0]}
    if dtype == "bf16":
        for key in BF16_TENSORS:
            if key in inp:
                bits = bf16_round(inp[key])
                inp[key + "_bits"] = bits
                inp[key] = bf16_to_f32(bits)
    elif dtype != "f32":
        raise ValueError(f"unknown dtype {dtype!r}")
    return inp

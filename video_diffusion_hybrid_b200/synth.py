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

``make_inputs`` draws on the host (NumPy PCG64) and suits the sizes the
oracle evaluates in full.  ``make_inputs_torch`` draws the same recipe with
torch's seeded generator directly on a device (its stream differs from
PCG64's), for the full-size workloads; ``head_slice`` then copies one
(batch, head) of those tensors back to the host for the oracle.
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
    """float32 -> nearest-even bf16, returned as uint16 bit patterns
    (finite inputs; the carry cannot overflow 32 bits below the NaN range)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
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


def make_inputs_torch(shape: Shape, seed: int, dtype: str = "bf16", device="cuda") -> dict:
    """The same recipe drawn with a seeded ``torch.Generator`` on `device`.
    Returns torch tensors in their storage types (bf16-stored tensors already
    rounded; beta/alpha/text_beta float32), with a leading batch axis."""
    import torch
    st = torch.bfloat16 if dtype == "bf16" else torch.float32
    T, N, H = shape.T, shape.N, shape.H
    parts = []
    for b in range(shape.B):
        g = torch.Generator(device=device)
        g.manual_seed(seed * 1000 + b)

        def rn(*sz):
            return torch.randn(*sz, generator=g, device=device, dtype=torch.float32)

        def l2n(x):
            return x / x.double().norm(dim=-1, keepdim=True).clamp_min(1e-30).float()

        p = {
            "q": l2n(rn(T, N, H, shape.d_k)).to(st),
            "k": l2n(rn(T, N, H, shape.d_k)).to(st),
            "v": rn(T, N, H, shape.d_v).to(st),
            "beta": torch.sigmoid(rn(T, N, H)),
            "alpha": torch.sigmoid(2.0 + 0.5 * rn(T, H)),
            "gate_sm": rn(T, N, H, shape.d_v).to(st),
            "gate_lin": rn(T, N, H, shape.d_v).to(st),
        }
        if shape.L > 0:
            p["text_k"] = l2n(rn(shape.L, H, shape.d_k)).to(st)
            p["text_v"] = rn(shape.L, H, shape.d_v).to(st)
            p["text_beta"] = torch.sigmoid(rn(shape.L, H))
        parts.append(p)
    return {k: torch.stack([p[k] for p in parts]).contiguous() for k in parts[0]}


def head_slice(t: dict, b: int, h: int) -> dict:
    """One (batch, head) of device inputs as float32 NumPy arrays with unit
    batch and head axes, for the oracle."""
    out = {}
    for k, x in t.items():
        if k in ("init_state",):
            y = x[b:b + 1, h:h + 1]
        elif k == "rms_weight":
            y = x[h:h + 1]
        elif x.dim() >= 3:
            y = x[b:b + 1, :, :, h:h + 1] if x.dim() >= 4 and k not in ("text_k", "text_v") else \
                x[b:b + 1, :, h:h + 1]
        else:
            y = x[b:b + 1, :, h:h + 1]
        out[k] = y.float().cpu().numpy()
    return out

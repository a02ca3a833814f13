"""Gradients of the two branches of the hybrid core: the linear (Video Delta
Attention) branch and, at the end of this file, the windowed softmax branch.

TEST INFRASTRUCTURE ONLY, like ``vdn_oracle``: only the test suite may import
it.  The pages describe the forward pass only; the gradient of that forward is
its plain definition.  Here the linear branch is written once more in float64
torch ops, step for step as ``vdn_oracle`` defines it (joint frame write
S_t = (alpha_t S + B_t)(I + A_t)^-1, both scans from their start states, the
read of the summed states, RMSNorm and the sigmoid gate: [P1] 三, 四; [P4]
closed form), and torch's reverse-mode autograd is the library step that
differentiates it.  The text state (and init_state) is held constant:
gradients reach the video tokens' q, k, v, beta, the decay alpha, the gate
logits, the RMSNorm weight and, when it is given, the streaming forward start
state fwd_init (the state carried in from the previous segment).

Pinned in the tests by (a) its forward equal to ``vdn_oracle``'s linear slot
and (b) central finite differences of ``vdn_oracle``'s numpy forward along
random directions.
"""
from __future__ import annotations

import numpy as np
import torch

from . import vdn_oracle as O

GRAD_INPUTS = ("q", "k", "v", "beta", "alpha", "gate_lin", "rms_weight", "fwd_init")


def start_states(inp: dict, cfg: O.Cfg, b: int, h: int):
    """(forward start, backward start) of one (batch, head): both half the
    text state, the forward one fwd_init when given (as ``head_states``)."""
    if cfg.L > 0 and inp.get("text_k") is not None:
        Sx = O.text_state(inp["text_k"][b, :, h], inp["text_v"][b, :, h], inp["text_beta"][b, :, h],
                          cfg.d_v, cfg.d_k)
    elif inp.get("init_state") is not None:
        Sx = np.asarray(inp["init_state"][b, h], np.float64)
    else:
        Sx = np.zeros((cfg.d_v, cfg.d_k))
    S0 = 0.5 * Sx
    F0 = np.asarray(inp["fwd_init"][b, h], np.float64) if inp.get("fwd_init") is not None else S0
    return F0, S0


def linear_branch(x: dict, cfg: O.Cfg, starts) -> torch.Tensor:
    """y_lin [B, T, N, H, d_v] from the float64 tensors x (q, k, v, beta,
    alpha, gate_lin, rms_weight or None, fwd_init or None); starts[(b, h)] =
    (F0, S0), F0 replaced by x["fwd_init"][b, h] when that is given."""
    B, T, H = cfg.B, cfg.T, cfg.H
    anc = set(O.anchor_frames(T, cfg.anchors))
    eye = torch.eye(cfg.d_k, dtype=torch.float64)
    out = []
    for b in range(B):
        heads = []
        for h in range(H):
            F0, S0 = (torch.from_numpy(s) for s in starts[(b, h)])
            if x.get("fwd_init") is not None:
                F0 = x["fwd_init"][b, h]

            def write(S, t):
                kt, vt, bt = x["k"][b, t, :, h], x["v"][b, t, :, h], x["beta"][b, t, :, h]
                A = (bt[:, None] * kt).T @ kt
                Bw = (bt[:, None] * vt).T @ kt
                return torch.linalg.solve(eye + A, (x["alpha"][b, t, h] * S + Bw).T).T

            F = [F0]
            for t in range(T):
                F.append(F[t] if t in anc else write(F[t], t))
            G = [None] * (T + 1)
            G[T] = S0
            for t in range(T - 1, -1, -1):
                G[t] = G[t + 1] if t in anc else write(G[t + 1], t)
            frames = []
            for t in range(T):
                if t in anc and cfg.anchors:
                    R = F[0] + G[T]
                else:
                    lo, hi = O.window_frames(t, T, cfg.chunk)
                    R = F[lo] + G[hi]
                o = x["q"][b, t, :, h] @ R.T
                n = o / torch.sqrt(torch.mean(o * o, dim=-1, keepdim=True) + cfg.rms_eps)
                if x.get("rms_weight") is not None:
                    n = n * x["rms_weight"][h]
                frames.append(torch.sigmoid(x["gate_lin"][b, t, :, h]) * n)
            heads.append(torch.stack(frames))          # [T, N, d_v]
        out.append(torch.stack(heads, dim=2))           # [T, N, H, d_v]
    return torch.stack(out)


def linear_branch_grads(inp: dict, cfg: O.Cfg, dy: np.ndarray) -> dict:
    """d<y_lin, dy> / d input for every input of GRAD_INPUTS present in inp
    (numpy float64 arrays in the inputs' shapes)."""
    starts = {(b, h): start_states(inp, cfg, b, h) for b in range(cfg.B) for h in range(cfg.H)}
    x = {}
    for name in GRAD_INPUTS:
        if inp.get(name) is not None:
            x[name] = torch.tensor(np.asarray(inp[name], np.float64), requires_grad=True)
    y = linear_branch(x, cfg, starts)
    (y * torch.from_numpy(np.asarray(dy, np.float64))).sum().backward()
    # an input the output does not reach (at T <= 10 every query reads the
    # start states only) has gradient zero
    return {name: (t.grad.numpy() if t.grad is not None else np.zeros(t.shape)) for name, t in x.items()}


def linear_branch_forward(inp: dict, cfg: O.Cfg) -> np.ndarray:
    """The same forward without gradients, as numpy."""
    starts = {(b, h): start_states(inp, cfg, b, h) for b in range(cfg.B) for h in range(cfg.H)}
    x = {n: torch.from_numpy(np.asarray(inp[n], np.float64)) for n in GRAD_INPUTS if inp.get(n) is not None}
    with torch.no_grad():
        return linear_branch(x, cfg, starts).numpy()


# ---------------------------------------------------------------------------
# The softmax branch: y_sm = sigmoid(g_sm) * softmax(s q K^T over the allowed
# keys) V, the allowed keys being the query chunk and its two neighbours plus
# the anchor frames, and every key for an anchor query frame ([P1] 二; [P4]
# and [P5], the windowed softmax with first/last-frame anchors).
# ---------------------------------------------------------------------------
SM_INPUTS = ("q", "k", "v", "gate_sm")


def _sm_frame(x: dict, cfg: O.Cfg, b: int, h: int, t: int, keys: np.ndarray) -> torch.Tensor:
    """y_sm of query frame t of (b, h) over the key frames `keys` (in order)."""
    N = cfg.N
    K = x["k"][b, keys, :, h].reshape(len(keys) * N, -1)
    V = x["v"][b, keys, :, h].reshape(len(keys) * N, -1)
    P = torch.softmax(cfg.scale * (x["q"][b, t, :, h] @ K.T), dim=-1)
    return torch.sigmoid(x["gate_sm"][b, t, :, h]) * (P @ V)


def softmax_branch(x: dict, cfg: O.Cfg) -> torch.Tensor:
    """y_sm [B, T, N, H, d_v]: every query frame over the key frames the
    frame mask allows it."""
    allowed = O.frame_mask(cfg.T, cfg.chunk, cfg.anchors)
    out = []
    for b in range(cfg.B):
        heads = []
        for h in range(cfg.H):
            heads.append(torch.stack([_sm_frame(x, cfg, b, h, t, np.flatnonzero(allowed[t]))
                                      for t in range(cfg.T)]))
        out.append(torch.stack(heads, dim=2))
    return torch.stack(out)


def _sm_leaves(inp: dict) -> dict:
    return {n: torch.tensor(np.asarray(inp[n], np.float64), requires_grad=True) for n in SM_INPUTS}


def softmax_branch_grads(inp: dict, cfg: O.Cfg, dy: np.ndarray) -> dict:
    """d<y_sm, dy> / d input for q, k, v, gate_sm (numpy float64)."""
    x = _sm_leaves(inp)
    y = softmax_branch(x, cfg)
    (y * torch.from_numpy(np.asarray(dy, np.float64))).sum().backward()
    return {n: t.grad.numpy() for n, t in x.items()}


def softmax_branch_grads_frames(inp: dict, cfg: O.Cfg, dy: np.ndarray, b: int, h: int, frames) -> dict:
    """The gradients of sum over the query frames `frames` of <y_sm(b, h, t),
    dy[b, t, :, h]> for one (b, h), one query frame at a time (so that at full
    size only one frame's score matrix is held).  With `frames` = every query
    frame that sees key frame f, the rows of k and v of frame f are complete;
    the rows of q and gate_sm of those query frames always are."""
    allowed = O.frame_mask(cfg.T, cfg.chunk, cfg.anchors)
    x = _sm_leaves(inp)
    for t in frames:
        y = _sm_frame(x, cfg, b, h, t, np.flatnonzero(allowed[t]))
        (y * torch.from_numpy(np.asarray(dy[b, t, :, h], np.float64))).sum().backward()
    return {n: (t.grad.numpy() if t.grad is not None else np.zeros(t.shape)) for n, t in x.items()}

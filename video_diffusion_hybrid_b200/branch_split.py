"""The two branches of the hybrid core on separate GPU groups.

The deepmagic post (section 實測數據) and the aimodeling news ("The speedup
ledger and a three-stage recipe") report that on 8 B200s the profiling-driven
split of the two branches over separate GPUs, 5 for the softmax branch and 3
for Video Delta Attention, is 13.3 % below the plain Ulysses layout (1.405 s
against 1.62 s per step).  The pages give no further detail; the reading
taken here: each group splits the heads among its ranks as evenly as possible
(24 heads: 5, 5, 5, 5, 4 on the softmax ranks and 8, 8, 8 on the VDA ranks), so
each rank runs one branch of the core on whole sequences of its heads.

Between layers every rank holds a shard of the token sequence (as in Ulysses,
S = T N tokens of a batch element in frame-major order, rank p holding
[p S/P, (p+1) S/P)).  One uneven all-to-all per input sends each shard's
columns of a rank's heads to that rank when its branch reads the input (q, k
and v go to both groups, the gates and beta to their own branch); the small
per-head inputs are replicated and sliced.  The core runs its branch's
stages only, and a second all-to-all brings each branch's output slot back to
the sequence shards, where y[..., 0, :] comes from the softmax ranks and
y[..., 1, :] from the VDA ranks.

The exchange is ``torch.distributed.all_to_all_single`` with split sizes
(NCCL on GPUs, gloo on the host); every step of the core runs in
``libvdn_hybrid.so``.
"""
from __future__ import annotations

from dataclasses import replace

import torch
import torch.distributed as dist

from . import _lib as L
from .ulysses import REPLICATED_HEAD_AXIS, _world, to_device

# per-token inputs [B, S/P, H, ...] and the branches that read them
READ_BY = {"q": ("sm", "lin"), "k": ("sm", "lin"), "v": ("sm", "lin"), "gate_sm": ("sm",),
           "beta": ("lin",), "gate_lin": ("lin",)}
STAGES = {"sm": L.STAGE_SOFTMAX, "lin": L.STAGE_TEXT | L.STAGE_SOLVE | L.STAGE_SCAN | L.STAGE_READ}


def even_split(H: int, P: int) -> list:
    """(first head, heads) of each of P ranks, as even as possible."""
    base, extra = divmod(H, P)
    out, h0 = [], 0
    for r in range(P):
        n = base + (1 if r < extra else 0)
        out.append((h0, n))
        h0 += n
    return out


class Layout:
    """Who computes what: ranks [0, n_softmax) the softmax branch, the rest
    the linear branch, each group's heads split evenly."""

    def __init__(self, H: int, world: int, n_softmax: int):
        if not 0 < n_softmax < world:
            raise ValueError(f"{n_softmax} softmax ranks of {world}: both groups need a rank")
        if H < max(n_softmax, world - n_softmax):
            raise ValueError(f"{H} heads cannot give every rank of a group a head")
        self.H, self.world, self.ns = H, world, n_softmax
        self.heads = even_split(H, n_softmax) + even_split(H, world - n_softmax)

    def branch(self, r: int) -> str:
        return "sm" if r < self.ns else "lin"


def _exchange(chunks: list, out_shapes: list, group) -> list:
    """Uneven all-to-all: chunks[j] (any shape) to rank j; returns what each
    rank i sent here, reshaped to out_shapes[i]."""
    send = torch.cat([c.reshape(-1) for c in chunks])
    recv = torch.empty(sum(int(torch.Size(s).numel()) for s in out_shapes), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(recv, send, [int(torch.Size(s).numel()) for s in out_shapes],
                           [c.numel() for c in chunks], group=group)
    out, o = [], 0
    for s in out_shapes:
        n = int(torch.Size(s).numel())
        out.append(recv[o:o + n].view(s))
        o += n
    return out


def split_inputs(t_local: dict, T: int, N: int, lay: Layout, group=None) -> dict:
    """This rank's branch inputs: whole sequences of its heads [B, T, N, h,
    ...] for the per-token inputs its branch reads, the replicated ones
    sliced to its heads."""
    P, rank = _world(group)
    if P != lay.world or (T * N) % P:
        raise ValueError(f"{T * N} tokens over {P} ranks with a layout for {lay.world}")
    me, (h0, hn) = lay.branch(rank), lay.heads[rank]
    out = {}
    for name, x in t_local.items():
        if x is None:
            continue
        if name in READ_BY:
            need = [lay.branch(j) in READ_BY[name] for j in range(P)]
            chunks = [x.narrow(2, lay.heads[j][0], lay.heads[j][1]) if need[j] else x.narrow(2, 0, 0)
                      for j in range(P)]
            if me in READ_BY[name]:
                shape = (x.shape[0], x.shape[1], hn) + tuple(x.shape[3:])
                parts = _exchange(chunks, [shape] * P, group)
                out[name] = torch.cat(parts, dim=1).unflatten(1, (T, N))
            else:
                empty = (x.shape[0], 0) + tuple(x.shape[2:])
                _exchange(chunks, [empty] * P, group)
        elif name in REPLICATED_HEAD_AXIS:
            out[name] = x.narrow(REPLICATED_HEAD_AXIS[name], h0, hn).contiguous()
        else:
            raise KeyError(f"unknown input {name!r}")
    return out


def merge_outputs(y_branch: torch.Tensor, lay: Layout, group=None) -> torch.Tensor:
    """This rank's branch output for its heads, [B, T, N, h, 2, d] (only its
    branch's slot is used), back to this rank's shard of the sequence for
    every head and both slots, [B, S/P, H, 2, d]."""
    P, rank = _world(group)
    B, T, N, hn, _, d = y_branch.shape
    S = T * N
    sl = S // P
    slot = 0 if lay.branch(rank) == "sm" else 1
    mine = y_branch.flatten(1, 2)[:, :, :, slot]  # [B, S, h, d]
    chunks = [mine.narrow(1, j * sl, sl) for j in range(P)]
    parts = _exchange(chunks, [(B, sl, lay.heads[i][1], d) for i in range(P)], group)
    y = torch.empty((B, sl, lay.H, 2, d), dtype=y_branch.dtype, device=y_branch.device)
    for i, part in enumerate(parts):
        h0, hn_i = lay.heads[i]
        y[:, :, h0:h0 + hn_i, 0 if lay.branch(i) == "sm" else 1] = part
    return y


class BranchSplitHybridAttention:
    """The hybrid attention core with its two branches on separate ranks (one
    per GPU): sequence-sharded inputs in, the sequence-sharded output with
    both slots out.  `cfg` is the whole problem's configuration (out_mode 0);
    T N must divide by the world size."""

    def __init__(self, cfg: L.HybridCfg, n_softmax: int, group=None, device="cuda"):
        from .api import HybridAttention
        P, rank = _world(group)
        if cfg.out_mode != 0:
            raise ValueError("the branch split returns the two slots apart (out_mode 0)")
        self.lay = Layout(cfg.H, P, n_softmax)
        self.cfg, self.group, self.branch = cfg, group, self.lay.branch(rank)
        self.local_cfg = replace(cfg, H=self.lay.heads[rank][1])
        self.core = HybridAttention(self.local_cfg, device)

    def __call__(self, t_local: dict, stream=None) -> torch.Tensor:
        # the exchange runs where the inputs are (GPU with NCCL, host copies
        # with gloo); the core runs on its device
        where = t_local["q"].device
        t = to_device(split_inputs(t_local, self.cfg.T, self.cfg.N, self.lay, self.group), self.core.device)
        # the other branch's per-token inputs are not sent here; the core's
        # argument checks want every pointer, so they alias one that is
        # (their stages do not run)
        for name in ("gate_sm", "gate_lin"):
            t.setdefault(name, t["q"])
        t.setdefault("beta", torch.empty(t["q"].shape[:4], dtype=torch.float32, device=t["q"].device))
        self._last = t  # the inputs of the last call, for device_status
        y = self.core(t, stages=STAGES[self.branch], stream=stream)
        return merge_outputs(y.to(where), self.lay, self.group)

    def device_status(self) -> tuple:
        """(status, kernel tag) of this rank's last core call (synchronises)."""
        return L.vdn_hybrid_device_status(self.local_cfg, self.core.args(self._last))

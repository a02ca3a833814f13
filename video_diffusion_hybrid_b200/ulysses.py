"""Head-sharded sequence parallelism (Ulysses) around the hybrid attention core.

The pages deploy the model on 8 B200s with Ulysses sequence parallelism, the
attention heads split over the GPUs (deepmagic post, section 實測數據: 1.62 s
per NFE on 8 B200s; aimodeling news, "The speedup ledger and a three-stage
recipe": the per-step latency drops from 6.46 s to 1.62 s).  Between
attention layers the activations are sharded along the sequence: with the
S = T N video tokens of a batch element in frame-major order, rank p holds
tokens [p S/P, (p+1) S/P) (a shard may end inside a frame).  The core needs
every token of a head, and its batch-heads are independent, so one
all-to-all turns the sequence shards into head shards (rank p then holds all
tokens of heads [p H/P, (p+1) H/P)), the core runs unchanged on its H/P
heads, and a second all-to-all turns the output back into sequence shards.
The per-frame decay alpha, the text tokens, the RMSNorm weight and per-head
states are small and replicated; each rank takes its heads' slice.

The exchange is ``torch.distributed.all_to_all_single`` (NCCL over
NVLink / NVSwitch on GPUs, gloo on the host); every byte of the core still runs
in ``libvdn_hybrid.so``.
"""
from __future__ import annotations

from dataclasses import replace

import torch
import torch.distributed as dist

from . import _lib as L

# per-token inputs, sequence-sharded as [B, S/P, H, ...] (head axis 2)
PER_TOKEN = ("q", "k", "v", "beta", "gate_sm", "gate_lin")
# replicated inputs: the head axis of each, sliced to the rank's heads
REPLICATED_HEAD_AXIS = {"alpha": 2, "text_k": 2, "text_v": 2, "text_beta": 2, "init_state": 1, "fwd_init": 1,
                        "rms_weight": 0}


def _world(group) -> tuple[int, int]:
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_head(x: torch.Tensor, group=None, head_axis: int = 2) -> torch.Tensor:
    """This rank's shard of the sequence (axis 1) for every head,
    [B, S/P, ..., H, ...], to the whole sequence for this rank's heads,
    [B, S, ..., H/P, ...]."""
    P, _ = _world(group)
    if P == 1:
        return x
    H = x.shape[head_axis]
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    # head group g goes to rank g: put the group index first
    xs = x.unflatten(head_axis, (P, H // P)).movedim(head_axis, 0).contiguous()
    out = torch.empty_like(xs)
    dist.all_to_all_single(out, xs, group=group)  # out[p]: rank p's shard of this rank's heads
    return out.movedim(0, 1).flatten(1, 2)


def head_to_seq(y: torch.Tensor, group=None, head_axis: int = 2) -> torch.Tensor:
    """The inverse of seq_to_head: the whole sequence for this rank's heads,
    [B, S, ..., H/P, ...], to this rank's shard for every head."""
    P, _ = _world(group)
    if P == 1:
        return y
    S = y.shape[1]
    if S % P:
        raise ValueError(f"a sequence of {S} does not split over {P} ranks")
    # sequence block p goes to rank p
    ys = y.unflatten(1, (P, S // P)).movedim(1, 0).contiguous()
    out = torch.empty_like(ys)
    dist.all_to_all_single(out, ys, group=group)  # out[p]: rank p's heads of this rank's shard
    return out.movedim(0, head_axis).flatten(head_axis, head_axis + 1)


def shard_inputs(t_local: dict, T: int, N: int, H: int, group=None) -> dict:
    """The core's inputs for this rank's heads, per-token ones [B, T, N, H/P,
    ...]: the sequence-sharded tensors [B, T N / P, H, ...] through the
    all-to-all, the replicated ones sliced."""
    P, rank = _world(group)
    if H % P or (T * N) % P:
        raise ValueError(f"{H} heads and {T * N} tokens must split over {P} ranks")
    hl = H // P
    out = {}
    for name, x in t_local.items():
        if x is None:
            continue
        if name in PER_TOKEN:
            out[name] = seq_to_head(x, group, 2).unflatten(1, (T, N))
        elif name in REPLICATED_HEAD_AXIS:
            out[name] = x.narrow(REPLICATED_HEAD_AXIS[name], rank * hl, hl).contiguous()
        else:
            raise KeyError(f"unknown input {name!r}")
    return out


def gather_output(y: torch.Tensor, group=None) -> torch.Tensor:
    """The core's output for this rank's heads, [B, T, N, H/P, ...], back to
    this rank's shard of the sequence for every head, [B, T N / P, H, ...]."""
    return head_to_seq(y.flatten(1, 2), group, 2)


def to_device(t: dict, device) -> dict:
    """The tensors of t on `device` (no copy for those already there)."""
    return {k: v.to(device, non_blocking=False) for k, v in t.items()}


class UlyssesHybridAttention:
    """The hybrid attention core over P ranks (one per GPU): sequence-sharded
    inputs in, sequence-sharded output out, heads split over the ranks inside.
    `cfg` is the whole problem's configuration; T N and H must divide by P."""

    def __init__(self, cfg: L.HybridCfg, group=None, device="cuda"):
        from .api import HybridAttention
        P, _ = _world(group)
        if cfg.H % P or (cfg.T * cfg.N) % P:
            raise ValueError(f"T N = {cfg.T * cfg.N} and H = {cfg.H} must divide by {P} ranks")
        self.cfg, self.group = cfg, group
        self.local_cfg = replace(cfg, H=cfg.H // P)
        self.core = HybridAttention(self.local_cfg, device)

    def __call__(self, t_local: dict, stream=None) -> torch.Tensor:
        # the exchange runs where the inputs are: on the GPU with NCCL, or on
        # host copies with a host backend (gloo), the core on the GPU either way
        where = t_local["q"].device
        t = to_device(shard_inputs(t_local, self.cfg.T, self.cfg.N, self.cfg.H, self.group), self.core.device)
        self._last = t  # the head-sharded inputs of the last call, for device_status
        return gather_output(self.core(t, stream=stream).to(where), self.group)

    def device_status(self) -> tuple:
        """(status, kernel tag) of this rank's last core call (synchronises)."""
        return L.vdn_hybrid_device_status(self.local_cfg, self.core.args(self._last))

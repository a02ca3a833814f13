"""Torch-facing helpers over the C ABI: device placement of the inputs and a
small callable that owns nothing but a workspace and an output buffer.

Every byte of compute runs in ``libvdn_hybrid.so``; torch provides device
memory and the current stream.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L
from .synth import Shape

TENSOR_NAMES = ("q", "k", "v", "beta", "alpha", "gate_sm", "gate_lin", "text_k", "text_v", "text_beta",
                "init_state", "rms_weight", "fwd_init")


def cfg_for(shape: Shape, dtype: str, **kw) -> L.HybridCfg:
    return L.HybridCfg(B=shape.B, T=shape.T, N=shape.N, H=shape.H, d_k=shape.d_k, d_v=shape.d_v, L=shape.L,
                       dtype=L.VDN_BF16 if dtype == "bf16" else L.VDN_F32, **kw)


def to_torch(inp: dict, dtype: str, device="cuda", pin: bool = False) -> dict:
    """Move the synthetic inputs to `device` in their storage types (bf16
    tensors from their exact bit patterns).  With device="cpu" and pin=True
    the result lives in pinned host memory."""
    out = {}
    for name in TENSOR_NAMES:
        if name not in inp:
            continue
        if dtype == "bf16" and name + "_bits" in inp:
            t = torch.from_numpy(np.ascontiguousarray(inp[name + "_bits"]).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(inp[name], dtype=np.float32))
        if pin:
            t = t.pin_memory()
        out[name] = t.to(device) if device != "cpu" else t
    return out


def output_shape(cfg: L.HybridCfg) -> tuple:
    base = (cfg.B, cfg.T, cfg.N, cfg.H)
    return base + ((2, cfg.d_v) if cfg.out_mode == 0 else (cfg.d_v,))


class HybridAttention:
    """Calls ``vdn_hybrid_attn_fwd`` on torch tensors.  Workspace and output
    are allocated once (by torch) and reused."""

    def __init__(self, cfg: L.HybridCfg, device="cuda", keep_lse: bool = False):
        self.cfg = cfg
        self.ws_bytes = L.vdn_hybrid_attn_workspace_size(cfg)
        if self.ws_bytes == 0:
            raise L.VdnError(L.VDN_ERR_INVALID_ARG, "vdn_hybrid_attn_workspace_size")
        self.device = torch.device(device)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        tdt = torch.bfloat16 if cfg.y_dtype == L.VDN_BF16 else torch.float32
        self.y = torch.empty(output_shape(cfg), dtype=tdt, device=self.device)
        # the forward's softmax log-sum-exp per query row, which the softmax
        # backward then takes in place of recomputing the row statistics
        self.sm_lse = (torch.empty((cfg.B, cfg.T, cfg.N, cfg.H), dtype=torch.float32, device=self.device)
                       if keep_lse else None)

    def args(self, t: dict) -> L.VdnArgs:
        return L.make_args(t["q"], t["k"], t["v"], t["beta"], t["alpha"], t["gate_sm"], t["gate_lin"], self.y,
                           self.workspace, self.ws_bytes, text_k=t.get("text_k"), text_v=t.get("text_v"),
                           text_beta=t.get("text_beta"), init_state=t.get("init_state"),
                           rms_weight=t.get("rms_weight"), fwd_init=t.get("fwd_init"), sm_lse=self.sm_lse)

    def __call__(self, t: dict, stages: int = L.STAGE_ALL, stream=None) -> torch.Tensor:
        a = self.args(t)
        if stages == L.STAGE_ALL:
            L.vdn_hybrid_attn_fwd(self.cfg, a, stream)
        else:
            L.vdn_hybrid_attn_fwd_stages(self.cfg, a, stages, stream)
        return self.y

    def linear_backward(self, t: dict, dy: torch.Tensor, want_rms: bool = False, want_fwd_init: bool = False,
                        stream=None) -> dict:
        """Gradients through the linear branch after a forward call on the same
        inputs `t` (the forward's workspace is read): dy has y's shape and
        dtype.  Returns float32 tensors dq, dk, dv, dbeta, dalpha, dgate_lin
        (and drms_weight, dfwd_init when asked)."""
        c = self.cfg
        if getattr(self, "bwd_workspace", None) is None:
            nb = L.vdn_hybrid_lin_bwd_workspace_size(c)
            if nb == 0:
                raise L.VdnError(L.VDN_ERR_UNSUPPORTED, "vdn_hybrid_lin_bwd_workspace_size")
            self.bwd_workspace = torch.empty(nb, dtype=torch.uint8, device=self.device)
        f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=self.device)
        tok = (c.B, c.T, c.N, c.H)
        g = {"dq": f(*tok, c.d_k), "dk": f(*tok, c.d_k), "dv": f(*tok, c.d_v), "dbeta": f(*tok),
             "dalpha": f(c.B, c.T, c.H), "dgate_lin": f(*tok, c.d_v)}
        if want_rms:
            g["drms_weight"] = f(c.H, c.d_v)
        if want_fwd_init:
            g["dfwd_init"] = f(c.B, c.H, c.d_v, c.d_k)
        lg = L.make_lin_grads(dy, g["dq"], g["dk"], g["dv"], g["dbeta"], g["dalpha"], g["dgate_lin"],
                              self.bwd_workspace, drms_weight=g.get("drms_weight"), dfwd_init=g.get("dfwd_init"))
        L.vdn_hybrid_lin_bwd(c, self.args(t), lg, stream)
        return g

    def softmax_backward(self, t: dict, dy: torch.Tensor, stream=None) -> dict:
        """Gradients through the windowed softmax branch: float32 tensors dq,
        dk, dv, dgate_sm.  With keep_lse, the forward's log-sum-exp (kept by
        the last forward call on the same inputs) replaces the recomputed row
        statistics."""
        c = self.cfg
        if getattr(self, "sm_workspace", None) is None:
            nb = L.vdn_hybrid_sm_bwd_workspace_size(c)
            if nb == 0:
                raise L.VdnError(L.VDN_ERR_UNSUPPORTED, "vdn_hybrid_sm_bwd_workspace_size")
            self.sm_workspace = torch.empty(nb, dtype=torch.uint8, device=self.device)
        f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=self.device)
        tok = (c.B, c.T, c.N, c.H)
        g = {"dq": f(*tok, c.d_k), "dk": f(*tok, c.d_k), "dv": f(*tok, c.d_v), "dgate_sm": f(*tok, c.d_v)}
        sg = L.make_sm_grads(dy, g["dq"], g["dk"], g["dv"], g["dgate_sm"], self.sm_workspace, sm_lse=self.sm_lse)
        L.vdn_hybrid_sm_bwd(c, self.args(t), sg, stream)
        return g

    def softmax_backward_status(self, stream=None) -> tuple:
        """(status, kernel tag) of the last softmax backward's bounded waits,
        from the status words at the head of its scratch."""
        a = L.VdnArgs()
        a.workspace = self.sm_workspace.data_ptr()
        a.workspace_bytes = self.sm_workspace.numel()
        return L.vdn_hybrid_device_status(self.cfg, a, stream)

    def backward(self, t: dict, dy: torch.Tensor, stream=None) -> dict:
        """The whole core's gradients after a forward call on the same inputs,
        in one library call (``vdn_hybrid_bwd``): dq, dk, dv with both
        branches' shares summed on the device, and the branch-specific
        gradients (drms_weight / dfwd_init when those inputs are given)."""
        c = self.cfg
        if getattr(self, "whole_bwd_workspace", None) is None:
            nb = L.vdn_hybrid_bwd_workspace_size(c)
            if nb == 0:
                raise L.VdnError(L.VDN_ERR_UNSUPPORTED, "vdn_hybrid_bwd_workspace_size")
            self.whole_bwd_workspace = torch.empty(nb, dtype=torch.uint8, device=self.device)
        f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=self.device)
        tok = (c.B, c.T, c.N, c.H)
        g = {"dq": f(*tok, c.d_k), "dk": f(*tok, c.d_k), "dv": f(*tok, c.d_v), "dbeta": f(*tok),
             "dalpha": f(c.B, c.T, c.H), "dgate_lin": f(*tok, c.d_v), "dgate_sm": f(*tok, c.d_v)}
        if t.get("rms_weight") is not None:
            g["drms_weight"] = f(c.H, c.d_v)
        if t.get("fwd_init") is not None:
            g["dfwd_init"] = f(c.B, c.H, c.d_v, c.d_k)
        gr = L.make_grads(dy, g["dq"], g["dk"], g["dv"], g["dbeta"], g["dalpha"], g["dgate_lin"], g["dgate_sm"],
                          self.whole_bwd_workspace, drms_weight=g.get("drms_weight"), dfwd_init=g.get("dfwd_init"),
                          sm_lse=self.sm_lse)
        L.vdn_hybrid_bwd(c, self.args(t), gr, stream)
        return g

    def backward_status(self, stream=None) -> tuple:
        """(status, kernel tag) of the last whole-core backward: the softmax
        branch's status words (head of the shared scratch), else the linear
        branch's (head of the forward's workspace)."""
        a = L.VdnArgs()
        a.workspace = self.whole_bwd_workspace.data_ptr()
        a.workspace_bytes = self.whole_bwd_workspace.numel()
        st = L.vdn_hybrid_device_status(self.cfg, a, stream)
        if st[0] != L.VDN_OK:
            return st
        a.workspace = self.workspace.data_ptr()
        a.workspace_bytes = self.ws_bytes
        return L.vdn_hybrid_device_status(self.cfg, a, stream)

    def intermediates(self) -> dict:
        """Views of the workspace's intermediate values (float32)."""
        lay = L.vdn_hybrid_workspace_layout(self.cfg)
        c = self.cfg
        C = c.C
        f = lambda off, shape: self.workspace[off:off + 4 * int(np.prod(shape))].view(torch.float32).view(*shape)
        return {
            "half_text": f(lay["half_text"], (c.B, c.H, c.d_v, c.d_k)),
            "M": f(lay["frame_M"], (c.B, c.T, c.H, c.d_k, c.d_k)),
            "C": f(lay["frame_C"], (c.B, c.T, c.H, c.d_v, c.d_k)),
            "fwd_snap": f(lay["fwd_snap"], (c.B, c.H, C + 1, c.d_v, c.d_k)),
            "bwd_snap": f(lay["bwd_snap"], (c.B, c.H, C + 1, c.d_v, c.d_k)),
            "R": f(lay["read_table"], (c.B, c.H, C + 1, c.d_v, c.d_k)),
        }

    def forward_end_state(self) -> torch.Tensor:
        """A copy of the forward state after the last frame (fwd_snap slot C),
        [B, H, d_v, d_k] float32: the next appended segment's ``fwd_init``."""
        return self.intermediates()["fwd_snap"][:, :, self.cfg.C].clone()

    def chunk_maps(self) -> dict:
        """The chunk maps of the chunk-stepped tensor-core scan (bf16 mode,
        d = 128, C >= 4): P_c as hi + lo (float32), Cf_c, Cb_c, Lam_c."""
        lay = L.vdn_hybrid_workspace_layout(self.cfg)
        c = self.cfg
        C, d = c.C, c.d_k
        n = c.B * C * c.H
        if lay["chunk_C"] == lay["chunk_P16"]:
            raise ValueError("no chunk maps for this configuration")
        p16 = self.workspace[lay["chunk_P16"]:lay["chunk_P16"] + 2 * n * 2 * d * d].view(torch.bfloat16)
        p16 = p16.view(c.B, C, c.H, 2, d, d).float()
        cc = self.workspace[lay["chunk_C"]:lay["chunk_C"] + 4 * 2 * n * d * d].view(torch.float32)
        cc = cc.view(2, c.B, C, c.H, d, d)
        lam = self.workspace[lay["chunk_lam"]:lay["chunk_lam"] + 4 * n].view(torch.float32).view(c.B, C, c.H)
        return {"P": p16[:, :, :, 0] + p16[:, :, :, 1], "Cf": cc[0], "Cb": cc[1], "Lam": lam}

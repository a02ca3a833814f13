"""The allocation-free entry point against the regular one.

vdn_hybrid_attn_fwd_noalloc serves callers that cannot allocate device
memory where they run the core (allocation-free runtimes, plug-ins handed
only their buffers): it runs the same kernels on a library-owned fixed
scratch array instead of a caller workspace.  Its output must equal
vdn_hybrid_attn_fwd's bit for bit (the same deterministic kernels on the same
inputs), on two calls in a row with different inputs (the second call sees
the first call's leftovers in the shared array).  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from video_diffusion_hybrid_b200 import _lib as L
from video_diffusion_hybrid_b200.api import HybridAttention, cfg_for, output_shape, to_torch
from video_diffusion_hybrid_b200.build import build
from video_diffusion_hybrid_b200.synth import Shape, make_inputs
from video_diffusion_hybrid_b200.workloads import WORKLOADS

TOL = 2e-2  # bf16-input / fp32-accumulate parity bound, relative to output RMS


def _noalloc_args(t, y):
    return L.make_args(t["q"], t["k"], t["v"], t["beta"], t["alpha"], t["gate_sm"], t["gate_lin"], y,
                       workspace=None, workspace_bytes=0, text_k=t.get("text_k"), text_v=t.get("text_v"),
                       text_beta=t.get("text_beta"))


D128 = Shape(B=1, T=20, N=64, H=2, d_k=128, d_v=128, L=16)
CASES = [
    ("small", WORKLOADS["small"].shape, {}),
    # bf16 d = 128: tensor-core Gram, solve, scan and read; the scan stepped by
    # frames and by composed chunk maps (the chunk-map regions of the array)
    ("d128_frames", D128, {"scan_mode": 1}),
    ("d128_chunks", D128, {"scan_mode": 2}),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,shape,kw", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_regular_entry_point_twice(cuda_ok, name, shape, kw):
    """Same kernels, same inputs: the output must equal the regular entry
    point's bit for bit.  The forward is deterministic (no atomics), so any
    difference means a scratch region read before this call wrote it."""
    build()
    cfg = cfg_for(shape, "bf16", **kw)
    assert L.vdn_hybrid_attn_workspace_size(cfg) <= L.NOALLOC_SCRATCH_BYTES
    ha = HybridAttention(cfg)
    y = torch.empty(output_shape(cfg), dtype=torch.float32, device="cuda")
    for seed in (5, 55):
        t = to_torch(make_inputs(shape, seed, "bf16"), "bf16", "cuda")
        ref = ha(t).clone()
        y.fill_(float("nan"))
        L.vdn_hybrid_attn_fwd_noalloc(cfg, _noalloc_args(t, y))
        torch.cuda.synchronize()
        # the no-alloc call's own status words (every bounded wait completed)
        assert L.vdn_hybrid_noalloc_device_status() == (L.VDN_OK, 0)
        if not torch.equal(y, ref):
            got, want = y.double().cpu().numpy(), ref.double().cpu().numpy()
            errs = [np.nanmax(np.abs(got[..., s, :] - want[..., s, :])) / np.sqrt(np.mean(want[..., s, :] ** 2))
                    for s in (0, 1)]
            pytest.fail(f"{name} seed {seed}: not bit-identical to the regular entry point; max error x RMS "
                        f"per slot {errs} (the bf16 parity bound is {TOL})")


@pytest.mark.gpu
def test_noalloc_rejects_what_does_not_fit(cuda_ok):
    build()
    big = cfg_for(WORKLOADS["768p"].shape, "bf16")
    assert L.vdn_hybrid_attn_workspace_size(big) > L.NOALLOC_SCRATCH_BYTES
    p = 1 << 20
    a = L.make_args(p, p, p, p, p, p, p, p, workspace=None, workspace_bytes=0, text_k=p, text_v=p, text_beta=p)
    assert L.vdn_hybrid_attn_fwd_noalloc(big, a, check=False) == L.VDN_ERR_WORKSPACE
    small = cfg_for(WORKLOADS["small"].shape, "bf16")
    a.workspace = p
    assert L.vdn_hybrid_attn_fwd_noalloc(small, a, check=False) == L.VDN_ERR_INVALID_ARG

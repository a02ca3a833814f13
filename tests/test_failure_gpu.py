"""The device-side failure path on the GPU, made to happen without a fault.

Every wait of the tensor-core kernels is bounded; when one runs out, the
kernel records VDN_ERR_TIMEOUT and its tag in the workspace status words, its
roles stop issuing, drain what they issued, free the TMEM and exit, and the
context stays usable.  Here the state read's epilogue warps get a wait limit
of a few hundred clock cycles, far shorter than the first tile's load and
products take, so their first wait runs out.  The test checks the status the
host reads back, then restores the default limit and checks that the next
call in the same process is correct again (bit for bit against the output
before the failure, and against the fp64 oracle).
"""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O
from video_diffusion_hybrid_b200 import _lib as L
from video_diffusion_hybrid_b200.api import HybridAttention, cfg_for, to_torch
from video_diffusion_hybrid_b200.build import build
from video_diffusion_hybrid_b200.synth import Shape, make_inputs

pytestmark = pytest.mark.gpu


def test_read_wait_timeout_is_reported_and_the_next_call_recovers(cuda_ok):
    build()
    shape = Shape(B=1, T=10, N=256, H=2, d_k=128, d_v=128, L=16)
    inp = make_inputs(shape, 91, "bf16")
    cfg = cfg_for(shape, "bf16")
    assert L.vdn_hybrid_stage_impl(cfg, L.STAGE_READ) == 1  # the tensor-core read
    t = to_torch(inp, "bf16", "cuda")
    ha = HybridAttention(cfg)
    ref = ha(t).clone()
    assert L.vdn_hybrid_device_status(cfg, ha.args(t))[0] == L.VDN_OK
    torch.cuda.synchronize()
    L.vdn_debug_set_read_wait_limit(300)
    try:
        ha.y[..., 1, :].fill_(float("nan"))
        ha(t, stages=L.STAGE_READ)
        st, where = L.vdn_hybrid_device_status(cfg, ha.args(t))
        torch.cuda.synchronize()
    finally:
        L.vdn_debug_set_read_wait_limit(0)
    assert st == L.VDN_ERR_TIMEOUT and where == L.TAG_READ, (st, where)
    assert torch.isnan(ha.y[..., 1, :]).any()  # CTAs that gave up left their rows unwritten
    # same process, default limit: the read is whole again, bit for bit
    ha(t, stages=L.STAGE_READ)
    assert L.vdn_hybrid_device_status(cfg, ha.args(t))[0] == L.VDN_OK
    assert torch.equal(ha.y, ref)
    # and a whole call agrees with the oracle
    y = ha(t).double().cpu().numpy()
    assert L.vdn_hybrid_device_status(cfg, ha.args(t))[0] == L.VDN_OK
    want = O.hybrid_attn({k: v for k, v in inp.items() if not k.endswith("_bits")},
                         O.Cfg(B=1, T=10, N=256, H=2, d_k=128, d_v=128, L=16))
    for s in (0, 1):
        err = np.max(np.abs(y[..., s, :] - want[..., s, :])) / np.sqrt(np.mean(want[..., s, :] ** 2))
        assert err <= 2e-2, (s, err)

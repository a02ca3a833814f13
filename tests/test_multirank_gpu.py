"""The multi-rank layouts with the CUDA core on every rank.

Ulysses head sharding (world size 2) and the branch split (world size 3: two
softmax ranks with 3 and 2 of 5 heads, one Video Delta Attention rank with
all 5), as the pages deploy them on 8 B200s (deepmagic post, section 實測數據;
aimodeling news, "The speedup ledger and a three-stage recipe").  Every rank
is a process of its own that calls libvdn_hybrid.so on cuda:0 for its heads
and its branch; the exchanges run on host copies through gloo (one GPU is all
these tests get, so there is no NCCL and no peer memory, and no kernel of one
rank waits on another's).  Each rank's sequence shard of the output is
compared with the fp64 oracle on the whole problem at the bf16 bar, 2e-2 of
the slot's RMS.  The shards end inside a frame, and T = 16 leaves a
one-frame last chunk.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOL = 2e-2


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _problem(H, seed):
    from video_diffusion_hybrid_b200.synth import Shape, make_inputs
    shp = Shape(B=1, T=16, N=66, H=H, d_k=128, d_v=128, L=16)  # 1056 tokens: 528 or 352 a rank
    return shp, make_inputs(shp, seed, "bf16")


def _errors(y, ref):
    return [float(np.max(np.abs(y[..., s, :] - ref[..., s, :])) / np.sqrt(np.mean(ref[..., s, :] ** 2)))
            for s in (0, 1)]


def _worker(rank, world, port, kind, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import vdn_oracle as O
    from video_diffusion_hybrid_b200 import _lib as L
    from video_diffusion_hybrid_b200.api import cfg_for, to_torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        shp, inp = _problem(4 if kind == "ulysses" else 5, 31 if kind == "ulysses" else 37)
        T, N, H = shp.T, shp.N, shp.H
        sl = T * N // world
        full = to_torch(inp, "bf16", "cpu")
        cfg = cfg_for(shp, "bf16")
        if kind == "ulysses":
            from video_diffusion_hybrid_b200 import ulysses as M
            per_token = M.PER_TOKEN
            core = M.UlyssesHybridAttention(cfg, device="cuda:0")
        else:
            from video_diffusion_hybrid_b200 import branch_split as M
            per_token = M.READ_BY
            core = M.BranchSplitHybridAttention(cfg, n_softmax=2, device="cuda:0")
        local = {k: (v.flatten(1, 2).narrow(1, rank * sl, sl).contiguous() if k in per_token else v)
                 for k, v in full.items()}
        y = core(local)
        torch.cuda.synchronize()
        st, where = core.device_status()
        assert st == L.VDN_OK, (st, where)
        assert y.device.type == "cpu" and y.shape == (1, sl, H, 2, 128)
        oc = O.Cfg(B=1, T=T, N=N, H=H, d_k=128, d_v=128, L=shp.L)
        ref = O.hybrid_attn({k: v for k, v in inp.items() if not k.endswith("_bits")}, oc)
        ref = ref.reshape(1, T * N, H, 2, 128)[:, rank * sl:(rank + 1) * sl]
        out[rank] = _errors(y.double().numpy(), ref)
    finally:
        dist.destroy_process_group()


def _run(kind, world):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), kind, out), nprocs=world, join=True,
                           start_method="spawn")
        errs = dict(out)
    assert sorted(errs) == list(range(world)), errs
    for r, e in errs.items():
        assert max(e) <= TOL, (kind, r, e)


@pytest.mark.gpu
@pytest.mark.timeout(900)
def test_ulysses_two_ranks_cuda_core(cuda_ok):
    _run("ulysses", 2)


@pytest.mark.gpu
@pytest.mark.timeout(900)
def test_branch_split_three_ranks_cuda_core(cuda_ok):
    _run("branch_split", 3)

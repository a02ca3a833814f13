"""The branch split on the host (gloo, world size 3: two softmax ranks, one
linear rank; 5 heads, so the softmax ranks hold 3 and 2): the sequence-
sharded inputs reach each rank as whole sequences of its heads for the inputs
its branch reads, and the oracle run per rank on its branch, merged back,
equals the oracle on the whole problem restricted to the rank's tokens.  The
batch-heads of the core are independent and so are its two branches ([P1] 三:
separate gates and output projections), which is what makes the split exact."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _full_inputs():
    from video_diffusion_hybrid_b200.synth import Shape, make_inputs
    shp = Shape(B=2, T=11, N=6, H=5, d_k=8, d_v=8, L=3)  # 22 tokens a rank: 3.67 frames
    inp = make_inputs(shp, seed=7)
    r = np.random.default_rng(11)
    inp["rms_weight"] = (1 + 0.3 * r.standard_normal((5, 8))).astype(np.float32)
    return shp, {k: v for k, v in inp.items() if not k.endswith("_bits")}


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import vdn_oracle as O
    from video_diffusion_hybrid_b200 import branch_split as BS
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shp, inp = _full_inputs()
        T, N, H = shp.T, shp.N, shp.H
        lay = BS.Layout(H, world, 2)
        sl = T * N // world
        full = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in inp.items()}
        local = {k: (v.flatten(1, 2).narrow(1, rank * sl, sl).contiguous() if k in BS.READ_BY else v)
                 for k, v in full.items()}
        t = BS.split_inputs(local, T, N, lay)
        h0, hn = lay.heads[rank]
        branch = lay.branch(rank)
        # pure data movement: exact, and only what the branch reads
        for k in BS.READ_BY:
            if branch in BS.READ_BY[k]:
                assert torch.equal(t[k], full[k].narrow(3, h0, hn)), k
            else:
                assert k not in t, k
        # the rank's branch by the oracle on its heads (the other slot is not sent)
        t_np = {k: v.numpy() for k, v in t.items()}
        for k in BS.READ_BY:
            t_np.setdefault(k, np.zeros_like(t_np["q"][..., 0]) if k == "beta" else t_np["q"])
        cfg_l = O.Cfg(B=shp.B, T=T, N=N, H=hn, d_k=shp.d_k, d_v=shp.d_v, L=shp.L)
        y_l = torch.from_numpy(O.hybrid_attn(t_np, cfg_l))
        y = BS.merge_outputs(y_l, lay).numpy()
        cfg = O.Cfg(B=shp.B, T=T, N=N, H=H, d_k=shp.d_k, d_v=shp.d_v, L=shp.L)
        ref = O.hybrid_attn(inp, cfg).reshape(shp.B, T * N, H, 2, shp.d_v)[:, rank * sl:(rank + 1) * sl]
        out[rank] = float(np.max(np.abs(y - ref)))
    finally:
        dist.destroy_process_group()


def test_branch_split_equals_whole_problem():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(3, _free_port(), out), nprocs=3, join=True, start_method="spawn")
        assert all(out[r] <= 1e-12 for r in range(3)), dict(out)


def test_layout_splits_each_group_evenly():
    sys.path.insert(0, ROOT)
    from video_diffusion_hybrid_b200 import branch_split as BS
    lay = BS.Layout(24, 8, 5)  # the pages' 5 softmax + 3 linear GPUs
    assert [n for _, n in lay.heads] == [5, 5, 5, 5, 4, 8, 8, 8]
    assert [lay.branch(r) for r in range(8)] == ["sm"] * 5 + ["lin"] * 3
    for grp in (lay.heads[:5], lay.heads[5:]):
        assert grp[0][0] == 0 and sum(n for _, n in grp) == 24
        assert all(a[0] + a[1] == b[0] for a, b in zip(grp, grp[1:]))
    for bad in ((24, 8, 0), (24, 8, 8), (2, 8, 5)):
        with pytest.raises(ValueError):
            BS.Layout(*bad)

"""Ulysses head sharding on the host (world size 2, gloo): the sequence-sharded
inputs reach each rank as every token of its heads, and the oracle run on each
rank's heads, sent back through the inverse exchange, equals the oracle on the
whole problem restricted to the rank's tokens (a shard ends inside a frame).  The batch-heads of the core are
independent ([P1] 三: one state pair per head), which is what makes the split
exact."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _full_inputs():
    from video_diffusion_hybrid_b200.synth import Shape, make_inputs
    shp = Shape(B=2, T=11, N=6, H=4, d_k=8, d_v=8, L=3)  # 33 tokens a rank: 5.5 frames
    inp = make_inputs(shp, seed=5)
    r = np.random.default_rng(9)
    inp["rms_weight"] = (1 + 0.3 * r.standard_normal((4, 8))).astype(np.float32)
    inp["fwd_init"] = (0.2 * r.standard_normal((2, 4, 8, 8))).astype(np.float32)
    return shp, {k: v for k, v in inp.items() if not k.endswith("_bits")}


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import vdn_oracle as O
    from video_diffusion_hybrid_b200 import ulysses as U
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shp, inp = _full_inputs()
        T, N, H = shp.T, shp.N, shp.H
        sl, hl = T * N // world, H // world
        full = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in inp.items()}
        local = {k: (v.flatten(1, 2).narrow(1, rank * sl, sl).contiguous() if k in U.PER_TOKEN else v)
                 for k, v in full.items()}
        t = U.shard_inputs(local, T, N, H)
        # pure data movement: exact
        for k in U.PER_TOKEN:
            assert torch.equal(t[k], full[k].narrow(3, rank * hl, hl)), k
        for k, ax in U.REPLICATED_HEAD_AXIS.items():
            if k in full:
                assert torch.equal(t[k], full[k].narrow(ax, rank * hl, hl)), k
        cfg_l = O.Cfg(B=shp.B, T=T, N=shp.N, H=hl, d_k=shp.d_k, d_v=shp.d_v, L=shp.L)
        y_l = O.hybrid_attn({k: v.numpy() for k, v in t.items()}, cfg_l)
        y = U.gather_output(torch.from_numpy(y_l)).numpy()
        cfg = O.Cfg(B=shp.B, T=T, N=shp.N, H=H, d_k=shp.d_k, d_v=shp.d_v, L=shp.L)
        ref = O.hybrid_attn(inp, cfg).reshape(shp.B, T * N, H, 2, shp.d_v)[:, rank * sl:(rank + 1) * sl]
        out[rank] = float(np.max(np.abs(y - ref)))
    finally:
        dist.destroy_process_group()


def test_ulysses_split_equals_whole_problem():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert out[0] <= 1e-12 and out[1] <= 1e-12, dict(out)


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    from video_diffusion_hybrid_b200 import ulysses as U
    x = torch.randn(1, 15, 4, 2)
    assert U.seq_to_head(x) is x and U.head_to_seq(x) is x
    t = U.shard_inputs({"q": x, "rms_weight": torch.ones(4, 2)}, 5, 3, 4)
    assert t["q"].shape == (1, 5, 3, 4, 2) and torch.equal(t["q"].flatten(1, 2), x)
    assert t["rms_weight"].shape == (4, 2)

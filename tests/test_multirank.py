"""The multi-process path on CPU (world size 2, gloo): the bench's timing is
the maximum over the ranks, and under torchrun the reference arm prints one
line from rank 0 while the other rank exits without work.  The core itself
has no exchange step (every batch-head is independent), so these are the only
multi-rank paths."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank])
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert out[0] == [2.0, 5.0] and out[1] == [2.0, 5.0]


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3, 4.5]) == [3.0, 4.5]


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0", "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_bench_backward_work_counts():
    """The backward bench's pair count uses the mask density; it must be the
    oracle's (19.975 % at T = 90), and the linear branch's algorithmic work
    scales with the token-heads."""
    import bench
    from oracle import vdn_oracle as O
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    s = WORKLOADS["768p"].shape
    assert abs(bench.O_density(s) - O.mask_density(s.T, 5, 4)) < 1e-15
    f1, b1 = bench.bwd_work(s, True)
    assert f1 > 4.5e11 and b1 == s.B * s.T * s.N * s.H * (4 * s.d_k * 2 + 4 + 4 * s.d_k + 16 * s.d_k + 4)

#!/usr/bin/env python
"""Throughput of the Video DeltaNet hybrid attention core on B200.

One step = one pass of the whole core (text solve, per-frame Gram/solve,
bidirectional scan, windowed softmax, state read + epilogue) over one batch
of synthetic input of the named workload (default: the 768p single-block
stand-in, T=90, N=1008, H=24, d=128, L=512, bf16).  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 it runs under torchrun, one rank per GPU; every rank processes its
own independent problem (weak scaling, no collective on the data path) and
the time is the max over ranks.  ``--impl reference`` times the fp64 CPU
oracle on the host cores instead (rank 0 only), on a bounded sample.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "video tokens/s per hybrid-attn layer on 1 B200; % tensor-pipe / HBM roofline"
UNIT = "video tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="768p")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--vda-only", action="store_true",
                    help="the Video Delta Attention stages only (the d = 256 sweep shapes have no softmax)")
    ap.add_argument("--xattn", action="store_true",
                    help="time the text cross-attention (every video query over the L text tokens) at the "
                         "workload's shape instead of the core")
    ap.add_argument("--fp8", action="store_true",
                    help="with --proj: e4m3 operands (the activation quantised in the timed region)")
    ap.add_argument("--update", type=int, choices=(0, 1, 2), default=0,
                    help="the linear branch's frame write: 0 the joint solve; ablation baselines 1 frame-level "
                         "independent writes (1/N rescaled), 2 the token-wise delta rule")
    ap.add_argument("--ulysses", action="store_true",
                    help="one problem of the workload's shape over the launched ranks, heads split across them "
                         "(sequence-sharded in and out, two all-to-alls around the core): strong scaling")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward of the linear branch (vdn_hybrid_lin_bwd) after one forward")
    ap.add_argument("--proj", action="store_true",
                    help="time the layer's output projection (one GEMM over the core's concat axis) at the "
                         "workload's shape instead of the core")
    return ap.parse_args()


# ----------------------------------------------------------------- oracle --
def oracle_prepare(workload, seed_offset=0):
    """Inputs of head 0 of the workload for the oracle (generated once, untimed)."""
    from oracle import vdn_oracle as O
    from video_diffusion_hybrid_b200.synth import Shape, make_inputs
    s = workload.shape
    one = Shape(B=1, T=s.T, N=s.N, H=1, d_k=s.d_k, d_v=s.d_v, L=s.L)
    inp = make_inputs(one, workload.seed + seed_offset, workload.dtype)
    cfg = O.Cfg(B=1, T=s.T, N=s.N, H=1, d_k=s.d_k, d_v=s.d_v, L=s.L)
    return inp, cfg


def oracle_sample(workload, prep, frames=None, n_anchor_q=None, target_s=None, vda_only=False):
    """Time the fp64 oracle on a bounded sample of head 0 of the workload: the
    full bidirectional VDA chain of the head (text solve, every frame's solve,
    both scans), both branches for every query of the non-anchor frames in
    `frames`, and both branches for `n_anchor_q` queries of anchor frame 0.
    With `target_s`, further whole non-anchor frames (spread over the
    sequence) are added until the sample holds about that much CPU work.
    The per-frame costs are extrapolated to all frames of the head and the
    head's cost to all B x H heads.  With `vda_only`, the frames' cost is the
    linear branch alone (the read and its RMSNorm and gate).  Returns
    (tokens/s, seconds of CPU work, description)."""
    from oracle import vdn_oracle as O
    inp, cfg = prep
    s = workload.shape
    frames = frames if frames is not None else (s.T // 2, s.T // 4)
    n_anchor_q = min(n_anchor_q if n_anchor_q is not None else s.N, s.N)
    t0 = time.perf_counter()
    F, G = O.head_states(inp, cfg, 0, 0)
    t_chain = time.perf_counter() - t0
    q = inp["q"][0, :, :, 0].astype(np.float64)
    k, v = inp["k"][0, :, :, 0], inp["v"][0, :, :, 0]

    def frame_cost(t, n):
        t1 = time.perf_counter()
        R = O.read_state(F, G, t, s.T, cfg.chunk, cfg.anchors)
        O.rms_gate(q[t, :n] @ R.T, inp["gate_lin"][0, t, :n, 0], cfg.rms_eps)
        if not vda_only:
            o = O.softmax_frame(q[t, :n], k, v, t, s.T, cfg.chunk, cfg.anchors, cfg.scale)
            O.sigmoid(inp["gate_sm"][0, t, :n, 0]) * o
        return time.perf_counter() - t1

    frames = list(frames)
    c_frames = [frame_cost(t, s.N) for t in frames]
    c_anchor = frame_cost(0, n_anchor_q)
    if target_s:
        # positions spread over the sequence first, then the remaining frames:
        # at most the whole head is timed
        spread = [s.T * (2 * i + 1) // 64 for i in range(32)] + list(range(1, s.T - 1))
        order = list(dict.fromkeys(t for t in spread if 0 < t < s.T - 1 and t not in frames))
        while order and t_chain + sum(c_frames) + c_anchor < target_s:
            frames.append(order.pop(0))
            c_frames.append(frame_cost(frames[-1], s.N))
    n_anchor = 2 if cfg.anchors else 0
    per_head = (t_chain + (s.T - n_anchor) * statistics.mean(c_frames)
                + n_anchor * c_anchor * s.N / n_anchor_q)
    layer = per_head * s.H * s.B
    work = t_chain + sum(c_frames) + c_anchor
    what = "the linear branch" if vda_only else "both branches"
    desc = (f"head 0 of {workload.name}: the full VDA chain over {s.T} frames, {what} for all {s.N} "
            f"queries of {len(frames)} non-anchor frames spread over the sequence and {n_anchor_q} queries of "
            f"anchor frame 0; costs extrapolated to {s.T} frames x {s.B * s.H} heads")
    return s.B * s.T * s.N / layer, work, desc


def max_over_ranks(vals, device=None):
    """Each value's maximum over the ranks of the process group (the slowest
    rank defines a step); the values themselves on a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    x = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return x.tolist()


def host_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    if int(os.environ.get("RANK", "0")) != 0:
        return
    w = WORKLOADS[args.workload]
    prep = oracle_prepare(w)
    vals, times = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        val, _work, desc = oracle_sample(w, prep, frames=(w.shape.T // 2,), n_anchor_q=128)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            vals.append(val)
            times.append(dt)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.shape.B, "T": w.shape.T, "N": w.shape.N, "H": w.shape.H,
                   "d": w.shape.d_k, "L": w.shape.L, "inputs": w.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- ours ----
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(kernel_file: str, key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (matching hash); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(key)
    if not d:
        return None
    src = open(os.path.join(ROOT, "video_diffusion_hybrid_b200", "csrc", kernel_file), "rb").read()
    if hashlib.sha256(src).hexdigest()[:16] != d.get("source_sha256_16"):
        return None
    return d.get("dram_bytes_per_launch")


def stage_rooflines(s, cfg, ms, y_elem, peaks, sm_mhz):
    """Each stage's time (CUDA events, the stage launched alone on resident
    inputs) against the roofline of what it must compute or move."""
    from video_diffusion_hybrid_b200 import roofline as R
    from video_diffusion_hybrid_b200 import _lib as L
    elem = 2 if cfg.dtype == 1 else 4
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]  # each stage is timed alone: burst
    simt = R.fp32_simt_tflops(sm_mhz)
    out = {"text": {"ms": ms["text"]}}
    if "softmax" in ms:
        f = R.softmax_flops(s.B, s.T, s.N, s.H, s.d_k, cfg.chunk, cfg.anchors)
        a = f / (ms["softmax"] / 1e3) / 1e12
        out["softmax"] = {"ms": ms["softmax"], "bound": "tensor", "achieved": a, "peak": tc, "unit": "TFLOP/s",
                          "frac": a / tc, "work": f}
    for name, by in (("read", R.read_bytes(s.B, s.T, s.N, s.H, s.d_k, elem, y_elem)),
                     ("scan", R.scan_bytes(s.B, s.T, s.H, s.d_k, cfg.chunk, cfg.anchors))):
        a = by / (ms[name] / 1e3) / 1e9
        out[name] = {"ms": ms[name], "bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm,
                     "work": by}
    gb = R.gram_bytes(s.B, s.T, s.N, s.H, s.d_k, cfg.anchors, elem)
    if cfg.update == 1 and L.vdn_hybrid_stage_impl(cfg, L.STAGE_TEXT) == 1 and s.d_k <= 128:
        # frame-level writes from the tensor-core Gram, then the in-place
        # rescale (reads and writes the M and C slots once)
        by = gb + 4 * R.written_frames(s.T, cfg.anchors) * s.B * s.H * s.d_k * s.d_k * 4
        a = by / (ms["solve"] / 1e3) / 1e9
        out["solve"] = {"ms": ms["solve"], "kernel": "gram_tc+rescale", "bound": "hbm", "achieved": a, "peak": hbm,
                        "unit": "GB/s", "frac": a / hbm, "work": by}
        return out
    if cfg.update != 0:
        # the ablation writes' map kernel: fp32 FMA per token on the 2d x d
        # stacked map (the update; the token rule adds the dot product)
        f = R.variant_map_flops(s.B, s.T, s.N, s.H, s.d_k, cfg.anchors, cfg.update)
        a = f / (ms["solve"] / 1e3) / 1e12
        out["solve"] = {"ms": ms["solve"], "kernel": "variant_map", "bound": "alu", "achieved": a, "peak": simt,
                        "unit": "TFLOP/s", "frac": a / simt, "work": f, "hbm_floor_ms": 1e3 * gb / (hbm * 1e9)}
        return out
    # per-frame Gram (HBM-bound) followed by the SPD sweep (fp32 SIMT-bound):
    # the floor is the sum of the two
    # the tensor-core scan takes B_t itself, so its solve forms no C = B M
    sf = R.sweep_flops(s.B, s.T, s.H, s.d_k, cfg.anchors, with_c=L.vdn_hybrid_stage_impl(cfg, L.STAGE_SCAN) != 1)
    floor_ms = 1e3 * (gb / (hbm * 1e9) + sf / (simt * 1e12))
    out["solve"] = {"ms": ms["solve"], "bound": "hbm+alu", "floor_ms": floor_ms, "frac": floor_ms / ms["solve"],
                    "gram_bytes": gb, "sweep_flops": sf, "alu_peak_tflops": simt}
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    from video_diffusion_hybrid_b200 import _lib as L
    from video_diffusion_hybrid_b200.api import HybridAttention, cfg_for
    from video_diffusion_hybrid_b200.roofline import softmax_flops
    from video_diffusion_hybrid_b200.synth import make_inputs_torch
    from video_diffusion_hybrid_b200.workloads import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    L.lib()  # fail loudly if the extension is missing

    w = WORKLOADS[args.workload]
    s = w.shape
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.update == 0:
        val, work, desc = oracle_sample(w, oracle_prepare(w), target_s=12.0, vda_only=args.vda_only)
        cpu = {"value": val, "unit": UNIT, "cores": host_cores(), "kind": "oracle", "sample": desc,
               "sample_cpu_seconds": round(work, 2)}

    t = make_inputs_torch(s, w.seed + 17 * rank, w.dtype, dev)
    # y in the mode's type: bf16 in the bf16 mode (both gated branches rounded
    # to nearest even on store), fp32 in the fp32 mode
    y_dtype = L.VDN_BF16 if w.dtype == "bf16" else L.VDN_F32
    cfg = cfg_for(s, w.dtype, update=args.update, y_dtype=y_dtype)
    ha = HybridAttention(cfg, dev)
    stream = torch.cuda.current_stream(dev)
    pre = L.STAGE_TEXT | L.STAGE_SOLVE | L.STAGE_SCAN
    vda_only = args.vda_only
    # kernels a step launches: text (Gram + sweep on tensor cores, else one
    # SIMT kernel), frame Gram + sweep (else one SIMT solve), scan, softmax,
    # read table + read (else one SIMT read)
    tc = lambda st: L.vdn_hybrid_stage_impl(cfg, st) == 1
    text_k = (2 if tc(L.STAGE_TEXT) else 1) if s.L > 0 else 0  # no text: a memset, no kernel
    # the frame-level ablation write on bf16 inputs: tensor-core Gram + rescale
    variant_gram = args.update == 1 and tc(L.STAGE_TEXT) and s.d_k <= 128
    launches_per_step = (text_k + (2 if tc(L.STAGE_SOLVE) or variant_gram else 1) + 1 + (0 if vda_only else 1)
                         + (2 if tc(L.STAGE_READ) else 1))
    K, W = args.steps, args.warmup
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    # the dominant kernel's events: the softmax, or the read in the VDA-only mode
    dom = L.STAGE_READ if vda_only else L.STAGE_SOFTMAX

    def step(i=None):
        ha(t, stages=pre)
        if i is not None:
            ev[i][0].record(stream)
        ha(t, stages=dom)
        if i is not None:
            ev[i][1].record(stream)
        if not vda_only:
            ha(t, stages=L.STAGE_READ)

    for _ in range(W):
        step()
    torch.cuda.synchronize(dev)
    st, where = L.vdn_hybrid_device_status(cfg, ha.args(t))
    if st != L.VDN_OK:
        raise SystemExit(f"device status {st} at kernel tag {where}")

    props = torch.cuda.get_device_properties(dev)
    clk = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if rank == 0:
        clk.start()
        time.sleep(0.3)
    start.record(stream)
    for i in range(K):
        step(i)
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = clk.stop() if rank == 0 else None
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end) / K
    sm_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms, sm_ms = max_over_ranks([ms, sm_ms], dev)

    # end to end: pinned host inputs -> device, the call, the whole output back,
    # every step.  Two device buffer sets let the upload of step i + 1 (copy
    # stream) and the download of step i - 1 (second copy stream) run while
    # step i computes; each step still moves all of its inputs and its result.
    e2e = None
    if not args.no_e2e:
        host = {k: v.cpu().pin_memory() for k, v in t.items()}
        yh = [torch.empty(ha.y.shape, dtype=ha.y.dtype, pin_memory=True) for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = yh[0].numel() * yh[0].element_size()
        sets = [(t, ha), ({k: torch.empty_like(v) for k, v in t.items()}, HybridAttention(cfg, dev))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        e2e_stages = (pre | L.STAGE_READ) if vda_only else L.STAGE_ALL

        def pipeline(n):
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            in_ev = [torch.cuda.Event() for _ in range(2)]
            comp_ev = [torch.cuda.Event() for _ in range(2)]
            out_ev = [torch.cuda.Event() for _ in range(2)]
            start.record(stream)
            s_in.wait_event(start)
            s_out.wait_event(start)
            for i in range(n):
                slot = i % 2
                ti, hi = sets[slot]
                if i >= 2:
                    s_in.wait_event(comp_ev[slot])  # step i - 2 has read these inputs
                with torch.cuda.stream(s_in):
                    for k, v in host.items():
                        ti[k].copy_(v, non_blocking=True)
                in_ev[slot].record(s_in)
                stream.wait_event(in_ev[slot])
                if i >= 2:
                    stream.wait_event(out_ev[slot])  # step i - 2's result has been read back
                hi(ti, stages=e2e_stages, stream=stream)
                comp_ev[slot].record(stream)
                s_out.wait_event(comp_ev[slot])
                with torch.cuda.stream(s_out):
                    yh[slot].copy_(hi.y, non_blocking=True)
                out_ev[slot].record(s_out)
            stream.wait_stream(s_out)
            end.record(stream)
            torch.cuda.synchronize(dev)
            return start.elapsed_time(end)

        pipeline(max(2, W))
        if world > 1:
            dist.barrier()
        ems = max_over_ranks([pipeline(K) / K], dev)[0]
        e2e = {"value": world * w.tokens / (ems / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "overlap": "upload of step i+1 and download of step i-1 run during step i (3 streams)"}
        del sets[1]
        torch.cuda.empty_cache()

    # stage by stage, each launched alone (inputs and earlier stages' results resident)
    stage_ms = {}
    for name, st in (("text", L.STAGE_TEXT), ("solve", L.STAGE_SOLVE), ("scan", L.STAGE_SCAN),
                     ("softmax", L.STAGE_SOFTMAX), ("read", L.STAGE_READ)):
        if vda_only and st == L.STAGE_SOFTMAX:
            continue
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ha(t, stages=st)
        a.record(stream)
        for _ in range(3):
            ha(t, stages=st)
        b.record(stream)
        torch.cuda.synchronize(dev)
        stage_ms[name] = a.elapsed_time(b) / 3

    if rank == 0:
        peaks, src = load_peaks()
        in_gb = 5 * s.B * s.T * s.N * s.H * s.d_k * (2 if w.dtype == "bf16" else 4) / 1e9
        if vda_only:
            from video_diffusion_hybrid_b200.roofline import read_bytes
            by = read_bytes(s.B, s.T, s.N, s.H, s.d_k, 2 if w.dtype == "bf16" else 4, ha.y.element_size())
            achieved = by / (sm_ms / 1e3) / 1e9
            roof = {"kernel": "state_read" + ("_tcgen05" if tc(L.STAGE_READ) else "_simt"), "bound": "hbm",
                    "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "peak_source": f"hbm_gbs ({src})", "ms_per_launch": sm_ms,
                    "bytes_per_launch": by, "traffic": None}
        else:
            flops = softmax_flops(s.B, s.T, s.N, s.H, s.d_k, cfg.chunk, cfg.anchors)
            achieved = flops / (sm_ms / 1e3) / 1e12
            # the kernel is timed inside a timed region of well under a second,
            # so the burst peak applies; the sustained fraction is given beside it
            peak = peaks["bf16_tflops"]
            impl = L.vdn_hybrid_stage_impl(cfg, L.STAGE_SOFTMAX)
            roof = {"kernel": "window_softmax" + ("_tcgen05" if impl == 1 else "_simt"), "bound": "tensor",
                    "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                    "peak_source": f"bf16_tflops, burst ({src})",
                    "frac_sustained": achieved / peaks["bf16_tflops_sustained"], "ms_per_launch": sm_ms,
                    "flops_per_launch": flops,
                    "traffic": kernel_traffic("vdn_softmax_tc.cu" if impl == 1 else "vdn_simt.cu", "window_softmax")}
        line = {
            "metric": METRIC, "value": world * w.tokens / (ms / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": s.B, "T": s.T, "N": s.N, "H": s.H, "d": s.d_k, "L": s.L,
                       "chunk": 5, "anchors": 4, "state": "fp32", "accumulate": "fp32",
                       "y": "bf16" if y_dtype == L.VDN_BF16 else "fp32",
                       "stages": "vda" if vda_only else "all",
                       "frame_write": ("joint solve", "frame-level independent (1/N)", "token-wise delta rule")[args.update],
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": f"inputs exceed L2 ({in_gb:.1f} GB of q/k/v/gates per step)"},
            "roofline": roof,
            "stages": stage_rooflines(s, cfg, stage_ms, ha.y.element_size(), peaks,
                                      (clocks or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * K,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_proj(args):
    """The layer's output projection out = y W at the workload's layer shape:
    M = B*T*N tokens, K = H*2*d_v (the core's concat axis), N = H*d_v (the
    model width), bf16 operands and output, fp32 accumulation.  One GPU."""
    import torch
    from video_diffusion_hybrid_b200 import _lib as L
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    s = w.shape
    M, K, N = s.B * s.T * s.N, s.H * 2 * s.d_v, s.H * s.d_v
    gen = torch.Generator(device="cuda").manual_seed(w.seed)
    y = torch.randn((M, K), device="cuda", generator=gen).to(torch.bfloat16)
    wt = (torch.randn((K, N), device="cuda", generator=gen) / K ** 0.5).to(torch.bfloat16)
    out = torch.empty((M, N), device="cuda", dtype=torch.bfloat16)
    if args.fp8:
        # the weight once (transposed, [N, K]); the activation every step
        qy = torch.empty((M, K), device="cuda", dtype=torch.uint8)
        qw = torch.empty((N, K), device="cuda", dtype=torch.uint8)
        scales = torch.zeros(2, device="cuda", dtype=torch.float32)
        L.vdn_quantize_fp8(wt.t().contiguous(), L.VDN_BF16, N * K, qw, scales[1:2])

        def step():
            L.vdn_quantize_fp8(y, L.VDN_BF16, M * K, qy, scales[0:1])
            L.vdn_out_proj_fp8(M, K, N, L.VDN_BF16, qy, qw, scales, out)
    else:
        def step():
            L.vdn_out_proj(M, K, N, L.VDN_BF16, y, wt, out)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    clk = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0])
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks = clk.stop()
    ms = e0.elapsed_time(e1) / args.steps
    gemm_ms = None
    if args.fp8:  # the GEMM alone, for its roofline
        e0.record()
        for _ in range(args.steps):
            L.vdn_out_proj_fp8(M, K, N, L.VDN_BF16, qy, qw, scales, out)
        e1.record()
        torch.cuda.synchronize()
        gemm_ms = e0.elapsed_time(e1) / args.steps
    peaks, src = load_peaks()
    tflops = 2.0 * M * K * N / ((gemm_ms or ms) * 1e-3) / 1e12
    # fp8 dense peak: the measured bf16 figure times the nominal fp8 / bf16 ratio (4.5 / 2.25)
    peak = peaks.get("bf16_tflops", 1590.0) * (2.0 if args.fp8 else 1.0)
    print(json.dumps({
        "metric": "layer output projection (one GEMM over the concat axis)", "value": tflops, "unit": "TFLOP/s",
        "ms_per_step": ms, "gemm_ms": gemm_ms, "steps": args.steps, "n_gpus": 1, "higher_is_better": True,
        "dtype": "fp8_e4m3" if args.fp8 else "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "kernel": "k_gemm_tc (tcgen05, CTA pairs)",
                   "step": "quantise y + FP8 GEMM" if args.fp8 else "bf16 GEMM"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                     "peak_source": f"bf16_tflops ({src})" + (" x 2 (nominal fp8 / bf16)" if args.fp8 else "")},
        "clocks": clocks}), flush=True)


def run_xattn(args):
    """The block's text cross-attention at the workload's shape: B*T*N video
    queries per head over the L text tokens, bf16 q / k / v, fp32 output."""
    import torch
    from video_diffusion_hybrid_b200 import _lib as L
    from video_diffusion_hybrid_b200.api import cfg_for
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    s = w.shape
    cfg = cfg_for(s, "bf16")
    gen = torch.Generator(device="cuda").manual_seed(w.seed)
    q = torch.randn((s.B, s.T, s.N, s.H, s.d_k), device="cuda", generator=gen).to(torch.bfloat16)
    tk = torch.randn((s.B, s.L, s.H, s.d_k), device="cuda", generator=gen).to(torch.bfloat16)
    tv = torch.randn((s.B, s.L, s.H, s.d_v), device="cuda", generator=gen).to(torch.bfloat16)
    y = torch.empty((s.B, s.T, s.N, s.H, s.d_v), device="cuda", dtype=torch.float32)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    a = L.make_args(q, None, None, None, None, None, None, y, ws, text_k=tk, text_v=tv)
    for _ in range(max(args.warmup, 3)):
        L.vdn_text_cross_attn(cfg, a)
    torch.cuda.synchronize()
    clk = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0])
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        L.vdn_text_cross_attn(cfg, a)
    e1.record()
    torch.cuda.synchronize()
    clocks = clk.stop()
    assert L.vdn_hybrid_device_status(cfg, a)[0] == L.VDN_OK
    ms = e0.elapsed_time(e1) / args.steps
    peaks, src = load_peaks()
    flops = 4.0 * s.d_k * s.L * s.B * s.T * s.N * s.H
    tflops = flops / (ms * 1e-3) / 1e12
    hbm = (2 * s.B * s.T * s.N * s.H * s.d_k + 4 * s.B * s.T * s.N * s.H * s.d_v) / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "text cross-attention", "value": s.B * s.T * s.N / (ms * 1e-3), "unit": "video tokens/s",
        "ms_per_step": ms, "steps": args.steps, "n_gpus": 1, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": args.workload, "B": s.B, "T": s.T, "N": s.N, "H": s.H,
                                        "d": s.d_k, "L": s.L},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks.get("bf16_tflops", 1590.0),
                     "unit": "TFLOP/s", "frac": tflops / peaks.get("bf16_tflops", 1590.0),
                     "peak_source": f"bf16_tflops ({src})", "hbm_gbs": hbm},
        "clocks": clocks}), flush=True)


def bwd_work(s, bf16: bool):
    """Algorithmic work of one backward of the linear branch: fp32 flops and
    the bytes it must move.  Per token-head 12 d^2 multiply-adds pairs (o = R q
    again, dq = R^T do, dR += do q^T; K dA, V dB, K dB^T); per written
    frame-head four d^3 products for the two state and the two adjoint chains
    and two for dA.  Bytes: q, k, v, gate_lin in their storage type, beta,
    dy's linear slot (fp32), and the fp32 dq, dk, dv, dgate_lin, dbeta out."""
    tok = s.B * s.T * s.N * s.H
    fh = s.B * (s.T - 2) * s.H
    d = s.d_k
    flops = 2.0 * (6 * d * d) * tok + 2.0 * 6 * d ** 3 * fh
    el = 2 if bf16 else 4
    byts = tok * (4 * d * el + 4 + 4 * d + 4 * 4 * d + 4)
    return flops, byts


def run_bwd(args):
    """The core's backward at the workload's size: one forward (which leaves
    M_t and the write matrices in the workspace and the softmax log-sum-exp
    in its own buffer), then the timed steps, each
    one call of each branch's backward for a fixed upstream gradient dy: the
    linear branch (gradients of q, k, v, beta, alpha, gate_lin, the RMS weight)
    and the windowed softmax branch (q, k, v, gate_sm).  Each branch is timed
    with CUDA events of its own on the launching stream."""
    import torch
    from video_diffusion_hybrid_b200 import _lib as L
    from video_diffusion_hybrid_b200.api import HybridAttention, cfg_for, output_shape
    from video_diffusion_hybrid_b200.synth import make_inputs_torch
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    s = w.shape
    t = make_inputs_torch(s, w.seed, w.dtype, "cuda")
    cfg = cfg_for(s, w.dtype)
    ha = HybridAttention(cfg, keep_lse=True)  # the forward keeps the softmax log-sum-exp for the backward
    ha(t)
    gen = torch.Generator(device="cuda").manual_seed(w.seed + 1)
    dy = torch.randn(output_shape(cfg), generator=gen, device="cuda")
    g = ha.linear_backward(t, dy, want_rms=True)
    lg = L.make_lin_grads(dy, g["dq"], g["dk"], g["dv"], g["dbeta"], g["dalpha"], g["dgate_lin"],
                          ha.bwd_workspace, drms_weight=g["drms_weight"])
    gs = ha.softmax_backward(t, dy)
    sg = L.make_sm_grads(dy, gs["dq"], gs["dk"], gs["dv"], gs["dgate_sm"], ha.sm_workspace, sm_lse=ha.sm_lse)
    a = ha.args(t)
    for _ in range(max(args.warmup, 3)):
        L.vdn_hybrid_lin_bwd(cfg, a, lg)
        L.vdn_hybrid_sm_bwd(cfg, a, sg)
    torch.cuda.synchronize()
    clk = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0])
    clk.start()
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps + 1)]
    ev[0].record(stream)
    for i in range(args.steps):
        L.vdn_hybrid_lin_bwd(cfg, a, lg)
        ev[2 * i + 1].record(stream)
        L.vdn_hybrid_sm_bwd(cfg, a, sg)
        ev[2 * i + 2].record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop()
    lin_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps)) / args.steps
    sm_ms = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(args.steps)) / args.steps
    ms = lin_ms + sm_ms
    flops, byts = bwd_work(s, w.dtype == "bf16")
    pairs = O_density(s) * (s.T * s.N) ** 2 * s.H * s.B
    sm_flops = 10.0 * s.d_k * pairs  # s, dP, dq, dk, dv: 2 d flops each per allowed pair
    simt_peak = 148 * 128 * 2 * 1.965e9 / 1e12  # fp32 FMA lanes x 2 flops x max SM clock
    peaks, src = load_peaks()
    # the softmax backward runs on the tensor cores for bf16 inputs (fp16 operands:
    # the dense fp16 rate equals the bf16 one); a step of both branches is long,
    # so the sustained GEMM rate is the denominator
    sm_tc = L.vdn_hybrid_stage_impl(cfg, L.STAGE_SOFTMAX_BWD) == 1
    tc_peak = peaks.get("bf16_tflops_sustained", 1400.0)
    sm_peak = tc_peak if sm_tc else simt_peak
    sm_tf = sm_flops / (sm_ms * 1e-3) / 1e12
    lin_tf = flops / (lin_ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "hybrid-attn core backward", "value": w.tokens / (ms * 1e-3), "unit": "video tokens/s",
        "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup, "n_gpus": 1, "higher_is_better": True,
        "dtype": "f32" if w.dtype == "f32" else "bf16 in; fp16 tensor-core operands (softmax), f32 SIMT (linear)",
        "data": "synthetic",
        "config": {"workload": w.name, "B": s.B, "T": s.T, "N": s.N, "H": s.H, "d": s.d_k, "L": s.L,
                   "l2": "inputs larger than L2"},
        "gpu_launches": (6 + (5 if sm_tc else 2)) * args.steps,
        "branches": {
            "linear": {"ms": lin_ms, "kernels": 6, "bound": "alu", "flops": flops, "hbm_bytes": byts,
                       "tflops": lin_tf, "peak": simt_peak, "frac": lin_tf / simt_peak},
            "softmax": {"ms": sm_ms, "kernels": 5 if sm_tc else 2, "bound": "tensor" if sm_tc else "alu",
                        "flops": sm_flops, "pairs": pairs, "tflops": sm_tf, "peak": sm_peak,
                        "frac": sm_tf / sm_peak}},
        "roofline": {"bound": "tensor" if sm_tc else "alu", "kernel": "softmax-branch backward (dq + dk/dv kernels)",
                     "achieved": sm_tf, "peak": sm_peak, "unit": "TFLOP/s", "frac": sm_tf / sm_peak,
                     "peak_source": (f"bf16_tflops_sustained ({src})" if sm_tc else
                                     "148 SMs x 128 fp32 lanes x 2 x 1.965 GHz (SIMT fp32)"),
                     "flops": sm_flops, "traffic": None},
        "clocks": clocks}), flush=True)


def O_density(s) -> float:
    """Fraction of (query, key) frame pairs the mask allows (chunk 5, anchors)."""
    c = [t // 5 for t in range(s.T)]
    anc = {0, s.T - 1}
    n = sum(1 for a in range(s.T) for b in range(s.T) if abs(c[a] - c[b]) <= 1 or a in anc or b in anc)
    return n / s.T ** 2


def run_ulysses(args):
    """The workload's one problem over the launched ranks with the heads split
    (Ulysses): every rank holds 1/P of the token sequence of every head, two
    all-to-alls (NCCL) move it to and from head shards around the core.  The
    whole job is one problem, so value = its tokens / the slowest rank's time."""
    import datetime

    import torch
    import torch.distributed as dist
    from video_diffusion_hybrid_b200 import _lib as L
    from video_diffusion_hybrid_b200.api import cfg_for
    from video_diffusion_hybrid_b200.synth import make_inputs_torch
    from video_diffusion_hybrid_b200.ulysses import PER_TOKEN, UlyssesHybridAttention
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    L.lib()
    w = WORKLOADS[args.workload]
    s = w.shape
    # the same problem on every rank; each keeps its shard of the token sequence
    full = make_inputs_torch(s, w.seed, w.dtype, dev)
    sl = s.T * s.N // world
    t = {k: (v.flatten(1, 2).narrow(1, rank * sl, sl).contiguous() if k in PER_TOKEN else v)
         for k, v in full.items()}
    del full
    u = UlyssesHybridAttention(cfg_for(s, w.dtype), None, dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(args.warmup, 3)):
        y = u(t)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        y = u(t)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev)[0]
    # the core's device status words (bounded waits that gave up, if any)
    st, where = u.device_status()
    if st != L.VDN_OK:
        raise SystemExit(f"rank {rank}: device status {st} (kernel tag {where})")
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": w.tokens / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "B": s.B, "T": s.T, "N": s.N, "H": s.H, "d": s.d_k, "L": s.L,
                       "parallelism": f"ulysses{world}", "heads_per_rank": s.H // world,
                       "exchange": "NCCL all_to_all_single, sequence <-> heads, before and after the core"},
            "output_shape": list(y.shape)}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.ulysses:
        run_ulysses(args)
        return
    if args.xattn:
        run_xattn(args)
        return
    if args.bwd:
        run_bwd(args)
        return
    if args.proj:
        run_proj(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

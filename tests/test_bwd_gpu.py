"""GPU parity of the core's backward through the C ABI: the linear branch
(``vdn_hybrid_lin_bwd``) and the windowed softmax branch (``vdn_hybrid_sm_bwd``)
against the float64 autograd oracles of those branches, on the same seeded
inputs.

Bar, per gradient: max |g_gpu - g_oracle| <= tol * RMS(g_oracle).  tol is
1e-3 in fp32 mode: the backward runs two adjoint scans whose every step is a
d x d fp32 product (rounding about d * 2^-24 per step) compounded over up to T
frames, ten times the forward's fp32 bar.  In bf16-input mode both sides see
the same bf16-rounded inputs and the backward computes in fp32, so the
forward's bf16 bar (2e-2) is kept.
"""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O
from oracle import vdn_oracle_grad as OG
from video_diffusion_hybrid_b200 import _lib as L
from video_diffusion_hybrid_b200.api import HybridAttention, cfg_for, output_shape, to_torch
from video_diffusion_hybrid_b200.build import build
from video_diffusion_hybrid_b200.synth import Shape, bf16_round, bf16_to_f32, make_inputs

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-3, "bf16": 2e-2}
NAMES = ("q", "k", "v", "beta", "alpha", "gate_lin", "rms_weight", "fwd_init")


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    build()


def _ocfg(cfg: L.HybridCfg) -> O.Cfg:
    return O.Cfg(B=cfg.B, T=cfg.T, N=cfg.N, H=cfg.H, d_k=cfg.d_k, d_v=cfg.d_v, L=cfg.L, chunk=cfg.chunk,
                 anchors=cfg.anchors, rms_eps=cfg.rms_eps or 1e-6, out_mode=cfg.out_mode,
                 softmax_scale=cfg.softmax_scale)


def _dy(cfg: L.HybridCfg, seed: int) -> np.ndarray:
    """A seeded upstream gradient in y's shape, rounded to y's dtype."""
    dy = np.random.default_rng(seed).standard_normal(output_shape(cfg))
    return bf16_to_f32(bf16_round(dy)).astype(np.float64) if cfg.y_dtype == L.VDN_BF16 else \
        dy.astype(np.float32).astype(np.float64)


def _lin_slot(cfg: L.HybridCfg, dy: np.ndarray) -> np.ndarray:
    return dy[..., 1, :] if cfg.out_mode == 0 else dy


def _rel(got, ref):
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.max(np.abs(got - ref))
    return float(err / rms) if rms > 0 else (0.0 if err == 0 else float("inf"))


def _run(shape: Shape, dtype: str, seed: int, rms=True, fwd_init=False, **kw):
    inp = make_inputs(shape, seed, dtype)
    r = np.random.default_rng(seed + 7)
    if rms:
        inp["rms_weight"] = (1 + 0.3 * r.standard_normal((shape.H, shape.d_v))).astype(np.float32).astype(np.float64)
    if fwd_init:
        inp["fwd_init"] = (0.3 * r.standard_normal((shape.B, shape.H, shape.d_v, shape.d_k))).astype(
            np.float32).astype(np.float64)
    cfg = cfg_for(shape, dtype, **kw)
    t = to_torch(inp, dtype, "cuda")
    ha = HybridAttention(cfg)
    ha(t)
    dy = _dy(cfg, seed + 11)
    tdt = torch.bfloat16 if cfg.y_dtype == L.VDN_BF16 else torch.float32
    dyt = torch.from_numpy(dy.astype(np.float32)).to(tdt).cuda()
    g = ha.linear_backward(t, dyt, want_rms=True, want_fwd_init=True)
    torch.cuda.synchronize()
    ref = OG.linear_branch_grads(inp, _ocfg(cfg), _lin_slot(cfg, dy))
    return cfg, g, ref


CASES = [
    # (shape, dtype, options): fp32 SIMT forward at d = 32 with text and anchors;
    # d = 64 with a short last chunk, three token tiles (ragged), no anchors,
    # summed output and no RMS weight; bf16 d = 128 (tensor-core forward, the
    # B-form write slot) with a bf16 y and a carried forward state; bf16 d = 64
    # (tensor-core Gram, C-form write slot); fp32 d = 128 with a forward state.
    (Shape(B=1, T=12, N=37, H=2, d_k=32, d_v=32, L=3), "f32", dict()),
    (Shape(B=1, T=23, N=70, H=2, d_k=64, d_v=64, L=5), "f32", dict(anchors=0, out_mode=1, rms=False)),
    (Shape(B=1, T=12, N=40, H=2, d_k=128, d_v=128, L=8), "bf16", dict(y_dtype=L.VDN_BF16, fwd_init=True)),
    (Shape(B=2, T=15, N=33, H=3, d_k=64, d_v=64, L=4), "bf16", dict()),
    (Shape(B=1, T=10, N=20, H=1, d_k=128, d_v=128, L=0), "f32", dict(fwd_init=True)),
    # bf16 d = 128 with a summed output: the tensor-core read backward reads dy itself
    (Shape(B=1, T=16, N=150, H=2, d_k=128, d_v=128, L=6), "bf16", dict(out_mode=1)),
]


@pytest.mark.parametrize("shape,dtype,opts", CASES)
def test_lin_bwd_matches_oracle(shape, dtype, opts):
    opts = dict(opts)
    rms, fwd = opts.pop("rms", True), opts.pop("fwd_init", False)
    cfg, g, ref = _run(shape, dtype, seed=31, rms=rms, fwd_init=fwd, **opts)
    errs = {}
    for name in NAMES:
        key = "d" + name if name != "gate_lin" else "dgate_lin"
        if name not in ref:
            continue
        got = g[key].cpu().numpy().astype(np.float64)
        errs[name] = _rel(got, ref[name])
    print("relative errors:", {k: f"{v:.2e}" for k, v in errs.items()})
    for name, e in errs.items():
        assert e <= TOL[dtype], (name, e)
    # anchor frames are not written: exact zeros
    if cfg.anchors:
        for key in ("dk", "dv", "dbeta"):
            assert torch.all(g[key][:, 0] == 0) and torch.all(g[key][:, -1] == 0)
        assert torch.all(g["dalpha"][:, 0] == 0) and torch.all(g["dalpha"][:, -1] == 0)


def test_lin_bwd_rms_weight_gradient_at_ones():
    """Without an RMS weight the call still returns the gradient at weight = 1,
    which the oracle gives when it is handed explicit ones."""
    shape = Shape(B=1, T=12, N=25, H=2, d_k=32, d_v=32, L=3)
    inp = make_inputs(shape, 41, "f32")
    cfg = cfg_for(shape, "f32")
    t = to_torch(inp, "f32", "cuda")
    ha = HybridAttention(cfg)
    ha(t)
    dy = _dy(cfg, 42)
    g = ha.linear_backward(t, torch.from_numpy(dy.astype(np.float32)).cuda(), want_rms=True)
    torch.cuda.synchronize()
    inp1 = dict(inp)
    inp1["rms_weight"] = np.ones((2, 32))
    ref = OG.linear_branch_grads(inp1, _ocfg(cfg), dy[..., 1, :])
    assert _rel(g["drms_weight"].cpu().numpy(), ref["rms_weight"]) <= TOL["f32"]
    assert _rel(g["dq"].cpu().numpy(), ref["q"]) <= TOL["f32"]


def test_lin_bwd_repeatable():
    """Two backward calls on the same forward workspace give the same bits
    (no state carried between calls, no atomics)."""
    shape = Shape(B=1, T=12, N=40, H=2, d_k=128, d_v=128, L=8)
    inp = make_inputs(shape, 51, "bf16")
    cfg = cfg_for(shape, "bf16")
    t = to_torch(inp, "bf16", "cuda")
    ha = HybridAttention(cfg)
    ha(t)
    dyt = torch.from_numpy(_dy(cfg, 52).astype(np.float32)).cuda()
    g1 = {k: v.clone() for k, v in ha.linear_backward(t, dyt, want_rms=True, want_fwd_init=True).items()}
    g2 = ha.linear_backward(t, dyt, want_rms=True, want_fwd_init=True)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_lin_bwd_full_size_one_head():
    """At the 768p size (B=1, T=90, N=1008, H=24, d=128, L=512, bf16, inputs
    drawn on the device as the benchmark does): every gradient of one head
    against the oracle run on that head alone (the heads of the linear branch
    are independent)."""
    from video_diffusion_hybrid_b200.synth import head_slice, make_inputs_torch
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    w = WORKLOADS["768p"]
    s = w.shape
    t = make_inputs_torch(s, w.seed, w.dtype, "cuda")
    cfg = cfg_for(s, w.dtype)
    ha = HybridAttention(cfg)
    ha(t)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    dy = torch.randn(output_shape(cfg), generator=gen, device="cuda")
    g = ha.linear_backward(t, dy)
    torch.cuda.synchronize()
    h = s.H - 1
    inp = {k: v.astype(np.float64) for k, v in head_slice(t, 0, h).items()}
    oc = O.Cfg(B=1, T=s.T, N=s.N, H=1, d_k=s.d_k, d_v=s.d_v, L=s.L)
    ref = OG.linear_branch_grads(inp, oc, dy[0:1, :, :, h:h + 1, 1].double().cpu().numpy())
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("gate_lin", "dgate_lin")):
        got = g[key][0:1, :, :, h:h + 1].double().cpu().numpy()
        e = _rel(got, ref[name])
        print(name, f"{e:.2e}")
        assert e <= TOL["bf16"], (name, e)
    e = _rel(g["dalpha"][0:1, :, h:h + 1].double().cpu().numpy(), ref["alpha"])
    assert e <= TOL["bf16"], ("alpha", e)
    del t, g, ha, dy
    torch.cuda.empty_cache()


# ------------------------------------------------------------ softmax branch
SM_CASES = [
    # SIMT fp32 path: fp32 d = 32 with anchors; fp32 d = 64 without anchors, a
    # short last chunk, ragged 64-row tiles, summed output and a large scale
    # (the max subtraction matters); bf16 d = 32 with a summed output.
    # Tensor-core path (bf16, d = 64 or 128): d = 128 with a bf16 y; d = 64 with
    # two batch elements; d = 128 with ragged 128-row tiles over several frames,
    # no anchors and scale 10; d = 128 with N < 128 and a summed output.
    (Shape(B=1, T=12, N=37, H=2, d_k=32, d_v=32, L=0), "f32", dict()),
    (Shape(B=1, T=23, N=70, H=2, d_k=64, d_v=64, L=0), "f32", dict(anchors=0, out_mode=1, softmax_scale=10.0)),
    (Shape(B=1, T=12, N=40, H=2, d_k=32, d_v=32, L=0), "bf16", dict(out_mode=1)),
    (Shape(B=1, T=12, N=40, H=2, d_k=128, d_v=128, L=0), "bf16", dict(y_dtype=L.VDN_BF16)),
    (Shape(B=2, T=15, N=33, H=3, d_k=64, d_v=64, L=0), "bf16", dict()),
    (Shape(B=1, T=23, N=300, H=2, d_k=128, d_v=128, L=0), "bf16", dict(anchors=0, softmax_scale=10.0)),
    (Shape(B=1, T=20, N=100, H=3, d_k=128, d_v=128, L=0), "bf16", dict(out_mode=1)),
]


def _sm_slot(cfg, dy):
    return dy[..., 0, :] if cfg.out_mode == 0 else dy


@pytest.mark.parametrize("shape,dtype,opts", SM_CASES)
def test_sm_bwd_matches_oracle(shape, dtype, opts):
    inp = make_inputs(shape, 61, dtype)
    cfg = cfg_for(shape, dtype, **opts)
    t = to_torch(inp, dtype, "cuda")
    ha = HybridAttention(cfg)
    tc = dtype == "bf16" and shape.d_k in (64, 128)
    assert L.vdn_hybrid_stage_impl(cfg, L.STAGE_SOFTMAX_BWD) == (1 if tc else 0)
    dy = _dy(cfg, 62)
    tdt = torch.bfloat16 if cfg.y_dtype == L.VDN_BF16 else torch.float32
    g = ha.softmax_backward(t, torch.from_numpy(dy.astype(np.float32)).to(tdt).cuda())
    torch.cuda.synchronize()
    assert ha.softmax_backward_status()[0] == L.VDN_OK
    ref = OG.softmax_branch_grads(inp, _ocfg(cfg), _sm_slot(cfg, dy))
    errs = {n: _rel(g["d" + n].cpu().numpy().astype(np.float64), ref[n]) for n in ("q", "k", "v", "gate_sm")}
    print("relative errors:", {k: f"{v:.2e}" for k, v in errs.items()})
    for n, e in errs.items():
        assert e <= TOL[dtype], (n, e)


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128)])
def test_whole_core_backward_is_the_sum_of_the_branches(dtype, d):
    """vdn_hybrid_bwd (HybridAttention.backward, one library call): dq, dk, dv
    of the core equal the two oracles' branch gradients added, the gate
    gradients are each branch's own; and the one call equals the two branch
    entry points' outputs added, bit for bit (the linear branch adds its share
    in fp32 to what the softmax branch wrote).  fp32 d = 64 runs the SIMT
    kernels, bf16 d = 128 the tensor-core ones (with an RMS weight and a
    carried forward state)."""
    shape = Shape(B=1, T=12, N=30, H=2, d_k=d, d_v=d, L=4)
    inp = make_inputs(shape, 71, dtype)
    if dtype == "bf16":
        r = np.random.default_rng(73)
        inp["rms_weight"] = (1 + 0.2 * r.standard_normal((2, d))).astype(np.float32)
        inp["fwd_init"] = (0.1 * r.standard_normal((1, 2, d, d))).astype(np.float32)
    cfg = cfg_for(shape, dtype)
    t = to_torch(inp, dtype, "cuda")
    for k in ("rms_weight", "fwd_init"):
        if k in inp:
            t[k] = torch.from_numpy(inp[k]).cuda()
    ha = HybridAttention(cfg)
    ha(t)
    dy = _dy(cfg, 72)
    dyt = torch.from_numpy(dy.astype(np.float32)).cuda()
    g = {k: v.clone() for k, v in ha.backward(t, dyt).items()}
    torch.cuda.synchronize()
    assert ha.backward_status()[0] == L.VDN_OK
    oc = _ocfg(cfg)
    rl = OG.linear_branch_grads(inp, oc, dy[..., 1, :])
    rs = OG.softmax_branch_grads(inp, oc, dy[..., 0, :])
    for n in ("q", "k", "v"):
        assert _rel(g["d" + n].cpu().numpy(), rl[n] + rs[n]) <= TOL[dtype], n
    assert _rel(g["dgate_sm"].cpu().numpy(), rs["gate_sm"]) <= TOL[dtype]
    assert _rel(g["dgate_lin"].cpu().numpy(), rl["gate_lin"]) <= TOL[dtype]
    assert _rel(g["dbeta"].cpu().numpy(), rl["beta"]) <= TOL[dtype]
    lin = ha.linear_backward(t, dyt, want_rms="rms_weight" in t, want_fwd_init="fwd_init" in t)
    sm = ha.softmax_backward(t, dyt)
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv"):
        assert torch.equal(g[n], lin[n] + sm[n]), n
    for n in ("dbeta", "dalpha", "dgate_lin", "drms_weight", "dfwd_init"):
        if n in lin:
            assert torch.equal(g[n], lin[n]), n
    assert torch.equal(g["dgate_sm"], sm["dgate_sm"])


def test_sm_bwd_full_size_one_key_frame():
    """At the 768p size (inputs drawn on the device): for one head and key
    frame f = 47, the oracle, one query frame at a time, over every query frame
    that sees f (its chunk and the two neighbours, and the two anchor frames,
    which see every key): dk, dv of frame f's tokens and dq, dgate_sm of those
    query frames."""
    from video_diffusion_hybrid_b200.synth import head_slice, make_inputs_torch
    from video_diffusion_hybrid_b200.workloads import WORKLOADS
    w = WORKLOADS["768p"]
    s = w.shape
    t = make_inputs_torch(s, w.seed, w.dtype, "cuda")
    cfg = cfg_for(s, w.dtype)
    ha = HybridAttention(cfg)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6)
    dy = torch.randn(output_shape(cfg), generator=gen, device="cuda")
    assert L.vdn_hybrid_stage_impl(cfg, L.STAGE_SOFTMAX_BWD) == 1
    g = ha.softmax_backward(t, dy)
    torch.cuda.synchronize()
    assert ha.softmax_backward_status()[0] == L.VDN_OK
    h, f = 3, 47
    frames = np.flatnonzero(O.frame_mask(s.T, 5, 4)[f])
    inp = {k: v.astype(np.float64) for k, v in head_slice(t, 0, h).items()}
    oc = O.Cfg(B=1, T=s.T, N=s.N, H=1, d_k=s.d_k, d_v=s.d_v, L=0)
    dyh = dy[0:1, :, :, h:h + 1, 0].double().cpu().numpy()
    ref = OG.softmax_branch_grads_frames(inp, oc, dyh, 0, 0, frames)
    pick = lambda key, fr: g[key][0:1, fr, :, h:h + 1].double().cpu().numpy()
    for n in ("k", "v"):
        e = _rel(pick("d" + n, [f]), ref[n][:, [f]])
        print(n, f"{e:.2e}")
        assert e <= TOL["bf16"], (n, e)
    for n in ("q", "gate_sm"):
        e = _rel(pick("d" + n, frames), ref[n][:, frames])
        print(n, f"{e:.2e}")
        assert e <= TOL["bf16"], (n, e)
    del t, g, ha, dy
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 64), ("bf16", 128)])
def test_forward_softmax_lse_matches_oracle(dtype, d):
    """The forward's optional log-sum-exp output (args.sm_lse) against the
    oracle's. fp32 (SIMT): 1e-5 absolute. bf16 (tensor cores): the row sum adds
    bf16-rounded weights (each within 2^-9 relative), so the log is within
    about 2^-9; the bar is 2^-7."""
    shape = Shape(B=1, T=12, N=40, H=2, d_k=d, d_v=d, L=0)
    inp = make_inputs(shape, 81, dtype)
    cfg = cfg_for(shape, dtype, softmax_scale=3.0)
    t = to_torch(inp, dtype, "cuda")
    ha = HybridAttention(cfg, keep_lse=True)
    ha(t)
    torch.cuda.synchronize()
    err = np.max(np.abs(ha.sm_lse.cpu().numpy() - O.softmax_lse(inp, _ocfg(cfg))))
    print("lse max abs error", err)
    assert err <= (1e-5 if dtype == "f32" else 2.0 ** -7)


@pytest.mark.parametrize("shape,opts", [
    (Shape(B=1, T=12, N=40, H=2, d_k=128, d_v=128, L=0), dict(y_dtype=L.VDN_BF16)),
    (Shape(B=2, T=15, N=33, H=3, d_k=64, d_v=64, L=0), dict()),
    (Shape(B=1, T=23, N=300, H=2, d_k=128, d_v=128, L=0), dict(anchors=0, softmax_scale=10.0)),
])
def test_sm_bwd_with_forward_lse_matches_oracle(shape, opts):
    """The tensor-core softmax backward given the forward's log-sum-exp (no
    row-max pass): the same bar as without, and close to the result without."""
    inp = make_inputs(shape, 61, "bf16")
    cfg = cfg_for(shape, "bf16", **opts)
    t = to_torch(inp, "bf16", "cuda")
    dy = _dy(cfg, 62)
    tdt = torch.bfloat16 if cfg.y_dtype == L.VDN_BF16 else torch.float32
    dyt = torch.from_numpy(dy.astype(np.float32)).to(tdt).cuda()
    ha = HybridAttention(cfg, keep_lse=True)
    ha(t)
    g = {k: v.clone() for k, v in ha.softmax_backward(t, dyt).items()}
    torch.cuda.synchronize()
    assert ha.softmax_backward_status()[0] == L.VDN_OK
    plain = HybridAttention(cfg).softmax_backward(t, dyt)
    torch.cuda.synchronize()
    ref = OG.softmax_branch_grads(inp, _ocfg(cfg), _sm_slot(cfg, dy))
    for n in ("q", "k", "v", "gate_sm"):
        got = g["d" + n].cpu().numpy().astype(np.float64)
        e = _rel(got, ref[n])
        e2 = _rel(got, plain["d" + n].cpu().numpy().astype(np.float64))
        print(n, f"{e:.2e} (vs without: {e2:.2e})")
        assert e <= TOL["bf16"], (n, e)

"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Bar (element by element, per output slot): max |y_gpu - y_oracle| <= tol *
RMS(y_oracle slot), tol = 1e-4 in fp32 mode and 2e-2 in bf16-input /
fp32-accumulate mode.
"""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O
from video_diffusion_hybrid_b200 import _lib as L
from video_diffusion_hybrid_b200.api import HybridAttention, cfg_for, to_torch
from video_diffusion_hybrid_b200.build import build
from video_diffusion_hybrid_b200.synth import Shape, make_inputs
from video_diffusion_hybrid_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    build()


def ocfg(cfg: L.HybridCfg) -> O.Cfg:
    return O.Cfg(B=cfg.B, T=cfg.T, N=cfg.N, H=cfg.H, d_k=cfg.d_k, d_v=cfg.d_v, L=cfg.L, chunk=cfg.chunk,
                 anchors=cfg.anchors, softmax_scale=cfg.softmax_scale, rms_eps=cfg.rms_eps or 1e-6,
                 out_mode=cfg.out_mode, update=cfg.update)


def run(shape: Shape, dtype: str, seed: int, extra=None, drop_text=False, stages=L.STAGE_ALL, **kw):
    inp = make_inputs(shape, seed, dtype)
    if drop_text:
        for k in ("text_k", "text_v", "text_beta", "text_k_bits", "text_v_bits"):
            inp.pop(k, None)
    if extra:
        inp.update(extra)
    cfg = cfg_for(shape, dtype, **kw)
    if drop_text:
        cfg.L = 0
    t = to_torch(inp, dtype, "cuda")
    ha = HybridAttention(cfg)
    y = ha(t, stages=stages)
    torch.cuda.synchronize()
    st, where = L.vdn_hybrid_device_status(cfg, ha.args(t))
    assert st == L.VDN_OK, where
    return inp, cfg, ha, t, y.float().cpu().numpy().astype(np.float64)


VDA = L.STAGE_TEXT | L.STAGE_SOLVE | L.STAGE_SCAN | L.STAGE_READ


def rel_err(got, ref, allowance=None):
    """max |got - ref| / RMS(ref).  A slot that is exactly zero in the oracle
    (no state to read) must be exactly zero.  `allowance` (per element) is the
    rounding of a bf16 store, taken off before the comparison."""
    rms = np.sqrt(np.mean(ref ** 2))
    diff = np.abs(got - ref)
    if allowance is not None:
        diff = np.maximum(diff - allowance, 0.0)
    if rms == 0:
        return 0.0 if np.max(diff) == 0 else float("inf")
    return float(np.max(diff) / rms)


U_BF16 = 2.0 ** -8 * (1 + 1e-3)  # bf16 keeps 8 significant bits: half an ulp <= 2^-8 |y|


def check(got, ref_slots, cfg, dtype):
    """ref_slots: the oracle's [..., 2, d_v] output (slot 0 softmax, 1 linear)."""
    tol = TOL[dtype]
    sb = cfg.y_dtype == L.VDN_BF16
    if cfg.out_mode == 0:
        for s, name in ((0, "softmax"), (1, "linear")):
            ref = ref_slots[..., s, :]
            e = rel_err(got[..., s, :], ref, U_BF16 * np.abs(ref) if sb else None)
            assert e <= tol, f"{name} slot: max err {e:.3g} x RMS > {tol}"
    else:
        ref = ref_slots.sum(axis=-2)
        # summed bf16 output is rounded twice: the softmax slot, then the sum
        allow = U_BF16 * (np.abs(ref_slots[..., 0, :]) + np.abs(ref)) if sb else None
        e = rel_err(got, ref, allow)
        assert e <= tol, f"summed output: max err {e:.3g} x RMS > {tol}"


def oracle(inp, cfg):
    oc = ocfg(cfg)
    return O.hybrid_attn(inp, O.Cfg(**{**oc.__dict__, "out_mode": 0}))


@pytest.mark.parametrize("name", ["tiny", "tiny_scan", "small"])
def test_workload_full_parity(name):
    w = WORKLOADS[name]
    inp, cfg, _, _, y = run(w.shape, w.dtype, w.seed)
    check(y, oracle(inp, cfg), cfg, w.dtype)


CASES = {
    "d128": (Shape(1, 15, 40, 2, 128, 128, 16), {}),
    "d64_ragged_N": (Shape(1, 20, 17, 3, 64, 64, 5), {}),
    "no_anchors": (Shape(1, 25, 12, 2, 32, 32, 4), dict(anchors=0)),
    "partial_chunk_T23": (Shape(1, 23, 9, 2, 64, 64, 3), {}),
    "T2_all_anchor": (Shape(1, 2, 33, 2, 32, 32, 3), {}),
    "T7": (Shape(1, 7, 20, 1, 64, 64, 0), {}),
    "batch2": (Shape(2, 15, 24, 2, 64, 64, 6), {}),
    "scale10": (Shape(1, 20, 16, 2, 64, 64, 8), dict(softmax_scale=10.0)),
    "summed_out": (Shape(1, 20, 16, 2, 64, 64, 8), dict(out_mode=1)),
    "eps": (Shape(1, 10, 8, 2, 32, 32, 4), dict(rms_eps=0.5)),
    "y_bf16": (Shape(1, 20, 24, 2, 64, 64, 8), dict(y_dtype=L.VDN_BF16)),
    "y_bf16_summed": (Shape(1, 20, 24, 2, 64, 64, 8), dict(y_dtype=L.VDN_BF16, out_mode=1)),
    "d128_ragged_keys": (Shape(1, 30, 130, 1, 128, 128, 4), {}),
    "d128_scale40_rescale": (Shape(1, 25, 70, 2, 128, 128, 4), dict(softmax_scale=40.0)),
    "d64_scale40_no_anchor": (Shape(1, 25, 70, 2, 64, 64, 4), dict(softmax_scale=40.0, anchors=0)),
    # d = 128 scans with no written frame and with one (both ends anchors)
    "d128_T2_all_anchor": (Shape(1, 2, 40, 2, 128, 128, 4), {}),
    "d128_T3_one_written": (Shape(1, 3, 40, 3, 128, 128, 4), {}),
}


def test_bf16_softmax_runs_on_tensor_cores():
    """bf16 with d in {64, 128} takes the tcgen05 kernel, others the SIMT one."""
    for d in (64, 128):
        assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, d, d, 0), "bf16"), L.STAGE_SOFTMAX) == 1
    assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, 32, 32, 0), "bf16"), L.STAGE_SOFTMAX) == 0
    assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, 128, 128, 0), "f32"), L.STAGE_SOFTMAX) == 0
    for d in (64, 128):
        assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, d, d, 0), "bf16"), L.STAGE_READ) == 1
        assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, d, d, 0), "bf16"), L.STAGE_SOLVE) == 1
    assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, 64, 64, 0), "f32"), L.STAGE_READ) == 0
    assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, 128, 128, 0), "bf16"), L.STAGE_SCAN) == 1
    assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, 64, 64, 0), "bf16"), L.STAGE_SCAN) == 0
    assert L.vdn_hybrid_stage_impl(cfg_for(Shape(1, 10, 16, 2, 128, 128, 0), "f32"), L.STAGE_SCAN) == 0


@pytest.mark.parametrize("shape", [Shape(1, 20, 240, 2, 64, 64, 8), Shape(1, 12, 300, 2, 128, 128, 8),
                                   Shape(2, 8, 40, 1, 128, 128, 0)])
def test_bf16_frame_maps_match_oracle(shape):
    """M_t, C_t and the half-text state after the tensor-core Gram + SPD
    solve (bf16 inputs)."""
    inp, cfg, ha, _, _ = run(shape, "bf16", 13, drop_text=shape.L == 0)
    it = {k: v.double().cpu().numpy() for k, v in ha.intermediates().items()}
    for b in range(cfg.B):
        for h in range(cfg.H):
            ref = O.vda_intermediates(inp, ocfg(cfg), b, h)
            sx = np.abs(ref["S_init"]).max() + 1e-30
            np.testing.assert_allclose(it["half_text"][b, h], ref["S_init"], atol=2e-5 * sx)
            # the tensor-core scan (d = 128) steps S <- (alpha S + B_t) M_t: the C_t slot keeps B_t
            bform = L.vdn_hybrid_stage_impl(cfg, L.STAGE_SCAN) == 1
            for t in range(1, cfg.T - 1):
                np.testing.assert_allclose(it["M"][b, t, h], ref["M"][t], atol=2e-5)
                cref = O.gram_write(np.asarray(inp["k"][b, t, :, h], np.float64), np.asarray(inp["v"][b, t, :, h], np.float64),
                                    np.asarray(inp["beta"][b, t, :, h], np.float64))[1] if bform else ref["C"][t]
                np.testing.assert_allclose(it["C"][b, t, h], cref, atol=2e-5 * np.abs(cref).max())


@pytest.mark.parametrize("shape", [Shape(1, 12, 96, 2, 256, 256, 16), Shape(1, 10, 40, 1, 256, 256, 0)])
def test_d256_vda_matches_oracle(shape):
    """d = 256, the Video Delta Attention stages (the only ones at this size):
    M_t, B_t (the scan steps S <- (alpha S + B_t) M_t, so the C_t slot keeps
    B_t) and S_x / 2 after the block-mode Gram and the block solve, the
    read table after the chunked scans, and the linear slot of every output
    after the chunked read, against the oracle."""
    inp, cfg, ha, t, y = run(shape, "bf16", 21, drop_text=shape.L == 0, stages=VDA)
    it = {k: v.double().cpu().numpy() for k, v in ha.intermediates().items()}
    for b in range(cfg.B):
        for h in range(cfg.H):
            ref = O.vda_intermediates(inp, ocfg(cfg), b, h)
            sx = np.abs(ref["S_init"]).max() + 1e-30
            np.testing.assert_allclose(it["half_text"][b, h], ref["S_init"], atol=2e-5 * sx)
            for f in range(1, cfg.T - 1):
                np.testing.assert_allclose(it["M"][b, f, h], ref["M"][f], atol=2e-5)
                Bf = O.gram_write(np.asarray(inp["k"][b, f, :, h], np.float64),
                                  np.asarray(inp["v"][b, f, :, h], np.float64),
                                  np.asarray(inp["beta"][b, f, :, h], np.float64))[1]
                np.testing.assert_allclose(it["C"][b, f, h], Bf, atol=2e-5 * np.abs(Bf).max())
            # the tensor-core scan's three-term bf16 split leaves about 2^-18 relative per
            # product term and a step sums d of them: the bar of the d = 128 read table,
            # 1e-4 * RMS, scaled by d / 128
            np.testing.assert_allclose(it["R"][b, h], ref["R"], atol=2e-4 * np.sqrt(np.mean(ref["R"] ** 2)) + 1e-30)
    ref_y = O.hybrid_attn(inp, ocfg(cfg))
    assert rel_err(y[..., 1, :], ref_y[..., 1, :]) <= TOL["bf16"]
    # the softmax stage has no kernel at this size: refused before any launch
    assert L.vdn_hybrid_attn_fwd(cfg, ha.args(t), check=False) == L.VDN_ERR_UNSUPPORTED


D256_EDGE = {
    # anchors at both ends: no written frame (the scans only copy the start state)
    "T2": (Shape(1, 2, 24, 1, 256, 256, 8), {}),
    # one written frame between the anchors
    "T3": (Shape(1, 3, 24, 1, 256, 256, 0), {}),
    # no anchors: every frame written, a ragged last chunk
    "T7_no_anchors": (Shape(1, 7, 16, 2, 256, 256, 8), {"anchors": 0}),
    # two batch elements: chains of both in one launch
    "B2": (Shape(2, 11, 20, 1, 256, 256, 8), {}),
}


@pytest.mark.parametrize("case", sorted(D256_EDGE))
def test_d256_edge_cases(case):
    """d = 256 with few or no written frames, no anchors and two batch
    elements (the tensor-core scan's empty, single-step and multi-chain
    forms): the read table and the linear slot against the oracle."""
    shape, kw = D256_EDGE[case]
    inp, cfg, ha, t, y = run(shape, "bf16", 29, drop_text=shape.L == 0, stages=VDA, **kw)
    it = {k: v.double().cpu().numpy() for k, v in ha.intermediates().items()}
    for b in range(cfg.B):
        for h in range(cfg.H):
            ref = O.vda_intermediates(inp, ocfg(cfg), b, h)
            np.testing.assert_allclose(it["R"][b, h], ref["R"], atol=2e-4 * np.sqrt(np.mean(ref["R"] ** 2)) + 1e-30)
    ref_y = O.hybrid_attn(inp, ocfg(cfg))
    assert rel_err(y[..., 1, :], ref_y[..., 1, :]) <= TOL["bf16"]


@pytest.mark.parametrize("y_bf16,out_mode", [(False, 1), (True, 0), (True, 1)])
def test_d256_output_options(y_bf16, out_mode):
    """d = 256 with a caller-given text state, an RMSNorm weight, bf16 y and
    the summed output: the linear branch (the only one at this size, added
    into a zeroed y when summed) against the oracle."""
    shape = Shape(1, 12, 48, 2, 256, 256, 0)
    r = np.random.default_rng(7)
    inp = make_inputs(shape, 11, "bf16")
    for k in ("text_k", "text_v", "text_beta", "text_k_bits", "text_v_bits"):
        inp.pop(k, None)
    inp["init_state"] = r.standard_normal((1, 2, 256, 256)).astype(np.float32) * 0.1
    inp["rms_weight"] = (1 + 0.5 * r.standard_normal((2, 256))).astype(np.float32)
    cfg = cfg_for(shape, "bf16", out_mode=out_mode, y_dtype=L.VDN_BF16 if y_bf16 else L.VDN_F32)
    cfg.L = 0
    t = to_torch(inp, "bf16", "cuda")
    ha = HybridAttention(cfg)
    ha.y.zero_()
    ha(t, stages=VDA)
    torch.cuda.synchronize()
    assert L.vdn_hybrid_device_status(cfg, ha.args(t))[0] == L.VDN_OK
    y = ha.y.float().cpu().numpy().astype(np.float64)
    ref = oracle(inp, cfg)[..., 1, :]
    got = y[..., 1, :] if out_mode == 0 else y
    assert rel_err(got, ref, U_BF16 * np.abs(ref) if y_bf16 else None) <= TOL["bf16"]


def test_bf16_read_table_matches_oracle():
    """The read table the tensor-core read consumes (fp32 copy), bf16 mode."""
    w = WORKLOADS["small"]
    inp, cfg, ha, _, _ = run(w.shape, w.dtype, w.seed)
    R = ha.intermediates()["R"].double().cpu().numpy()
    for h in (0, cfg.H - 1):
        ref = O.vda_intermediates(inp, ocfg(cfg), 0, h)["R"]
        np.testing.assert_allclose(R[0, h], ref, atol=1e-4 * np.sqrt(np.mean(ref ** 2)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", sorted(CASES))
def test_edge_case_parity(case, dtype):
    shape, kw = CASES[case]
    inp, cfg, _, _, y = run(shape, dtype, 7, **kw)
    check(y, oracle(inp, cfg), cfg, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_init_state_and_rms_weight(dtype):
    shape = Shape(1, 20, 16, 2, 64, 64, 0)
    r = np.random.default_rng(5)
    extra = {"init_state": r.standard_normal((1, 2, 64, 64)).astype(np.float32) * 0.3,
             "rms_weight": (1 + 0.5 * r.standard_normal((2, 64))).astype(np.float32)}
    inp, cfg, _, _, y = run(shape, dtype, 9, extra=extra, drop_text=True)
    check(y, oracle(inp, cfg), cfg, dtype)


def test_zero_text_state():
    inp, cfg, _, _, y = run(Shape(1, 20, 8, 2, 32, 32, 0), "f32", 3, drop_text=True)
    check(y, oracle(inp, cfg), cfg, "f32")


def test_intermediates_match_oracle():
    """Stage outputs in the workspace: text state, (M_t, C_t), snapshots, R."""
    w = WORKLOADS["tiny_scan"]
    inp, cfg, ha, _, _ = run(w.shape, "f32", w.seed)
    it = {k: v.double().cpu().numpy() for k, v in ha.intermediates().items()}
    oc = ocfg(cfg)
    for h in range(cfg.H):
        ref = O.vda_intermediates(inp, oc, 0, h)
        scale = np.sqrt(np.mean(ref["R"] ** 2))
        np.testing.assert_allclose(it["half_text"][0, h], ref["S_init"], atol=1e-5 * scale)
        for t in range(1, cfg.T - 1):
            np.testing.assert_allclose(it["M"][0, t, h], ref["M"][t], atol=1e-5)
            np.testing.assert_allclose(it["C"][0, t, h], ref["C"][t], atol=1e-5 * np.abs(ref["C"][t]).max())
        for j in range(cfg.C + 1):
            fj = min(5 * j, cfg.T)
            np.testing.assert_allclose(it["fwd_snap"][0, h, j], ref["F"][fj], atol=1e-5 * scale)
            np.testing.assert_allclose(it["bwd_snap"][0, h, j], ref["G"][fj], atol=1e-5 * scale)
        np.testing.assert_allclose(it["R"][0, h], ref["R"], atol=1e-5 * scale)


@pytest.mark.parametrize("shape", [Shape(1, 22, 48, 2, 128, 128, 4), Shape(2, 40, 24, 1, 128, 128, 0)])
def test_chunk_maps_match_oracle(shape):
    """The composed chunk maps of the chunk-stepped scan (P_c from its bf16
    split, the two Horner constants, Lam_c) against the oracle's chunk_maps
    on the same frames; chunk 0 and the last chunk hold an anchor frame."""
    inp, cfg, ha, _, _ = run(shape, "bf16", 5)
    assert cfg.C >= 4  # the chunk-stepped scan runs
    cm = {k: v.double().cpu().numpy() for k, v in ha.chunk_maps().items()}
    for b in range(cfg.B):
        for h in range(cfg.H):
            f64 = lambda a: np.asarray(a, np.float64)
            P, Cf, Cb, Lam = O.chunk_maps(f64(inp["k"][b, :, :, h]), f64(inp["v"][b, :, :, h]),
                                          f64(inp["beta"][b, :, :, h]), f64(inp["alpha"][b, :, h]),
                                          chunk=cfg.chunk, anchors=cfg.anchors)
            for c in range(cfg.C):
                np.testing.assert_allclose(cm["P"][b, c, h], P[c], rtol=0, atol=2e-4 * np.abs(P[c]).max())
                sc = np.abs(Cf[c]).max()
                np.testing.assert_allclose(cm["Cf"][b, c, h], Cf[c], rtol=0, atol=2e-4 * sc)
                np.testing.assert_allclose(cm["Cb"][b, c, h], Cb[c], rtol=0, atol=2e-4 * np.abs(Cb[c]).max())
                np.testing.assert_allclose(cm["Lam"][b, c, h], Lam[c], rtol=1e-6)


@pytest.mark.parametrize("scan_mode", [1, 2])
def test_scan_modes_match_oracle(scan_mode):
    """The tensor-core scan stepped by frames (1) and by composed chunk maps
    (2) on the same inputs: both reach the oracle's output, and their
    chunk-boundary states agree with the oracle's frame scan."""
    shape = Shape(1, 30, 40, 3, 128, 128, 4)
    inp, cfg, ha, _, y = run(shape, "bf16", 13, scan_mode=scan_mode)
    check(y, oracle(inp, cfg), cfg, "bf16")
    it = {k: v.double().cpu().numpy() for k, v in ha.intermediates().items()}
    for h in range(cfg.H):
        ref = O.vda_intermediates(inp, ocfg(cfg), 0, h)
        scale = np.sqrt(np.mean(ref["R"] ** 2))
        for j in range(cfg.C + 1):
            fj = min(5 * j, cfg.T)
            # M_t, C_t carry ~2e-5 relative error (bf16-mode Gram, fp32 solve) and each
            # step's split keeps ~16 bits; over <= 28 non-expansive steps: < 1e-3
            np.testing.assert_allclose(it["fwd_snap"][0, h, j], ref["F"][fj], atol=1e-3 * scale)
            np.testing.assert_allclose(it["bwd_snap"][0, h, j], ref["G"][fj], atol=1e-3 * scale)


def test_stages_compose_to_full_call_and_are_deterministic():
    w = WORKLOADS["small"]
    inp, cfg, ha, t, y = run(w.shape, w.dtype, w.seed)
    y2 = ha(t).float().cpu().numpy()
    assert np.array_equal(y, y2)
    ha.y.zero_()
    for st in (L.STAGE_TEXT, L.STAGE_SOLVE, L.STAGE_SCAN, L.STAGE_SOFTMAX, L.STAGE_READ):
        ha(t, stages=st)
    torch.cuda.synchronize()
    assert np.array_equal(y, ha.y.float().cpu().numpy())


@pytest.mark.parametrize("d", [128, 256])
def test_text_stage_beside_frame_write_is_exact(d):
    """A problem large enough (B*T*H >= 1024, text tokens present) that one
    call runs the text stage on a stream of its own beside the frame write:
    the result must equal, bit for bit, the stages called one at a time (the
    text stage alone never forks), over the VDA stages and at d = 128 the
    whole core too."""
    shape = Shape(1, 45, 16, 24, d, d, 8)
    assert shape.B * shape.T * shape.H >= 1024
    stages = L.STAGE_ALL if d == 128 else VDA
    inp, cfg, ha, t, y = run(shape, "bf16", 41, stages=stages)
    ha.y.zero_()
    for st in (L.STAGE_TEXT, L.STAGE_SOLVE, L.STAGE_SCAN, L.STAGE_SOFTMAX, L.STAGE_READ):
        if st & stages:
            ha(t, stages=st)
    torch.cuda.synchronize()
    y2 = ha.y.float().cpu().numpy()
    if d == 128:
        assert np.array_equal(y, y2)
    else:
        # the VDA stages write the linear slot only (slot 0 is left as it was)
        assert np.array_equal(y[..., 1, :], y2[..., 1, :])
    # and the linear slot against the oracle
    ref = O.hybrid_attn(inp, ocfg(cfg))
    assert rel_err(y[..., 1, :], ref[..., 1, :]) <= TOL["bf16"]


def _sample_rows(cfg, heads, per_head, rng):
    T, N = cfg.T, cfg.N
    rows = []
    for b in range(cfg.B):
        for h in heads:
            frames = [0, 1, 4, 5, 9, 10, T // 2, T - 6, T - 5, T - 2, T - 1]
            for t in frames:
                for n in (0, N - 1, int(rng.integers(N))):
                    rows.append((b, t, n, h))
            for _ in range(per_head):
                rows.append((b, int(rng.integers(T)), int(rng.integers(N)), h))
    return rows


@pytest.mark.parametrize("name", ["768p", "long"])
def test_full_size_sampled_parity(name):
    """At the benchmark's size and launch configuration (inputs drawn on the
    device), and at the long-video size (T=180, two batch elements with their
    own seeds): sampled outputs against the oracle evaluated position by
    position on a head of the first and of the last batch element."""
    from video_diffusion_hybrid_b200.synth import head_slice, make_inputs_torch
    w = WORKLOADS[name]
    t = make_inputs_torch(w.shape, w.seed, w.dtype, "cuda")
    cfg = cfg_for(w.shape, w.dtype)
    ha = HybridAttention(cfg)
    y = ha(t)
    torch.cuda.synchronize()
    assert L.vdn_hybrid_device_status(cfg, ha.args(t))[0] == L.VDN_OK
    assert bool(torch.isfinite(y).all())
    rng = np.random.default_rng(0)
    s = w.shape
    for b, h in ((0, 0), (s.B - 1, s.H - 1)):
        inp = head_slice(t, b, h)
        oc = O.Cfg(B=1, T=s.T, N=s.N, H=1, d_k=s.d_k, d_v=s.d_v, L=s.L)
        rows = _sample_rows(oc, heads=(0,), per_head=24, rng=rng)
        ref = O.hybrid_attn_rows(inp, oc, rows)
        idx = torch.tensor([(t_, n) for (_, t_, n, _) in rows], device=y.device)
        got = y[b, idx[:, 0], idx[:, 1], h].float().cpu().numpy()
        for sl in (0, 1):
            rms = np.sqrt(np.mean(ref[:, sl] ** 2))
            err = np.max(np.abs(got[:, sl] - ref[:, sl])) / rms
            assert err <= TOL[w.dtype], (b, h, sl, err)
    del t, y, ha
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["sweep_N256_d64", "sweep_N1008_d64", "sweep_N4032_d64", "sweep_N256_d128",
                                  "sweep_N4032_d128", "sweep_N256_d256", "sweep_N1008_d256", "sweep_N4032_d256"])
def test_vda_sweep_sampled_parity(name):
    """The VDA-only sweep shapes (T=90, H=24): the four VDA stages alone
    (text, frame write + solve, scans, read), the linear slot of sampled
    outputs against the oracle on two heads."""
    from video_diffusion_hybrid_b200.synth import head_slice, make_inputs_torch
    w = WORKLOADS[name]
    t = make_inputs_torch(w.shape, w.seed, w.dtype, "cuda")
    cfg = cfg_for(w.shape, w.dtype)
    ha = HybridAttention(cfg)
    vda = L.STAGE_TEXT | L.STAGE_SOLVE | L.STAGE_SCAN | L.STAGE_READ
    y = ha(t, stages=vda)
    torch.cuda.synchronize()
    assert L.vdn_hybrid_device_status(cfg, ha.args(t))[0] == L.VDN_OK
    rng = np.random.default_rng(1)
    s = w.shape
    for h in (0, s.H - 1):
        inp = head_slice(t, 0, h)
        oc = O.Cfg(B=1, T=s.T, N=s.N, H=1, d_k=s.d_k, d_v=s.d_v, L=s.L)
        rows = _sample_rows(oc, heads=(0,), per_head=24, rng=rng)
        ref = O.hybrid_attn_rows(inp, oc, rows)[:, 1]
        idx = torch.tensor([(t_, n) for (_, t_, n, _) in rows], device=y.device)
        got = y[0, idx[:, 0], idx[:, 1], h, 1].float().cpu().numpy()
        err = np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref ** 2))
        assert err <= TOL[w.dtype], (h, err)
    del t, y, ha
    torch.cuda.empty_cache()


# ------------------------------------------------------------ output projection
def _bf16_tensor(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("out_dtype", [L.VDN_F32, L.VDN_BF16])
@pytest.mark.parametrize("M,H,dv,n", [(1000, 2, 64, 192), (77, 3, 128, 256)])
def test_out_proj_matches_oracle(out_dtype, M, H, dv, n):
    """y [M, H, 2, d_v] (bf16) times the stacked weight [H*2*d_v, n] (bf16),
    fp32 accumulation, against the oracle's product of the same bf16 values."""
    r = np.random.default_rng(M + n)
    yt = _bf16_tensor(r.standard_normal((M, H, 2, dv)))
    wt = _bf16_tensor(r.standard_normal((H * 2 * dv, n)) / np.sqrt(H * 2 * dv))
    out = torch.empty((M, n), dtype=torch.float32 if out_dtype == L.VDN_F32 else torch.bfloat16, device="cuda")
    L.vdn_out_proj(M, H * 2 * dv, n, out_dtype, yt, wt, out)
    torch.cuda.synchronize()
    ref = O.out_proj(yt.float().cpu().numpy(), wt.float().cpu().numpy())
    got = out.float().cpu().numpy().astype(np.float64)
    # fp32 accumulation of K = H*2*d_v products: ~sqrt(K) * 2^-24 relative; a bf16 store adds 2^-9
    tol = 2e-5 * np.abs(ref).max() + (2.0 ** -8 * np.abs(ref) if out_dtype == L.VDN_BF16 else 0.0)
    assert np.all(np.abs(got - ref) <= tol)


@pytest.mark.parametrize("out_dtype", [L.VDN_F32, L.VDN_BF16])
@pytest.mark.parametrize("M,K,N", [(2000, 144, 520), (4099, 1280, 768), (300, 6144, 3072)])
def test_out_proj_tile_edges(out_dtype, M, K, N):
    """The tensor-core projection at its tile edges: rows past M in the last
    256-row tile, columns past N in the last 256-column tile, a last K block
    of 16 of 64 values (K = 144), several tiles per CTA pair, and the layer's
    K = 6,144; against the oracle's float64 product of the same bf16 values."""
    r = np.random.default_rng(M + K + N)
    yt = _bf16_tensor(r.standard_normal((M, K)))
    wt = _bf16_tensor(r.standard_normal((K, N)) / np.sqrt(K))
    out = torch.full((M, N), float("nan"), dtype=torch.float32 if out_dtype == L.VDN_F32 else torch.bfloat16,
                     device="cuda")
    L.vdn_out_proj(M, K, N, out_dtype, yt, wt, out)
    torch.cuda.synchronize()
    assert L.vdn_proj_device_status() == (L.VDN_OK, 0)
    ref = O.out_proj(yt.float().cpu().numpy().reshape(M, 1, 1, K), wt.float().cpu().numpy())
    got = out.float().cpu().numpy().astype(np.float64)
    tol = 2e-5 * np.abs(ref).max() + (2.0 ** -8 * np.abs(ref) if out_dtype == L.VDN_BF16 else 0.0)
    assert np.all(np.abs(got - ref) <= tol)


def test_out_proj_on_core_output():
    """The projection of the core's own bf16 output (out_mode 0) matches the
    oracle's projection of the oracle's output within the bf16-mode tolerance."""
    w = WORKLOADS["small"]
    inp, cfg, ha, _, y = run(w.shape, w.dtype, w.seed, y_dtype=L.VDN_BF16)
    M, K, n = cfg.B * cfg.T * cfg.N, cfg.H * 2 * cfg.d_v, 96
    r = np.random.default_rng(4)
    wt = _bf16_tensor(r.standard_normal((K, n)) / np.sqrt(K))
    out = torch.empty((M, n), dtype=torch.float32, device="cuda")
    L.vdn_out_proj(M, K, n, L.VDN_F32, ha.y, wt, out)
    torch.cuda.synchronize()
    ref = O.out_proj(oracle(inp, cfg), wt.float().cpu().numpy()).reshape(M, n)
    e = rel_err(out.cpu().numpy().astype(np.float64), ref)
    assert e <= TOL["bf16"], e


# ------------------------------------------------------------ text cross-attention
@pytest.mark.parametrize("y_bf16", [False, True])
@pytest.mark.parametrize("shape", [Shape(1, 6, 50, 2, 64, 64, 40), Shape(2, 4, 70, 3, 128, 128, 300)])
def test_text_cross_attn_matches_oracle(shape, y_bf16):
    """Every video query over its batch's L text tokens (one partial key tile
    at L = 40; three tiles, the last partial, at L = 300), against the oracle."""
    inp = make_inputs(shape, 17, "bf16")
    cfg = cfg_for(shape, "bf16", y_dtype=L.VDN_BF16 if y_bf16 else L.VDN_F32)
    t = to_torch(inp, "bf16", "cuda")
    y = torch.empty((shape.B, shape.T, shape.N, shape.H, shape.d_v),
                    dtype=torch.bfloat16 if y_bf16 else torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    args = L.make_args(t["q"], None, None, None, None, None, None, y, ws, text_k=t["text_k"], text_v=t["text_v"])
    L.vdn_text_cross_attn(cfg, args)
    torch.cuda.synchronize()
    assert L.vdn_hybrid_device_status(cfg, args)[0] == L.VDN_OK
    got = y.float().cpu().numpy().astype(np.float64)
    scale = 1.0 / np.sqrt(shape.d_k)
    for b in range(shape.B):
        for h in range(shape.H):
            ref = O.text_cross_attn(inp["q"][b, :, :, h], inp["text_k"][b, :, h], inp["text_v"][b, :, h], scale)
            e = rel_err(got[b, :, :, h], ref, U_BF16 * np.abs(ref) if y_bf16 else None)
            assert e <= TOL["bf16"], (b, h, e)


# ------------------------------------------------------------ FP8 projection
@pytest.mark.parametrize("src", ["bf16", "f32"])
def test_quantize_fp8_matches_oracle(src):
    """e4m3 codes and the per-tensor scale, bit for bit against the oracle's
    quantisation of the same values."""
    r = np.random.default_rng(7)
    x = (r.standard_normal((1000, 256)) * 3).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    if src == "bf16":
        xt = xt.to(torch.bfloat16)
        x = xt.float().cpu().numpy()
    q = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(1, dtype=torch.float32, device="cuda")
    L.vdn_quantize_fp8(xt, L.VDN_BF16 if src == "bf16" else L.VDN_F32, x.size, q, sc)
    torch.cuda.synchronize()
    qo, so = O.quantize_e4m3(x)
    assert sc.item() == so
    np.testing.assert_array_equal(q.cpu().numpy(), qo.view(torch.uint8).numpy())


@pytest.mark.parametrize("out_dtype", [L.VDN_F32, L.VDN_BF16])
@pytest.mark.parametrize("M,K,N", [(777, 512, 256), (2000, 208, 528), (300, 6144, 3072)])
def test_out_proj_fp8_matches_oracle(out_dtype, M, K, N):
    """The FP8 projection of quantised operands against the oracle's float64
    product of the same dequantised values (ragged M and N tiles, a last K
    block of 80 of 128 values at K = 208, and the layer's K = 6,144)."""
    r = np.random.default_rng(9 + M)
    y = torch.from_numpy(r.standard_normal((M, K)).astype(np.float32)).cuda().to(torch.bfloat16)
    w_t = torch.from_numpy((r.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32)).cuda().to(torch.bfloat16)
    qy = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    qw = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(2, dtype=torch.float32, device="cuda")
    L.vdn_quantize_fp8(y, L.VDN_BF16, M * K, qy, scales[0:1])
    L.vdn_quantize_fp8(w_t, L.VDN_BF16, N * K, qw, scales[1:2])
    out = torch.empty((M, N), dtype=torch.float32 if out_dtype == L.VDN_F32 else torch.bfloat16, device="cuda")
    L.vdn_out_proj_fp8(M, K, N, out_dtype, qy, qw, scales, out)
    torch.cuda.synchronize()
    assert L.vdn_proj_device_status() == (L.VDN_OK, 0)
    sy, sw = scales.cpu().numpy()
    ref = O.out_proj_fp8(qy.cpu().view(torch.float8_e4m3fn), sy, qw.cpu().view(torch.float8_e4m3fn), sw)
    got = out.float().cpu().numpy().astype(np.float64)
    tol = 1e-5 * np.abs(ref).max() + (2.0 ** -8 * np.abs(ref) if out_dtype == L.VDN_BF16 else 0.0)
    assert np.all(np.abs(got - ref) <= tol)


STREAM_CASES = {
    "d64_simt_f32": (Shape(1, 20, 24, 2, 64, 64, 6), "f32", {}),
    "d64_bf16": (Shape(1, 20, 24, 2, 64, 64, 6), "bf16", {}),
    "d128_frames": (Shape(1, 22, 40, 2, 128, 128, 4), "bf16", dict(scan_mode=1)),
    "d128_chunks": (Shape(1, 22, 40, 2, 128, 128, 4), "bf16", dict(scan_mode=2)),
    "d128_f32": (Shape(1, 12, 30, 1, 128, 128, 4), "f32", {}),
}


@pytest.mark.parametrize("case", sorted(STREAM_CASES))
def test_stream_fwd_init_matches_oracle(case):
    """Streaming: a given forward start state (the state carried from the
    previous segment) on every scan kernel (SIMT, tensor-core frame steps,
    composed chunk steps), against the oracle with the same start."""
    shape, dtype, kw = STREAM_CASES[case]
    r = np.random.default_rng(17)
    extra = {"fwd_init": (0.3 * r.standard_normal((shape.B, shape.H, shape.d_v, shape.d_k))).astype(np.float32)}
    inp, cfg, ha, _, y = run(shape, dtype, 23, extra=extra, **kw)
    check(y, oracle(inp, cfg), cfg, dtype)
    it = ha.intermediates()["fwd_snap"].double().cpu().numpy()
    np.testing.assert_array_equal(it[:, :, 0], extra["fwd_init"].astype(np.float64))


def test_stream_d256_fwd_init_matches_oracle():
    shape = Shape(1, 12, 40, 1, 256, 256, 8)
    r = np.random.default_rng(18)
    extra = {"fwd_init": (0.3 * r.standard_normal((1, 1, 256, 256))).astype(np.float32)}
    inp, cfg, ha, t, y = run(shape, "bf16", 29, extra=extra, stages=VDA)
    ref_y = O.hybrid_attn(inp, ocfg(cfg))
    assert rel_err(y[..., 1, :], ref_y[..., 1, :]) <= TOL["bf16"]


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_stream_two_segments_match_oracle(dtype, d):
    """Two appended segments: the second call starts its forward scan from
    the first call's forward end state (read back from the workspace); the
    oracle chains its own end state the same way."""
    s1, s2 = Shape(1, 17, 32, 2, d, d, 6), Shape(1, 13, 32, 2, d, d, 0)
    inp1, cfg1, ha1, _, y1 = run(s1, dtype, 31)
    oc1 = ocfg(cfg1)
    ends = [O.head_states(inp1, oc1, 0, h)[0][cfg1.T] for h in range(cfg1.H)]
    carried = np.stack(ends)[None]
    got_end = ha1.forward_end_state().double().cpu().numpy()
    assert rel_err(got_end, carried) <= TOL[dtype]
    # the second segment's text state is zero: it reads only the carried past
    # and its own frames
    inp2 = make_inputs(s2, 32, dtype)
    for k in ("text_k", "text_v", "text_beta", "text_k_bits", "text_v_bits"):
        inp2.pop(k, None)
    cfg2 = cfg_for(s2, dtype)
    t2 = to_torch(inp2, dtype, "cuda")
    t2["fwd_init"] = ha1.forward_end_state()
    ha2 = HybridAttention(cfg2)
    y2 = ha2(t2).float().cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    ref2 = O.hybrid_attn({**inp2, "fwd_init": carried}, O.Cfg(**{**ocfg(cfg2).__dict__, "out_mode": 0}))
    check(y2, ref2, cfg2, dtype)


VARIANT_SHAPES = [Shape(1, 12, 40, 2, 32, 32, 4), Shape(1, 15, 70, 2, 64, 64, 8), Shape(1, 12, 50, 1, 128, 128, 8)]


@pytest.mark.parametrize("update", [1, 2])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", VARIANT_SHAPES, ids=lambda s: f"d{s.d_k}")
def test_ablation_write_matches_oracle(shape, dtype, update):
    """The ablation writes (1: frame-level independent writes with the 1/N
    rescaling; 2: the token-wise delta rule): their per-frame maps M'_t, C'_t
    in the M_t, C_t slots, the chunk-boundary states of both scans and the
    whole output, against the oracle with the same write."""
    inp, cfg, ha, _, y = run(shape, dtype, 41, update=update)
    oc = ocfg(cfg)
    check(y, O.hybrid_attn(inp, O.Cfg(**{**oc.__dict__, "out_mode": 0})), cfg, dtype)
    it = {k: v.double().cpu().numpy() for k, v in ha.intermediates().items()}
    for h in range(cfg.H):
        ref = O.vda_intermediates(inp, oc, 0, h)
        scale = np.sqrt(np.mean(ref["R"] ** 2))
        for t in range(1, cfg.T - 1):
            np.testing.assert_allclose(it["M"][0, t, h], ref["M"][t], rtol=0, atol=2e-5)
            np.testing.assert_allclose(it["C"][0, t, h], ref["C"][t], rtol=0, atol=2e-5 * np.abs(ref["C"][t]).max())
        for j in range(cfg.C + 1):
            fj = min(5 * j, cfg.T)
            np.testing.assert_allclose(it["fwd_snap"][0, h, j], ref["F"][fj], rtol=0, atol=1e-4 * scale)
            np.testing.assert_allclose(it["bwd_snap"][0, h, j], ref["G"][fj], rtol=0, atol=1e-4 * scale)


def test_ablation_write_ragged_frame():
    """A frame of 37 tokens: two full staged blocks and a partial third."""
    shape = Shape(1, 7, 37, 3, 64, 64, 0)
    for update in (1, 2):
        inp, cfg, _, _, y = run(shape, "bf16", 43, drop_text=True, update=update)
        oc = ocfg(cfg)
        check(y, O.hybrid_attn(inp, O.Cfg(**{**oc.__dict__, "out_mode": 0})), cfg, "bf16")


def test_ulysses_wrapper_single_rank_matches_oracle():
    """The Ulysses wrapper in one process (no exchange): sequence-flattened
    inputs in, [B, T N, H, 2, d_v] out, against the oracle."""
    from video_diffusion_hybrid_b200.ulysses import PER_TOKEN, UlyssesHybridAttention
    shape = Shape(1, 12, 40, 2, 64, 64, 6)
    inp = make_inputs(shape, 51, "bf16")
    cfg = cfg_for(shape, "bf16")
    t = to_torch(inp, "bf16", "cuda")
    t = {k: (v.flatten(1, 2) if k in PER_TOKEN else v) for k, v in t.items()}
    u = UlyssesHybridAttention(cfg)
    y = u(t)
    assert u.device_status()[0] == L.VDN_OK
    got = y.float().cpu().numpy().astype(np.float64).reshape(1, 12, 40, 2, 2, 64)
    check(got, oracle(inp, cfg), cfg, "bf16")

"""Pins of the gradient oracle of both branches: its forwards are the numpy
oracle's linear and softmax slots, and its gradients match central finite
differences of the numpy oracle along random directions."""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O
from oracle import vdn_oracle_grad as OG
from video_diffusion_hybrid_b200.synth import Shape, make_inputs


def _case(anchors=4, L=3, weight=True, T=12, fwd_init=False):
    shp = Shape(B=1, T=T, N=5, H=2, d_k=6, d_v=6, L=L)
    inp = {k: np.asarray(v, np.float64) for k, v in make_inputs(shp, seed=21).items() if not k.endswith("_bits")}
    r = np.random.default_rng(22)
    if weight:
        inp["rms_weight"] = 1 + 0.3 * r.standard_normal((2, 6))
    if fwd_init:
        inp["fwd_init"] = 0.5 * r.standard_normal((1, 2, 6, 6))
    cfg = O.Cfg(B=1, T=T, N=5, H=2, d_k=6, d_v=6, L=L, anchors=anchors)
    return inp, cfg


@pytest.mark.parametrize("anchors,fwd_init", [(4, False), (0, False), (4, True)])
def test_torch_forward_is_the_oracle(anchors, fwd_init):
    inp, cfg = _case(anchors, fwd_init=fwd_init)
    np.testing.assert_allclose(OG.linear_branch_forward(inp, cfg), O.hybrid_attn(inp, cfg)[..., 1, :],
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("anchors,weight,fwd_init", [(4, True, False), (0, False, False), (4, False, True)])
def test_gradients_match_finite_differences(anchors, weight, fwd_init):
    inp, cfg = _case(anchors, weight=weight, fwd_init=fwd_init)
    r = np.random.default_rng(23)
    dy = r.standard_normal((1, cfg.T, 5, 2, 6))
    grads = OG.linear_branch_grads(inp, cfg, dy)
    f = lambda d: float(np.sum(O.hybrid_attn(d, cfg)[..., 1, :] * dy))
    for name, g in grads.items():
        u = r.standard_normal(g.shape)
        if name == "beta":
            u *= 0.1
        eps = 1e-6
        plus, minus = dict(inp), dict(inp)
        plus[name] = inp[name] + eps * u
        minus[name] = inp[name] - eps * u
        fd = (f(plus) - f(minus)) / (2 * eps)
        an = float(np.sum(g * u))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_anchor_tokens_get_no_write_gradient():
    """Anchor frames are never written, so their k, v and beta do not reach
    the linear branch; their q still reads."""
    inp, cfg = _case(4)
    g = OG.linear_branch_grads(inp, cfg, np.ones((1, cfg.T, 5, 2, 6)))
    for name in ("k", "v", "beta"):
        assert np.all(g[name][:, 0] == 0) and np.all(g[name][:, -1] == 0)
        assert np.any(g[name][:, 1] != 0)
    assert np.any(g["q"][:, 0] != 0)


def test_unreached_inputs_get_zero_gradient():
    """At T = 10 (two chunks) every query reads only the start states, so the
    frame writes (k, v, beta, alpha) do not reach the output: zero gradients,
    as finite differences of the numpy oracle also give."""
    inp, cfg = _case(4, T=10)
    g = OG.linear_branch_grads(inp, cfg, np.ones((1, 10, 5, 2, 6)))
    for name in ("k", "v", "beta", "alpha"):
        assert g[name].shape == inp[name].shape and np.all(g[name] == 0)
    f = lambda d: float(np.sum(O.hybrid_attn(d, cfg)[..., 1, :]))
    plus = dict(inp)
    plus["k"] = inp["k"] + 1e-3
    assert f(plus) == f(inp)
    assert np.any(g["q"] != 0)


def _sm_case(T=12, anchors=4, N=4):
    shp = Shape(B=1, T=T, N=N, H=2, d_k=6, d_v=6, L=0)
    inp = {k: np.asarray(v, np.float64) for k, v in make_inputs(shp, seed=24).items() if not k.endswith("_bits")}
    cfg = O.Cfg(B=1, T=T, N=N, H=2, d_k=6, d_v=6, L=0, anchors=anchors, softmax_scale=3.0)
    return inp, cfg


@pytest.mark.parametrize("anchors", [4, 0])
def test_softmax_torch_forward_is_the_oracle(anchors):
    """The per-frame torch softmax equals the numpy oracle's softmax slot, which
    is itself pinned against dense attention under the explicit token mask."""
    inp, cfg = _sm_case(anchors=anchors)
    x = {n: torch.from_numpy(inp[n]) for n in OG.SM_INPUTS}
    with torch.no_grad():
        y = OG.softmax_branch(x, cfg).numpy()
    np.testing.assert_allclose(y, O.hybrid_attn(inp, cfg)[..., 0, :], rtol=0, atol=1e-12)


@pytest.mark.parametrize("anchors", [4, 0])
def test_softmax_gradients_match_finite_differences(anchors):
    inp, cfg = _sm_case(anchors=anchors)
    r = np.random.default_rng(25)
    dy = r.standard_normal((1, cfg.T, cfg.N, 2, 6))
    grads = OG.softmax_branch_grads(inp, cfg, dy)
    f = lambda d: float(np.sum(O.hybrid_attn(d, cfg)[..., 0, :] * dy))
    for name, g in grads.items():
        u = r.standard_normal(g.shape)
        eps = 1e-6
        plus, minus = dict(inp), dict(inp)
        plus[name] = inp[name] + eps * u
        minus[name] = inp[name] - eps * u
        fd = (f(plus) - f(minus)) / (2 * eps)
        an = float(np.sum(g * u))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_softmax_masked_keys_get_no_gradient_from_a_query_frame():
    """A query frame's output does not reach the keys its mask hides: with one
    non-anchor query frame, the k and v rows of frames outside its window and
    the anchors are exactly zero; and the frame-by-frame form over every
    frame equals the whole-problem gradient."""
    inp, cfg = _sm_case(T=20)
    dy = np.random.default_rng(26).standard_normal((1, 20, cfg.N, 2, 6))
    g = OG.softmax_branch_grads_frames(inp, cfg, dy, 0, 1, [12])
    allowed = O.frame_mask(20, 5, 4)[12]
    for f in range(20):
        nz = np.any(g["k"][0, f, :, 1] != 0)
        assert nz == bool(allowed[f]), f
    assert np.all(g["k"][..., 0, :] == 0)
    full = OG.softmax_branch_grads(inp, cfg, dy * (np.arange(2) == 1)[None, None, None, :, None])
    per = OG.softmax_branch_grads_frames(inp, cfg, dy, 0, 1, range(20))
    for n in OG.SM_INPUTS:
        np.testing.assert_allclose(per[n], full[n], rtol=0, atol=1e-12)

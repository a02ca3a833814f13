"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types an oracle formula: each checks the oracle against an
independent route (the objective itself, a stacked least-squares solve, the
token-space Woodbury form, the classic delta rule, a combinatorial count,
library routines, brute force) or an invariant the pages state.
"""
import os

import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O
from video_diffusion_hybrid_b200.synth import Shape, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _frame(n, dk, dv, seed=0, unit=True):
    r = np.random.default_rng(seed)
    K = r.standard_normal((n, dk))
    if unit:
        K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = r.standard_normal((n, dv))
    beta = 1 / (1 + np.exp(-r.standard_normal(n)))
    Sbar = r.standard_normal((dv, dk))
    return Sbar, K, V, beta


def _objective(S, Sbar, K, V, beta):
    """||S - S_bar||^2 + sum_i beta_i ||S k_i - v_i||^2, written token by
    token ([P1] section 四; deepmagic post, closed form paragraph)."""
    f = np.sum((S - Sbar) ** 2)
    for i in range(K.shape[0]):
        r = S @ K[i] - V[i]
        f += beta[i] * (r @ r)
    return f


# ---------------------------------------------------------------- mask ----
def _golden_rows():
    rows = {}
    with open(os.path.join(GOLDEN, "mask_density.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                q, T, ch, an, val, _src = line.split()
                rows[q] = (int(T), int(ch), int(an), float(val))
    return rows


def test_density_matches_page_value():
    T, ch, an, val = _golden_rows()["density"]
    assert round(100 * O.mask_density(T, ch, an), 2) == pytest.approx(val, abs=1e-9)


def test_anchor_overhead_matches_page_value():
    T, ch, an, val = _golden_rows()["anchor_overhead"]
    extra = 100 * (O.mask_density(T, ch, an) - O.mask_density(T, ch, 0))
    assert abs(extra - val) < 0.01


@pytest.mark.parametrize("T", [15, 20, 30, 45, 90, 180])
def test_mask_count_closed_form(T):
    """Allowed frame pairs counted combinatorially for T = 5C, C >= 3:
    25 (3C - 2) window pairs, plus the 4T - 4 anchor row/column pairs, minus
    the 38 of those already inside the window."""
    C = T // 5
    window = 25 * (3 * C - 2)
    assert O.frame_mask(T, 5, 0).sum() == window
    assert O.frame_mask(T, 5, 4).sum() == window + (4 * T - 4) - 38


def test_token_mask_is_frame_mask_blocks():
    T, N = 12, 3
    M = O.token_mask(T, N, 5, 4)
    Fm = O.frame_mask(T, 5, 4)
    for i in range(T * N):
        for j in range(T * N):
            assert M[i, j] == Fm[i // N, j // N]


# ---------------------------------------------------------- VDA update ----
@pytest.mark.parametrize("n,dk,dv", [(1, 8, 8), (7, 8, 5), (40, 16, 16), (3, 32, 32)])
def test_update_minimises_objective(n, dk, dv):
    """At the minimiser of a quadratic, f(S + D) - f(S) equals the quadratic
    form ||D||^2 + sum beta_i ||D k_i||^2 for every perturbation D."""
    Sbar, K, V, beta = _frame(n, dk, dv, seed=n)
    S = O.vda_update(Sbar, K, V, beta)
    f0 = _objective(S, Sbar, K, V, beta)
    for s in range(4):
        D = np.random.default_rng(s).standard_normal(S.shape) * 1e-2
        quad = np.sum(D ** 2) + sum(beta[i] * np.sum((D @ K[i]) ** 2) for i in range(n))
        assert _objective(S + D, Sbar, K, V, beta) - f0 == pytest.approx(quad, rel=1e-8, abs=1e-14)


def test_update_equals_stacked_least_squares():
    """The objective is an ordinary least-squares problem per row of S:
    rows [I ; sqrt(beta_i) k_i^T] against targets [s_bar ; sqrt(beta_i) v_i]."""
    Sbar, K, V, beta = _frame(50, 12, 9, seed=3)
    S = O.vda_update(Sbar, K, V, beta)
    sb = np.sqrt(beta)[:, None]
    Amat = np.vstack([np.eye(12), sb * K])
    for r in range(9):
        rhs = np.concatenate([Sbar[r], sb[:, 0] * V[:, r]])
        x, *_ = np.linalg.lstsq(Amat, rhs, rcond=None)
        np.testing.assert_allclose(S[r], x, rtol=0, atol=1e-11)


@pytest.mark.parametrize("n,d", [(5, 16), (60, 16), (33, 32)])
def test_update_matches_token_space_woodbury(n, d):
    """S = S_bar + W^T K with W = (D^-1 + K K^T)^-1 (V - K S_bar^T), D = diag(beta):
    the same minimiser reached through an n x n solve instead of d x d."""
    Sbar, K, V, beta = _frame(n, d, d, seed=n + d)
    W = np.linalg.solve(np.diag(1 / beta) + K @ K.T, V - K @ Sbar.T)
    np.testing.assert_allclose(O.vda_update(Sbar, K, V, beta), Sbar + W.T @ K, rtol=0, atol=1e-10)


def test_single_token_is_classic_delta_rule():
    """One token per frame: S = S_bar + beta' (v - S_bar k) k^T with the
    effective strength beta' = beta / (1 + beta ||k||^2) (the token-wise
    delta rule that VDA generalises, aimodeling news 'The VDN split')."""
    for s in range(5):
        Sbar, K, V, beta = _frame(1, 16, 12, seed=100 + s, unit=(s % 2 == 0))
        k, v, b = K[0], V[0], beta[0]
        want = Sbar + (b / (1 + b * k @ k)) * np.outer(v - Sbar @ k, k)
        np.testing.assert_allclose(O.vda_update(Sbar, K, V, beta), want, rtol=0, atol=1e-12)


def test_inherited_map_is_non_expansive():
    """S_bar -> S_bar (I + A)^-1 never amplifies the inherited state
    ([P1] section 四; deepmagic post; aimodeling news)."""
    for s in range(6):
        _, K, V, beta = _frame(30 + 20 * s, 16, 16, seed=200 + s)
        M, _ = O.frame_map(K, V, beta)
        assert np.linalg.norm(M, 2) <= 1 + 1e-12
        X = np.random.default_rng(s).standard_normal((16, 16))
        assert np.linalg.norm(X @ M) <= np.linalg.norm(X) * (1 + 1e-12)
        # the inherited part of the update is exactly that map
        np.testing.assert_allclose(O.vda_update(X, K, V, beta) - O.vda_update(0 * X, K, V, beta), X @ M,
                                   rtol=0, atol=1e-11)


def test_evidence_saturates_below_one():
    """n copies of one unit key written from zero give S k = n b / (1 + n b) v:
    a hundred patches push the weight toward, never past, one.  Orthogonal
    keys each keep b / (1 + b) (aimodeling news 'The VDN split')."""
    d, b = 16, 0.7
    k = np.zeros(d); k[3] = 1.0
    v = np.random.default_rng(0).standard_normal(d)
    for n in (1, 2, 10, 100):
        S = O.vda_update(np.zeros((d, d)), np.tile(k, (n, 1)), np.tile(v, (n, 1)), np.full(n, b))
        w = n * b / (1 + n * b)
        np.testing.assert_allclose(S @ k, w * v, rtol=0, atol=1e-12)
        assert w < 1
    K = np.eye(d)[:5]
    V = np.random.default_rng(1).standard_normal((5, d))
    S = O.vda_update(np.zeros((d, d)), K, V, np.full(5, b))
    for i in range(5):
        np.testing.assert_allclose(S @ K[i], b / (1 + b) * V[i], rtol=0, atol=1e-12)


def test_update_independent_of_token_order():
    """The joint frame write does not depend on an order of the tokens
    ([P1] section 四: no artificial scan order inside a frame)."""
    Sbar, K, V, beta = _frame(64, 16, 16, seed=9)
    p = np.random.default_rng(2).permutation(64)
    np.testing.assert_allclose(O.vda_update(Sbar, K, V, beta), O.vda_update(Sbar, K[p], V[p], beta[p]),
                               rtol=0, atol=1e-12)


def test_frame_map_expands_update():
    Sbar, K, V, beta = _frame(20, 8, 6, seed=5)
    M, C = O.frame_map(K, V, beta)
    np.testing.assert_allclose(Sbar @ M + C, O.vda_update(Sbar, K, V, beta), rtol=0, atol=1e-12)
    np.testing.assert_allclose(M, M.T, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- scan ----
def _scan_inputs(T, N, d, seed):
    r = np.random.default_rng(seed)
    k = r.standard_normal((T, N, d)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, N, d))
    beta = 1 / (1 + np.exp(-r.standard_normal((T, N))))
    alpha = 1 / (1 + np.exp(-(2 + 0.5 * r.standard_normal(T))))
    S0 = r.standard_normal((d, d))
    return S0, k, v, beta, alpha


def test_backward_scan_is_forward_scan_reversed():
    S0, k, v, beta, alpha = _scan_inputs(17, 6, 8, 1)
    G = O.backward_states(S0, k, v, beta, alpha, anchors=4)
    F = O.forward_states(S0, k[::-1], v[::-1], beta[::-1], alpha[::-1], anchors=4)
    np.testing.assert_allclose(G[::-1], F, rtol=0, atol=1e-12)


def test_zero_decay_forgets_history():
    S0, k, v, beta, alpha = _scan_inputs(8, 5, 8, 2)
    F = O.forward_states(S0, k, v, beta, np.zeros(8), anchors=0)
    for t in range(8):
        np.testing.assert_allclose(F[t + 1], O.vda_update(np.zeros((8, 8)), k[t], v[t], beta[t]), atol=1e-13)


def test_scan_equals_least_squares_chain():
    """Each forward step, computed by the stacked least-squares route from the
    previous step's state decayed by alpha, reproduces the scan."""
    S0, k, v, beta, alpha = _scan_inputs(12, 4, 6, 3)
    F = O.forward_states(S0, k, v, beta, alpha, anchors=4)
    S = S0.copy()
    for t in range(12):
        if t not in (0, 11):
            Sb = alpha[t] * S
            sb = np.sqrt(beta[t])[:, None]
            Amat = np.vstack([np.eye(6), sb * k[t]])
            S = np.stack([np.linalg.lstsq(Amat, np.concatenate([Sb[r], sb[:, 0] * v[t][:, r]]), rcond=None)[0]
                          for r in range(6)])
        np.testing.assert_allclose(F[t + 1], S, rtol=0, atol=1e-10)


@pytest.mark.parametrize("T,anchors", [(30, 4), (23, 4), (35, 0), (10, 4), (7, 4)])
def test_read_regions_cover_each_frame_once(T, anchors):
    """Tag every frame with its own orthogonal key/value (one token, alpha=1):
    the diagonal of a state then shows which frames it holds.  For every query
    frame, forward reads + backward reads + the softmax key frames cover every
    frame exactly once, and anchor frames are never written
    ([P1] section 三: the regions do not overlap; anchors are not re-written)."""
    d = T
    k = np.eye(d)[:T, None, :]
    v = np.eye(d)[:T, None, :]
    beta = np.ones((T, 1))
    alpha = np.ones(T)
    S0 = np.zeros((d, d))
    F = O.forward_states(S0, k, v, beta, alpha, anchors)
    G = O.backward_states(S0, k, v, beta, alpha, anchors)
    fm = O.frame_mask(T, 5, anchors)
    anc = set(O.anchor_frames(T, anchors))
    for t in range(T):
        R = O.read_state(F, G, t, T, 5, anchors)
        held = np.diag(R)
        np.testing.assert_allclose(held[held > 1e-9], 0.5, atol=1e-12)  # beta/(1+beta) with beta=1
        lin = set(np.nonzero(held > 1e-9)[0])
        soft = set(np.nonzero(fm[t])[0])
        assert not (lin & soft)
        assert not (lin & anc)
        assert lin | soft == set(range(T))


def test_half_text_reads_sum_to_one_text_read():
    """With no video written into a query's states (T=10: two chunks, all in
    window), its linear read is exactly the text state applied once
    ([P1] section 三; deepmagic post: each direction starts from half)."""
    shp = Shape(B=1, T=10, N=16, H=2, d_k=32, d_v=32, L=8)
    inp = make_inputs(shp, seed=0)
    cfg = O.Cfg(B=1, T=10, N=16, H=2, d_k=32, d_v=32, L=8)
    Y = O.hybrid_attn(inp, cfg)
    for h in range(2):
        Sx = O.vda_update(np.zeros((32, 32)), inp["text_k"][0, :, h], inp["text_v"][0, :, h], inp["text_beta"][0, :, h])
        o = inp["q"][0, :, :, h].astype(np.float64) @ Sx.T
        want = O.rms_gate(o, inp["gate_lin"][0, :, :, h], 1e-6)
        np.testing.assert_allclose(Y[0, :, :, h, 1], want, rtol=0, atol=1e-12)


# ------------------------------------------------------------- softmax ----
def _torch_sdpa(q, k, v, mask, scale):
    qt, kt, vt = (torch.from_numpy(np.asarray(x, np.float64))[None] for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask)[None],
                                                           scale=scale)
    return out[0].numpy()


@pytest.mark.parametrize("T,N,anchors,scale", [(10, 4, 4, None), (23, 3, 4, None), (30, 2, 0, 10.0),
                                               (20, 5, 4, 10.0)])
def test_windowed_softmax_equals_dense_masked_attention(T, N, anchors, scale):
    """The windowed + anchor softmax the oracle uses equals dense attention
    under the explicit hybrid token mask, computed by torch's SDPA."""
    r = np.random.default_rng(T)
    d = 8
    q, k, v = (r.standard_normal((T, N, d)) for _ in range(3))
    sc = scale or 1 / np.sqrt(d)
    want = _torch_sdpa(q.reshape(T * N, d), k.reshape(T * N, d), v.reshape(T * N, d),
                       O.token_mask(T, N, 5, anchors), sc).reshape(T, N, d)
    dense = O.softmax_dense_masked(q, k, v, T, N, 5, anchors, sc)
    np.testing.assert_allclose(dense, want, rtol=0, atol=1e-12)
    for t in range(T):
        np.testing.assert_allclose(O.softmax_frame(q[t], k, v, t, T, 5, anchors, sc), want[t], rtol=0, atol=1e-12)


def test_softmax_brute_force_tiny():
    """Pair-by-pair softmax with explicit exponentials on a tiny case."""
    T, N, d = 11, 2, 4
    r = np.random.default_rng(7)
    q, k, v = (r.standard_normal((T, N, d)) for _ in range(3))
    sc = 0.9
    for tq in range(T):
        for n in range(N):
            num = np.zeros(d); den = 0.0
            for tk in range(T):
                cq, ck = tq // 5, tk // 5
                if abs(cq - ck) <= 1 or tk in (0, T - 1) or tq in (0, T - 1):
                    for m in range(N):
                        e = np.exp(sc * q[tq, n] @ k[tk, m])
                        num += e * v[tk, m]; den += e
            got = O.softmax_frame(q[tq, n:n + 1], k, v, tq, T, 5, 4, sc)[0]
            np.testing.assert_allclose(got, num / den, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------ norm and gates ----
def test_rms_gate_matches_library():
    r = np.random.default_rng(3)
    o = r.standard_normal((7, 32)); g = r.standard_normal((7, 32)); w = r.standard_normal(32)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (32,), torch.from_numpy(w), eps=1e-6)
    ref = torch.sigmoid(torch.from_numpy(g)) * ref
    np.testing.assert_allclose(O.rms_gate(o, g, 1e-6, w), ref.numpy(), rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------ end to end --
def _cfg(shp, **kw):
    return O.Cfg(B=shp.B, T=shp.T, N=shp.N, H=shp.H, d_k=shp.d_k, d_v=shp.d_v, L=shp.L, **kw)


def test_rows_route_equals_full_route():
    shp = Shape(B=2, T=30, N=4, H=2, d_k=8, d_v=8, L=5)
    inp = make_inputs(shp, seed=11)
    cfg = _cfg(shp)
    Y = O.hybrid_attn(inp, cfg)
    Yd = O.hybrid_attn(inp, cfg, softmax="dense")
    np.testing.assert_allclose(Y, Yd, rtol=0, atol=1e-12)
    rows = [(b, t, n, h) for b in range(2) for t in (0, 4, 5, 13, 24, 29) for n in (0, 3) for h in range(2)]
    got = O.hybrid_attn_rows(inp, cfg, rows)
    for i, (b, t, n, h) in enumerate(rows):
        np.testing.assert_allclose(got[i], Y[b, t, n, h], rtol=0, atol=1e-12)
    Ys = O.hybrid_attn(inp, _cfg(shp, out_mode=1))
    np.testing.assert_allclose(Ys, Y.sum(axis=4), rtol=0, atol=1e-12)


def test_intermediates_reassemble_states():
    """The per-frame affine maps (M_t, C_t) chained from S_init reproduce the
    definitional forward scan, and the read table matches read_state."""
    shp = Shape(B=1, T=20, N=6, H=1, d_k=8, d_v=8, L=4)
    inp = make_inputs(shp, seed=5)
    cfg = _cfg(shp)
    it = O.vda_intermediates(inp, cfg, 0, 0)
    S = it["S_init"].copy()
    for t in range(20):
        if t not in (0, 19):
            S = inp["alpha"][0, t, 0] * S @ it["M"][t] + it["C"][t]
        np.testing.assert_allclose(S, it["F"][t + 1], rtol=0, atol=1e-11)
    for t in range(20):
        c = 4 if t in (0, 19) else t // 5
        np.testing.assert_allclose(it["R"][c], O.read_state(it["F"], it["G"], t, 20), rtol=0, atol=0)


# ------------------------------------------- planted mistakes must fail ---
def test_pins_catch_dropped_inherited_term(monkeypatch):
    orig = O.vda_update
    monkeypatch.setattr(O, "vda_update", lambda Sbar, K, V, b: orig(0 * np.asarray(Sbar), K, V, b))
    with pytest.raises(AssertionError):
        test_single_token_is_classic_delta_rule()


def test_pins_catch_shifted_read_window(monkeypatch):
    monkeypatch.setattr(O, "window_frames", lambda t, T, chunk=5: (max(0, chunk * (t // chunk)),
                                                                   min(T, chunk * (t // chunk + 2))))
    with pytest.raises(AssertionError):
        test_read_regions_cover_each_frame_once(30, 4)


def test_pins_catch_transposed_write(monkeypatch):
    orig = O.gram_write
    monkeypatch.setattr(O, "gram_write", lambda K, V, b: (orig(K, V, b)[0], orig(K, V, b)[1].T))
    with pytest.raises(AssertionError):
        test_update_matches_token_space_woodbury(5, 16)


# ---------------------------------------------------------------- chunk maps
@pytest.mark.parametrize("T,anchors", [(17, 4), (23, 4), (10, 0), (12, 4)])
def test_chunk_composed_scan_equals_frame_scan(T, anchors):
    """Stepping the two scans by composed chunk maps reproduces the
    frame-by-frame scans (each step a joint least-squares solve) at every
    chunk boundary, which is where the read takes its states."""
    S0, k, v, beta, alpha = _scan_inputs(T, 5, 6, 11 + T)
    F = O.forward_states(S0, k, v, beta, alpha, anchors=anchors)
    G = O.backward_states(S0, k, v, beta, alpha, anchors=anchors)
    Fc, Gc = O.chunk_scan(S0, *O.chunk_maps(k, v, beta, alpha, chunk=5, anchors=anchors))
    nc = O.num_chunks(T, 5)
    scale = np.abs(F).max()
    for j in range(nc + 1):
        b = min(5 * j, T)
        np.testing.assert_allclose(Fc[j], F[b], rtol=0, atol=1e-12 * scale)
        np.testing.assert_allclose(Gc[j], G[b], rtol=0, atol=1e-12 * scale)


def test_chunk_map_backward_uses_the_transpose():
    """Applying a chunk's frames in decreasing order, each as the joint solve
    from the decayed state, equals Lam S P^T + Cb: the reversed product of
    the symmetric M_t is the transpose of the forward product."""
    T = 15
    S0, k, v, beta, alpha = _scan_inputs(T, 7, 5, 5)
    P, Cf, Cb, Lam = O.chunk_maps(k, v, beta, alpha, chunk=5, anchors=4)
    S = rng.standard_normal((5, 5))
    for c in range(3):
        X = S.copy()
        for f in range(min(5 * c + 4, T - 1), 5 * c - 1, -1):
            if f not in (0, T - 1):
                X = O.vda_update(alpha[f] * X, k[f], v[f], beta[f])
        np.testing.assert_allclose(X, Lam[c] * S @ P[c].T + Cb[c], rtol=0, atol=1e-12 * np.abs(X).max())
        Y = S.copy()
        for f in range(5 * c, min(5 * c + 5, T)):
            if f not in (0, T - 1):
                Y = O.vda_update(alpha[f] * Y, k[f], v[f], beta[f])
        np.testing.assert_allclose(Y, Lam[c] * S @ P[c] + Cf[c], rtol=0, atol=1e-12 * np.abs(Y).max())


def test_chunk_map_special_cases():
    """A chunk of anchor frames only is the identity map; a chunk with one
    written frame is that frame's own map (M_t, C_t, alpha_t)."""
    S0, k, v, beta, alpha = _scan_inputs(2, 4, 6, 9)
    P, Cf, Cb, Lam = O.chunk_maps(k, v, beta, alpha, chunk=5, anchors=4)
    np.testing.assert_array_equal(P[0], np.eye(6))
    assert not Cf.any() and not Cb.any() and Lam[0] == 1.0
    S0, k, v, beta, alpha = _scan_inputs(3, 4, 6, 10)
    P, Cf, Cb, Lam = O.chunk_maps(k, v, beta, alpha, chunk=5, anchors=4)
    M, C = O.frame_map(k[1], v[1], beta[1])
    np.testing.assert_allclose(P[0], M, atol=1e-14)
    np.testing.assert_allclose(Cf[0], C, atol=1e-14)
    np.testing.assert_allclose(Cb[0], C, atol=1e-14)
    assert Lam[0] == alpha[1]


def test_out_proj_is_the_sum_of_the_branch_projections():
    """One product over the concat axis with the stacked weight equals the
    softmax branch projected by its weight plus the linear branch projected
    by its own, head by head (the reason the core puts the two branches on a
    size-2 axis)."""
    r = np.random.default_rng(21)
    H, dv, n = 3, 4, 5
    y = r.standard_normal((2, 7, H, 2, dv))
    W_sm = r.standard_normal((H, dv, n))
    W_lin = r.standard_normal((H, dv, n))
    W = np.stack([W_sm, W_lin], axis=1).reshape(H * 2 * dv, n)
    ref = np.zeros((2, 7, n))
    for h in range(H):
        ref += y[..., h, 0, :] @ W_sm[h] + y[..., h, 1, :] @ W_lin[h]
    np.testing.assert_allclose(O.out_proj(y, W), ref, rtol=0, atol=1e-12)


def test_text_cross_attn_equals_torch_sdpa():
    """The text cross-attention against torch's scaled-dot-product attention
    (no mask), a library routine, on random fp64 inputs."""
    r = np.random.default_rng(31)
    T, N, L, d = 3, 5, 7, 8
    q, k, v = r.standard_normal((T, N, d)), r.standard_normal((L, d)), r.standard_normal((L, d))
    got = O.text_cross_attn(q, k, v, 0.4)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.reshape(1, T * N, d)), torch.from_numpy(k[None]), torch.from_numpy(v[None]), scale=0.4)
    np.testing.assert_allclose(got, ref.numpy().reshape(T, N, d), rtol=0, atol=1e-12)


def test_quantize_e4m3_round_trip():
    """The per-tensor e4m3 quantisation: values on the scaled e4m3 grid come
    back exactly, every other normal-range value within half an e4m3 step
    (3 mantissa bits: 2^-4 relative), and nothing exceeds amax."""
    s0 = np.float32(0.5)
    grid = np.array([1.0, 1.125, 1.25, 2.0, 3.5, 448.0, 0.015625], np.float32) * s0
    q, s = O.quantize_e4m3(grid)
    assert s == np.float32(448.0) * s0 / np.float32(448.0)
    np.testing.assert_array_equal(q.float().numpy() * s, grid)
    r = np.random.default_rng(41)
    x = r.standard_normal(5000).astype(np.float32)
    q, s = O.quantize_e4m3(x)
    back = q.float().numpy().astype(np.float64) * s
    normal = np.abs(x) >= s * 2.0 ** -6
    assert np.all(np.abs(back - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal] * (1 + 1e-6))
    assert np.abs(back).max() <= np.abs(x).max() * (1 + 2.0 ** -4)
    assert O.quantize_e4m3(np.zeros(4))[1] == np.float32(1.0)


def _e4m3_decode(codes):
    """The value of each FP8 E4M3 byte from its bit fields, as the OCP 8-bit
    floating point specification defines them: bit 7 the sign, bits 6..3 the
    exponent with bias 7, bits 2..0 the mantissa; exponent 0 is subnormal
    (m / 8 * 2^-6); there is no infinity, and S.1111.111 is NaN.  Written
    from the format, not through any library conversion."""
    out = np.empty(codes.shape, np.float64)
    for idx, c in np.ndenumerate(np.asarray(codes, np.uint8)):
        c = int(c)
        sign = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            out[idx] = np.nan
        elif e == 0:
            out[idx] = sign * (m / 8.0) * 2.0 ** -6
        else:
            out[idx] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


def _e4m3_codes(byte_rows):
    return torch.tensor(np.asarray(byte_rows, np.uint8)).view(torch.float8_e4m3fn)


def test_e4m3_decoder_fixed_points():
    """The bit-field decoder itself, on values the format fixes: the largest
    finite code 0x7E = 448, the smallest normal 0x08 = 2^-6, the smallest
    subnormal 0x01 = 2^-9, 1.0 = 0x38, -1.5 = 0xBC, and NaN at 0x7F."""
    got = _e4m3_decode(np.array([0x7E, 0x08, 0x01, 0x38, 0xBC, 0x00, 0x80, 0x7F]))
    np.testing.assert_array_equal(got[:7], [448.0, 2.0 ** -6, 2.0 ** -9, 1.0, -1.5, 0.0, -0.0])
    assert np.isnan(got[7])


def test_out_proj_fp8_hand_worked():
    """A 2 x 3 by 3 x 2 product worked by hand.  y codes (row-major)
    [1, 2, 0.5; -1, 1.5, 0] with s_y = 2, the transposed weight's codes
    [1, 0, 2; 0.25, -1, 1] with s_w = 0.5.  Scaled: y = [2, 4, 1; -2, 3, 0],
    w^T = [0.5, 0, 1; 0.125, -0.5, 0.5], so
    out = [2*0.5 + 1*1, 2*0.125 - 4*0.5 + 1*0.5; -2*0.5, -2*0.125 - 3*0.5]
        = [2, -1.25; -1, -1.75]."""
    qy = _e4m3_codes([[0x38, 0x40, 0x30], [0xB8, 0x3C, 0x00]])
    qw_t = _e4m3_codes([[0x38, 0x00, 0x40], [0x28, 0xB8, 0x38]])
    got = O.out_proj_fp8(qy, np.float32(2.0), qw_t, np.float32(0.5))
    np.testing.assert_array_equal(got, [[2.0, -1.25], [-1.0, -1.75]])


def _out_proj_fp8_untransposed(qy, sy, qw_t, sw):
    """A planted mistake: the weight codes taken as [K, N] (no transpose)."""
    y = _e4m3_decode(qy.view(torch.uint8).numpy()) * float(sy)
    w = _e4m3_decode(qw_t.view(torch.uint8).numpy()) * float(sw)
    return y @ w


@pytest.mark.parametrize("M,K,N", [(5, 7, 3), (9, 16, 16)])
def test_out_proj_fp8_matches_bitfield_product(M, K, N):
    """out_proj_fp8 equals the float64 product of the bit-field-decoded,
    scaled codes, (s_y Y)(s_w W_t)^T, on random finite codes; non-square
    shapes catch a transposed weight, and the square case shows that the
    untransposed product differs."""
    r = np.random.default_rng(M * 100 + K)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    cy = r.choice(finite, size=(M, K))
    cw = r.choice(finite, size=(N, K))
    sy, sw = np.float32(0.013), np.float32(3.25)
    got = O.out_proj_fp8(_e4m3_codes(cy), sy, _e4m3_codes(cw), sw)
    want = (_e4m3_decode(cy) * float(sy)) @ (_e4m3_decode(cw) * float(sw)).T
    assert got.shape == (M, N)
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=1e-12 * np.abs(want).max())
    if K == N:
        wrong = _out_proj_fp8_untransposed(_e4m3_codes(cy), sy, _e4m3_codes(cw), sw)
        assert np.abs(wrong - want).max() > 1e-3 * np.abs(want).max()


# ----------------------------------------------------------- streaming ----
def _tag_segment(frames, d, T):
    """One head, one token per frame: frame f (global index) carries the key
    and value e_f, beta = 1, alpha = 1, so a state's diagonal lists the
    frames written into it (each at beta / (1 + beta) = 1/2)."""
    k = np.zeros((1, T, 1, 1, d))
    for i, f in enumerate(frames):
        k[0, i, 0, 0, f] = 1.0
    return {"k": k, "v": k.copy(), "beta": np.ones((1, T, 1, 1)), "alpha": np.ones((1, T, 1))}


@pytest.mark.parametrize("T1,T2,anchors", [(12, 13, 4), (10, 7, 4), (9, 11, 0)])
def test_stream_carried_state_holds_the_past(T1, T2, anchors):
    """Streaming ([P2] livestream setting): the second segment's forward
    scan starts from the state the first segment's forward scan ended with.
    With one tagged frame per key, every query of the second segment then
    reads each written frame of the first segment once, plus its own
    segment's written frames outside its window, and never a frame in its
    window or an anchor; an anchor query reads the carried past alone."""
    d = T1 + T2
    seg1 = _tag_segment(range(T1), d, T1)
    c1 = O.Cfg(B=1, T=T1, N=1, H=1, d_k=d, d_v=d, L=0, anchors=anchors)
    F1, _ = O.head_states(seg1, c1, 0, 0)
    seg2 = _tag_segment(range(T1, d), d, T2)
    seg2["fwd_init"] = F1[T1][None, None]
    c2 = O.Cfg(B=1, T=T2, N=1, H=1, d_k=d, d_v=d, L=0, anchors=anchors)
    F2, G2 = O.head_states(seg2, c2, 0, 0)
    past = {f for f in range(T1) if f not in O.anchor_frames(T1, anchors)}
    anc2 = set(O.anchor_frames(T2, anchors))
    for t in range(T2):
        held_d = np.diag(O.read_state(F2, G2, t, T2, 5, anchors))
        np.testing.assert_allclose(held_d[held_d > 1e-9], 0.5, atol=1e-12)
        held = set(np.nonzero(held_d > 1e-9)[0])
        if t in anc2:
            assert held == past
            continue
        lo, hi = O.window_frames(t, T2, 5)
        own = {T1 + f for f in range(T2) if f not in anc2 and not lo <= f < hi}
        assert held == past | own


def test_stream_forward_continues_one_long_scan():
    """Cutting a sequence in two and carrying the forward state gives the
    forward states of the uncut sequence (no anchors, so the cut writes
    every frame either way)."""
    shp = Shape(B=1, T=14, N=6, H=1, d_k=8, d_v=8, L=0)
    inp = make_inputs(shp, seed=3)
    long_cfg = O.Cfg(B=1, T=14, N=6, H=1, d_k=8, d_v=8, L=0, anchors=0)
    F, _ = O.head_states(inp, long_cfg, 0, 0)
    T1 = 6
    seg = {n: inp[n][:, T1:] for n in ("q", "k", "v", "beta", "alpha", "gate_sm", "gate_lin")}
    seg["fwd_init"] = F[T1][None, None]
    F2, _ = O.head_states(seg, O.Cfg(B=1, T=14 - T1, N=6, H=1, d_k=8, d_v=8, L=0, anchors=0), 0, 0)
    np.testing.assert_allclose(F2, F[T1:], rtol=0, atol=1e-13)


def test_stream_default_start_is_half_the_text_state():
    """fwd_init = S_x / 2 reproduces the call without it, bit for bit."""
    shp = Shape(B=1, T=12, N=8, H=2, d_k=16, d_v=16, L=6)
    inp = make_inputs(shp, seed=4)
    cfg = O.Cfg(B=1, T=12, N=8, H=2, d_k=16, d_v=16, L=6)
    half = np.stack([0.5 * O.text_state(inp["text_k"][0, :, h], inp["text_v"][0, :, h], inp["text_beta"][0, :, h],
                                        16, 16) for h in range(2)])[None]
    want = O.hybrid_attn(inp, cfg)
    got = O.hybrid_attn({**inp, "fwd_init": half}, cfg)
    np.testing.assert_array_equal(got, want)


# ------------------------------------------------------ ablation writes ----
def _explicit_token_chain(Sbar, K, V, beta):
    """The token-wise rule as explicit matrices: S_bar P_1 ... P_N + sum_i
    beta_i v_i k_i^T P_{i+1} ... P_N with P_i = I - beta_i k_i k_i^T."""
    d = K.shape[1]
    P = [np.eye(d) - b * np.outer(k, k) for k, b in zip(K, beta)]
    tail = [np.linalg.multi_dot(P[i + 1:] + [np.eye(d), np.eye(d)]) for i in range(len(P))]
    S = Sbar @ np.linalg.multi_dot(P + [np.eye(d)])
    for i in range(len(P)):
        S = S + beta[i] * np.outer(V[i], K[i]) @ tail[i]
    return S


def test_token_rule_equals_explicit_matrix_chain():
    Sbar, K, V, beta = _frame(7, 6, 5, seed=11)
    np.testing.assert_allclose(O.token_delta_update(Sbar, K, V, beta), _explicit_token_chain(Sbar, K, V, beta),
                               rtol=0, atol=1e-13)


def test_token_rule_recalls_the_last_write_exactly():
    """beta = 1 with a unit key is the classic delta rule's exact overwrite:
    afterwards S k_N = v_N whatever came before."""
    Sbar, K, V, _ = _frame(9, 8, 8, seed=12)
    S = O.token_delta_update(Sbar, K, V, np.ones(9))
    np.testing.assert_allclose(S @ K[-1], V[-1], atol=1e-13)


def test_token_rule_depends_on_order_the_others_do_not():
    """Only the token-wise rule sees the token order (the joint solve and the
    frame-level writes treat the frame as a set)."""
    Sbar, K, V, beta = _frame(6, 4, 4, seed=13)
    perm = np.arange(6)[::-1]
    for u in (0, 1):
        f = O.frame_update(u)
        np.testing.assert_allclose(f(Sbar, K, V, beta), f(Sbar, K[perm], V[perm], beta[perm]), atol=1e-13)
    a = O.token_delta_update(Sbar, K, V, beta)
    b = O.token_delta_update(Sbar, K[perm], V[perm], beta[perm])
    assert np.max(np.abs(a - b)) > 1e-3


def test_frame_rule_is_size_invariant_and_averages_orthogonal_writes():
    """Frame-level writes with the 1/N rescaling: N copies of one token write
    what the single token writes; with orthonormal keys (where the token rule's
    steps do not interact) the frame rule moves S_bar 1/N of the way the token
    rule does."""
    Sbar, K, V, beta = _frame(1, 6, 5, seed=14)
    one = O.frame_independent_update(Sbar, K, V, beta)
    many = O.frame_independent_update(Sbar, np.repeat(K, 9, 0), np.repeat(V, 9, 0), np.repeat(beta, 9))
    np.testing.assert_allclose(many, one, atol=1e-13)
    Q = np.linalg.qr(np.random.default_rng(15).standard_normal((6, 6)))[0][:4]
    V4 = np.random.default_rng(16).standard_normal((4, 5))
    b4 = np.array([0.3, 0.9, 0.5, 0.7])
    tok = O.token_delta_update(Sbar, Q, V4, b4)
    frm = O.frame_independent_update(Sbar, Q, V4, b4)
    np.testing.assert_allclose(frm - Sbar, (tok - Sbar) / 4, atol=1e-13)


@pytest.mark.parametrize("update", [0, 1, 2])
def test_every_write_is_the_affine_map_of_its_frame(update):
    """S = S_bar M + C for any S_bar, with (M, C) from variant_frame_map; for
    the joint solve (M, C) equal frame_map's closed form."""
    _, K, V, beta = _frame(11, 8, 6, seed=17)
    M, C = O.variant_frame_map(K, V, beta, update)
    f = O.frame_update(update)
    for s in range(3):
        Sbar = np.random.default_rng(20 + s).standard_normal((6, 8))
        np.testing.assert_allclose(f(Sbar, K, V, beta), Sbar @ M + C, atol=1e-12)
    if update == 0:
        M0, C0 = O.frame_map(K, V, beta)
        np.testing.assert_allclose(M, M0, atol=1e-13)
        np.testing.assert_allclose(C, C0, atol=1e-13)


def test_frame_rule_needs_its_rescaling_to_stay_non_expansive():
    """With unit keys and beta <= 1, I - A/N has spectral norm <= 1; the
    unrescaled I - A of a frame of many aligned tokens does not ([P5]: the
    joint solve needs no frame-size rescaling, unlike SANA-WM)."""
    r = np.random.default_rng(18)
    k0 = r.standard_normal(8)
    K = k0 + 0.1 * r.standard_normal((50, 8))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    beta = 1 / (1 + np.exp(-r.standard_normal(50)))
    M, _ = O.variant_frame_map(K, np.zeros((50, 8)), beta, 1)
    assert np.linalg.norm(M, 2) <= 1 + 1e-12
    A = (beta[:, None] * K).T @ K
    assert np.linalg.norm(np.eye(8) - A, 2) > 1


def test_softmax_lse_normalises_the_softmax_output():
    """exp(s q.k - LSE) over the allowed keys are the softmax weights: they
    sum to one and, times v and the gate, give the softmax slot of the output."""
    shp = Shape(B=1, T=12, N=4, H=2, d_k=8, d_v=8, L=0)
    inp = {k: np.asarray(v, np.float64) for k, v in make_inputs(shp, seed=31).items() if not k.endswith("_bits")}
    cfg = O.Cfg(B=1, T=12, N=4, H=2, d_k=8, d_v=8, L=0, softmax_scale=2.0)
    lse = O.softmax_lse(inp, cfg)
    allowed = O.frame_mask(12, 5, 4)
    y = O.hybrid_attn(inp, cfg)[..., 0, :]
    for h in range(2):
        for t in (0, 3, 7, 11):
            keys = np.flatnonzero(allowed[t])
            K = inp["k"][0, keys, :, h].reshape(-1, 8)
            V = inp["v"][0, keys, :, h].reshape(-1, 8)
            W = np.exp(2.0 * inp["q"][0, t, :, h] @ K.T - lse[0, t, :, h][:, None])
            np.testing.assert_allclose(W.sum(axis=1), 1.0, rtol=0, atol=1e-12)
            np.testing.assert_allclose(O.sigmoid(inp["gate_sm"][0, t, :, h]) * (W @ V), y[0, t, :, h], rtol=0,
                                       atol=1e-12)


def test_softmax_lse_two_keys_closed_form():
    """T = 2 (both frames anchors) with one token per frame: each query sees
    the two keys, LSE = ln(exp(s q.k0) + exp(s q.k1))."""
    shp = Shape(B=1, T=2, N=1, H=1, d_k=4, d_v=4, L=0)
    inp = {k: np.asarray(v, np.float64) for k, v in make_inputs(shp, seed=32).items() if not k.endswith("_bits")}
    cfg = O.Cfg(B=1, T=2, N=1, H=1, d_k=4, d_v=4, L=0, softmax_scale=3.0)
    lse = O.softmax_lse(inp, cfg)
    for t in range(2):
        q = inp["q"][0, t, 0, 0]
        a, b = 3.0 * q @ inp["k"][0, 0, 0, 0], 3.0 * q @ inp["k"][0, 1, 0, 0]
        assert abs(lse[0, t, 0, 0] - np.log(np.exp(a) + np.exp(b))) < 1e-13


@pytest.mark.parametrize("T", [2, 7, 10, 12, 23, 90, 102])
@pytest.mark.parametrize("anchors", [0, 4])
def test_frame_mask_is_symmetric(T, anchors):
    """The window (chunks within one of each other) and the anchors (an anchor
    frame sees and is seen by every frame) are symmetric relations: the query
    frames that see key frame f are the frames f itself sees. The key-side
    backward kernels of the softmax walk the query tiles of a key frame by
    this."""
    m = O.frame_mask(T, 5, anchors)
    assert np.array_equal(m, m.T)
    assert np.all(np.diag(m))

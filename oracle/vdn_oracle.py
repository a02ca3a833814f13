"""Plain fp64 CPU oracle for the Video DeltaNet hybrid attention core.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may
import this module.  The product path (the CUDA library and its Python
binding) never calls it and shares no code with it.

Every function computes the method *as the pages define it*, in float64, with
NumPy's ``solve`` / ``@`` as the only library steps, so that a reader can
check it against the pages by eye.  Nothing is blocked, fused or reordered.

Sources (web pages on "Video DeltaNet: A Video-Native Hybrid Attention for
Livestream Video Generation", arXiv 2609.20744):

* [P1] PaperDaily digest "伯克利与Impossible视频生成:14.3秒视频6.70秒去噪"
  (longzhangge.com), sections 二 (local window + anchors), 三 (bidirectional
  states, half-text init, gates, RMSNorm), 四 (frame-wise joint write).
* [P2] shd-paper.top abstract page of arXiv 2609.20744.
* [P4] deepmagic.app post "生成比播放還快：Video DeltaNet 用 11 秒產出 14 秒
  768p 影片", section "用兩條分支取代一條" (closed form, 4-way anchors).
* [P5] aimodeling.com news "video-deltanet-h3-hybrid-attention", section
  "The VDN split" (frame-wise (I+A) solve, non-expansive, saturation).
* The page at juejin.cn (per-frame-independent kernel, K=3 window, optical
  flow gate) contradicts the four others and is NOT followed.

Readings taken where the pages are silent (each one is listed with its
reason in the design notes of the repository):

* alpha enters as the inherited state S_bar = alpha_t * S_{t-1};
* both scan directions use the same alpha_t, beta, k, v of frame t;
* anchor frames are an identity step of either scan (no write, no decay);
* an anchor query frame reads S_init_f + S_init_b (its softmax already
  sees every frame); ``anchor_read="chunk"`` gives the other reading;
* the window is clipped at the sequence ends;
* softmax scale defaults to 1/sqrt(d_k); RMSNorm is over d_v with eps;
* gates are elementwise sigmoid(logit) over [.., d_v];
* the output keeps the two gated branches apart on a size-2 axis
  (slot 0 = softmax, slot 1 = linear), or sums them (out_mode=1).

Parity: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, an independent least-squares route, brute
force on tiny inputs, library routines and the pages' printed densities.
The end-to-end output has no printed worked example on the pages (no page
prints one), so the end-to-end *value* is pinned only through its parts.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# configuration
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class Cfg:
    """Problem sizes and switches.  Layouts used throughout:

    q, k, v, gate_sm, gate_lin : [B, T, N, H, d]
    beta : [B, T, N, H]     alpha : [B, T, H]
    text_k, text_v : [B, L, H, d]   text_beta : [B, L, H]
    """
    B: int
    T: int
    N: int
    H: int
    d_k: int
    d_v: int
    L: int = 0
    chunk: int = 5
    anchors: int = 4          # 0 = none, 4 = 4-way first/last-frame anchors
    softmax_scale: float = 0.0  # <= 0 -> 1/sqrt(d_k)
    rms_eps: float = 1e-6
    out_mode: int = 0         # 0 = [.., 2, d_v] slots, 1 = summed [.., d_v]
    update: int = 0           # frame write: 0 joint solve, 1 frame-level independent, 2 token-wise

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else 1.0 / np.sqrt(self.d_k)


# ---------------------------------------------------------------------------
# the hybrid mask  ([P1] 二; [P4] 用兩條分支取代一條; [P5] The VDN split)
# ---------------------------------------------------------------------------
def num_chunks(T: int, chunk: int) -> int:
    """Chunks of `chunk` consecutive latent frames; a short last chunk if
    T is not a multiple of the chunk size."""
    return -(-T // chunk)


def anchor_frames(T: int, anchors: int) -> tuple:
    """The boundary anchors are the first and the last latent frame."""
    if anchors == 0:
        return ()
    return tuple(sorted({0, T - 1}))


def frame_mask(T: int, chunk: int = 5, anchors: int = 4) -> np.ndarray:
    """allowed[tq, tk]: may a query in frame tq attend by softmax to a key in
    frame tk?  A query chunk sees itself and its two neighbour chunks; every
    frame sees the anchor frames and the anchor frames see every frame."""
    c = np.arange(T) // chunk
    allowed = np.abs(c[:, None] - c[None, :]) <= 1
    for a in anchor_frames(T, anchors):
        allowed[:, a] = True
        allowed[a, :] = True
    return allowed


def token_mask(T: int, N: int, chunk: int = 5, anchors: int = 4) -> np.ndarray:
    """The frame mask expanded to tokens (frame-major, N tokens per frame)."""
    return np.kron(frame_mask(T, chunk, anchors), np.ones((N, N), dtype=bool)).astype(bool)


def mask_density(T: int, chunk: int = 5, anchors: int = 4) -> float:
    """Fraction of (query, key) video pairs kept on the softmax path."""
    return float(frame_mask(T, chunk, anchors).mean())


def window_frames(t: int, T: int, chunk: int = 5) -> tuple:
    """[lo, hi): the frames of the query chunk and its two neighbours,
    clipped to the sequence."""
    c = t // chunk
    return max(0, chunk * (c - 1)), min(T, chunk * (c + 2))


# ---------------------------------------------------------------------------
# Video Delta Attention  ([P1] 四; [P4] closed form; [P5] The VDN split)
# ---------------------------------------------------------------------------
def gram_write(K: np.ndarray, V: np.ndarray, beta: np.ndarray):
    """A = sum_i beta_i k_i k_i^T  (d_k x d_k), the beta-weighted key Gram
    matrix, and B = sum_i beta_i v_i k_i^T  (d_v x d_k), the value-key write
    matrix, over the n tokens of one frame.  K [n, d_k], V [n, d_v], beta [n]."""
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    Kb = K * np.asarray(beta, F64)[:, None]
    return K.T @ Kb, V.T @ Kb


def vda_update(S_bar: np.ndarray, K: np.ndarray, V: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """The frame-wise joint write: the S that minimises
        ||S - S_bar||_F^2 + sum_i beta_i ||S k_i - v_i||^2
    over all tokens of the frame at once, i.e. the closed form
        S = (S_bar + B)(I + A)^{-1}.
    (I + A) is symmetric, so S^T solves (I + A) S^T = (S_bar + B)^T."""
    A, Bw = gram_write(K, V, beta)
    G = np.eye(A.shape[0]) + A
    return np.linalg.solve(G, (np.asarray(S_bar, F64) + Bw).T).T


def frame_map(K: np.ndarray, V: np.ndarray, beta: np.ndarray):
    """The frame update written as an affine map of the inherited state:
    S = S_bar M + C with M = (I + A)^{-1} and C = B M (the same closed form,
    expanded).  Returned for intermediate-value checks."""
    A, Bw = gram_write(K, V, beta)
    M = np.linalg.solve(np.eye(A.shape[0]) + A, np.eye(A.shape[0]))
    return M, Bw @ M


# ---------------------------------------------------------------------------
# ablation baselines of the frame write  ([P4] VDA paragraph: earlier
# frame-level updates such as SANA-WM let every token update a frozen state on
# its own; [P5] The VDN split: unlike SANA-WM, no frame-size rescaling is
# needed; [P1] 四: the classic token-by-token delta rule is the one-token case)
# ---------------------------------------------------------------------------
def frame_independent_update(S_bar: np.ndarray, K: np.ndarray, V: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """Frame-level independent writes (the SANA-WM style baseline): each token
    i proposes the delta-rule step beta_i (v_i - S_bar k_i) k_i^T against the
    same frozen inherited state, and the N proposals are summed and divided
    by the frame size N (the rescaling that keeps the map non-expansive)."""
    S_bar = np.asarray(S_bar, F64)
    K, V, beta = np.asarray(K, F64), np.asarray(V, F64), np.asarray(beta, F64)
    resid = V - K @ S_bar.T                     # row i: v_i - S_bar k_i
    return S_bar + (beta[:, None] * resid).T @ K / K.shape[0]


def token_delta_update(S_bar: np.ndarray, K: np.ndarray, V: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """The token-wise delta rule: tokens write one after another in token
    order, S <- S + beta_i (v_i - S k_i) k_i^T, each against the state the
    previous token left."""
    S = np.array(S_bar, F64)
    for i in range(K.shape[0]):
        k = np.asarray(K[i], F64)
        S = S + beta[i] * np.outer(np.asarray(V[i], F64) - S @ k, k)
    return S


def frame_update(update: int):
    """The frame write of mode `update` (0 joint solve, 1 frame-level
    independent, 2 token-wise delta rule)."""
    return {0: vda_update, 1: frame_independent_update, 2: token_delta_update}[update]


def variant_frame_map(K: np.ndarray, V: np.ndarray, beta: np.ndarray, update: int):
    """Every mode's write is affine in the inherited state, S = S_bar M + C:
    M is the write of the identity with zero values, C the write of the zero
    state.  Returned for intermediate-value checks of the per-frame maps."""
    f = frame_update(update)
    dk, dv = K.shape[1], V.shape[1]
    M = f(np.eye(dk), K, np.zeros((K.shape[0], dk)), beta)
    C = f(np.zeros((dv, dk)), K, V, beta)
    return M, C


def text_state(text_k: np.ndarray, text_v: np.ndarray, text_beta: np.ndarray, d_v: int, d_k: int) -> np.ndarray:
    """Text is pre-written by one joint solve from the zero state over the L
    text tokens ([P1] 三: the prompt is written into both states, half each).
    Returns the full text state S_x; each direction starts from S_x / 2."""
    if text_k is None or len(text_k) == 0:
        return np.zeros((d_v, d_k))
    return vda_update(np.zeros((d_v, d_k)), text_k, text_v, text_beta)


def forward_states(S0, k, v, beta, alpha, anchors: int = 4, update=vda_update) -> np.ndarray:
    """Forward scan for one (batch, head).  k [T, N, d_k], v [T, N, d_v],
    beta [T, N], alpha [T].  F[t] is the state that covers frames < t
    (F[0] = S0); at a non-anchor frame the inherited state is alpha_t F[t]
    and the frame is written jointly (or by the ablation write `update`);
    anchor frames are not written."""
    T = k.shape[0]
    anc = set(anchor_frames(T, anchors))
    F = np.empty((T + 1,) + np.shape(S0))
    F[0] = S0
    for t in range(T):
        if t in anc:
            F[t + 1] = F[t]
        else:
            F[t + 1] = update(alpha[t] * F[t], k[t], v[t], beta[t])
    return F


def backward_states(S0, k, v, beta, alpha, anchors: int = 4, update=vda_update) -> np.ndarray:
    """Backward scan: G[t] covers frames >= t (G[T] = S0), built from the
    last frame down with the same per-frame update (the tokens of a frame
    keep their order under the token-wise rule)."""
    T = k.shape[0]
    anc = set(anchor_frames(T, anchors))
    G = np.empty((T + 1,) + np.shape(S0))
    G[T] = S0
    for t in range(T - 1, -1, -1):
        if t in anc:
            G[t] = G[t + 1]
        else:
            G[t] = update(alpha[t] * G[t + 1], k[t], v[t], beta[t])
    return G


def chunk_maps(k, v, beta, alpha, chunk: int = 5, anchors: int = 4):
    """Chunk composition of the frame maps for one (batch, head).

    Each written frame acts on the state as the affine map S -> alpha_t S M_t
    + C_t (frame_map; [P4] closed form), so the frames of one chunk compose
    into one map of the same form (the north star's "prefix composition of
    the affine frame maps where it helps").  For chunk c, with its written
    frames f_1 < ... < f_n (anchor frames are identity maps and drop out):

    * forward (frames in increasing order): S -> Lam_c S P_c + Cf_c with
      P_c = M_{f_1} ... M_{f_n}, Lam_c = alpha_{f_1} ... alpha_{f_n}, and
      Cf_c by Horner's rule, Cf <- alpha_f Cf M_f + C_f from Cf = 0;
    * backward (decreasing order): S -> Lam_c S P_c^T + Cb_c, since each
      M_f = (I + A_f)^{-1} is symmetric and the reversed product is the
      transpose; Cb <- alpha_f Cb M_f + C_f for f from f_n down to f_1.

    Returns P [C, d_k, d_k], Cf, Cb [C, d_v, d_k], Lam [C]; a chunk with no
    written frame gives the identity map (P = I, Cf = Cb = 0, Lam = 1)."""
    T, d_k, d_v = k.shape[0], k.shape[-1], v.shape[-1]
    anc = set(anchor_frames(T, anchors))
    nc = num_chunks(T, chunk)
    P = np.empty((nc, d_k, d_k))
    Cf = np.empty((nc, d_v, d_k))
    Cb = np.empty((nc, d_v, d_k))
    Lam = np.empty(nc)
    for c in range(nc):
        frames = [f for f in range(c * chunk, min((c + 1) * chunk, T)) if f not in anc]
        maps = {f: frame_map(k[f], v[f], beta[f]) for f in frames}
        Pc, cf, cb, lam = np.eye(d_k), np.zeros((d_v, d_k)), np.zeros((d_v, d_k)), 1.0
        for f in frames:
            M, Cm = maps[f]
            Pc = Pc @ M
            cf = alpha[f] * cf @ M + Cm
            lam *= alpha[f]
        for f in reversed(frames):
            M, Cm = maps[f]
            cb = alpha[f] * cb @ M + Cm
        P[c], Cf[c], Cb[c], Lam[c] = Pc, cf, cb, lam
    return P, Cf, Cb, Lam


def chunk_scan(S0, P, Cf, Cb, Lam):
    """The two scans stepped by whole chunks with the maps of chunk_maps.
    Returns Fc [C+1, ...] with Fc[j] the forward state over the first j
    chunks (Fc[0] = S0) and Gc [C+1, ...] with Gc[j] the backward state over
    chunks >= j (Gc[C] = S0): the forward / backward states at every chunk
    boundary, which is all the read needs."""
    nc = len(Lam)
    Fc = np.empty((nc + 1,) + np.shape(S0))
    Gc = np.empty((nc + 1,) + np.shape(S0))
    Fc[0] = S0
    for c in range(nc):
        Fc[c + 1] = Lam[c] * Fc[c] @ P[c] + Cf[c]
    Gc[nc] = S0
    for c in range(nc - 1, -1, -1):
        Gc[c] = Lam[c] * Gc[c + 1] @ P[c].T + Cb[c]
    return Fc, Gc


def read_state(F, G, t: int, T: int, chunk: int = 5, anchors: int = 4, anchor_read: str = "text"):
    """The state a query in frame t reads: the forward state over the frames
    before its window plus the backward state over the frames after it
    ([P1] 三; [P4] the two regions do not overlap).  An anchor query frame
    reads the two half-text initial states (anchor_read="text"), or its chunk
    window like any other frame (anchor_read="chunk")."""
    if anchor_read == "text" and t in anchor_frames(T, anchors):
        return F[0] + G[T]
    lo, hi = window_frames(t, T, chunk)
    return F[lo] + G[hi]


def read_table(F, G, T: int, chunk: int = 5, anchors: int = 4):
    """Per query chunk c the summed read state, plus one entry (index C) for
    the anchor query frames.  Returned for intermediate-value checks."""
    C = num_chunks(T, chunk)
    R = np.empty((C + 1,) + F.shape[1:])
    for c in range(C):
        lo, hi = window_frames(c * chunk, T, chunk)
        R[c] = F[lo] + G[hi]
    R[C] = F[0] + G[T]
    return R


def out_proj(y, W):
    """The layer's output projection over the core's concat axis ([P1] 三:
    each gated branch is projected back to the model width; with the two
    branches on a size-2 axis, one product with the stacked weight is the
    sum of the two projections).  y [..., H, 2, d_v] is flattened per token
    to H*2*d_v values, row (h*2 + slot)*d_v + i, times W [H*2*d_v, n]."""
    y = np.asarray(y, F64)
    H, two, dv = y.shape[-3:]
    return y.reshape(y.shape[:-3] + (H * two * dv,)) @ np.asarray(W, F64)


def quantize_e4m3(x):
    """FP8 E4M3 with one scale per tensor (deepmagic post, section 實測數據:
    FP8 linear layers): s = amax|x| / 448 in float32 (448 is the largest
    finite e4m3; s = 1 for an all-zero tensor), q = e4m3(x * (1 / s)) with the
    product in float32 and the rounding to nearest even of torch's
    float8_e4m3fn conversion (a library routine).  Returns the codes as a
    torch float8 tensor and s (float32), so that x ~ q * s."""
    import torch
    x32 = np.asarray(x, np.float32)
    amax = np.float32(np.abs(x32).max()) if x32.size else np.float32(0.0)
    s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    inv = np.float32(np.float32(1.0) / s)
    return torch.from_numpy(np.ascontiguousarray(x32 * inv)).to(torch.float8_e4m3fn), s


def out_proj_fp8(qy, sy, qw_t, sw):
    """The output projection with e4m3 operands: (s_y q_y)(s_w q_w_t)^T in
    float64, q_y [M, K], q_w_t [N, K] (the weight transposed)."""
    y = qy.to(dtype=__import__("torch").float64).numpy() * float(sy)
    w = qw_t.to(dtype=__import__("torch").float64).numpy() * float(sw)
    return y @ w.T


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, F64)))


def rms_gate(o, g, eps: float, weight=None):
    """Linear-branch epilogue ([P1] 三): RMS-normalise over d_v, then the
    content-dependent sigmoid gate.  o, g [..., d_v]."""
    o = np.asarray(o, F64)
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    if weight is not None:
        r = r * np.asarray(weight, F64)
    return sigmoid(g) * r


# ---------------------------------------------------------------------------
# softmax branch  ([P1] 二; [P4]; [P5])
# ---------------------------------------------------------------------------
def softmax_attend(q, keys, vals, scale: float):
    """Plain softmax attention of queries q [n, d_k] over keys [m, d_k]."""
    s = scale * (np.asarray(q, F64) @ np.asarray(keys, F64).T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ np.asarray(vals, F64)


def text_cross_attn(q_bh, text_k_bh, text_v_bh, scale: float):
    """The block's softmax cross-attention from the video tokens to the text
    tokens ([P1] 三: the prompt reaches the block through cross-attention as
    well as through the half-text states): every query of one (batch, head),
    q_bh [T, N, d_k], over all L text tokens of that batch, no mask, no gate.
    Returns [T, N, d_v]."""
    T, N, dk = np.shape(q_bh)
    o = softmax_attend(np.reshape(q_bh, (T * N, dk)), text_k_bh, text_v_bh, scale)
    return o.reshape(T, N, -1)


def softmax_frame(q_t, k_bh, v_bh, t: int, T: int, chunk: int, anchors: int, scale: float):
    """Softmax output for the queries of frame t of one (batch, head):
    keys are the tokens of every frame the frame mask allows."""
    allowed = np.nonzero(frame_mask(T, chunk, anchors)[t])[0]
    keys = k_bh[allowed].reshape(-1, k_bh.shape[-1])
    vals = v_bh[allowed].reshape(-1, v_bh.shape[-1])
    return softmax_attend(q_t, keys, vals, scale)


def softmax_dense_masked(q_bh, k_bh, v_bh, T, N, chunk, anchors, scale):
    """Dense attention over all T*N video tokens with the explicit token mask
    (masked logits = -inf).  Only for small sizes."""
    Q = np.asarray(q_bh, F64).reshape(T * N, -1)
    K = np.asarray(k_bh, F64).reshape(T * N, -1)
    V = np.asarray(v_bh, F64).reshape(T * N, -1)
    s = scale * (Q @ K.T)
    s = np.where(token_mask(T, N, chunk, anchors), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return (p @ V).reshape(T, N, -1)


# ---------------------------------------------------------------------------
# the whole core
# ---------------------------------------------------------------------------
def softmax_lse(inp: dict, cfg: Cfg) -> np.ndarray:
    """[B, T, N, H]: the log-sum-exp ln sum_j exp(s q . k_j) of every query row
    over the keys its mask allows ([P1] 二; the normaliser of the softmax
    branch, which a backward pass reuses)."""
    allowed = frame_mask(cfg.T, cfg.chunk, cfg.anchors)
    out = np.empty((cfg.B, cfg.T, cfg.N, cfg.H))
    for b in range(cfg.B):
        for h in range(cfg.H):
            for t in range(cfg.T):
                keys = np.flatnonzero(allowed[t])
                K = np.asarray(inp["k"][b, keys, :, h], F64).reshape(len(keys) * cfg.N, -1)
                S = cfg.scale * (np.asarray(inp["q"][b, t, :, h], F64) @ K.T)
                m = S.max(axis=1)
                out[b, t, :, h] = m + np.log(np.exp(S - m[:, None]).sum(axis=1))
    return out


def head_states(inp: dict, cfg: Cfg, b: int, h: int):
    """F, G (forward / backward states for every frame boundary) of one
    (batch, head), both started from half the text state; with
    inp["fwd_init"] [B, H, d_v, d_k] the forward scan starts from that state
    instead (streaming: the state the previous segment's forward scan ended
    with, carried across appended chunks, [P2] livestream setting)."""
    if cfg.L > 0 and inp.get("text_k") is not None:
        Sx = text_state(inp["text_k"][b, :, h], inp["text_v"][b, :, h], inp["text_beta"][b, :, h],
                        cfg.d_v, cfg.d_k)
    elif inp.get("init_state") is not None:
        Sx = np.asarray(inp["init_state"][b, h], F64)
    else:
        Sx = np.zeros((cfg.d_v, cfg.d_k))
    S0 = 0.5 * Sx
    k = inp["k"][b, :, :, h]
    v = inp["v"][b, :, :, h]
    beta = inp["beta"][b, :, :, h]
    alpha = inp["alpha"][b, :, h]
    F0 = np.asarray(inp["fwd_init"][b, h], F64) if inp.get("fwd_init") is not None else S0
    f = frame_update(cfg.update)
    F = forward_states(F0, k, v, beta, alpha, cfg.anchors, f)
    G = backward_states(S0, k, v, beta, alpha, cfg.anchors, f)
    return F, G


def hybrid_attn(inp: dict, cfg: Cfg, anchor_read: str = "text", softmax: str = "frames") -> np.ndarray:
    """The video-to-video hybrid attention core for every token.

    Returns Y [B, T, N, H, 2, d_v] (slot 0 = gated softmax branch, slot 1 =
    gated, RMS-normalised linear branch) or, with out_mode=1, their sum
    [B, T, N, H, d_v].  softmax="dense" uses the explicit token mask."""
    B, T, N, H, dv = cfg.B, cfg.T, cfg.N, cfg.H, cfg.d_v
    Y = np.zeros((B, T, N, H, 2, dv))
    w = inp.get("rms_weight")
    for b in range(B):
        for h in range(H):
            F, G = head_states(inp, cfg, b, h)
            q_bh = np.asarray(inp["q"][b, :, :, h], F64)
            k_bh = np.asarray(inp["k"][b, :, :, h], F64)
            v_bh = np.asarray(inp["v"][b, :, :, h], F64)
            wh = None if w is None else w[h]
            if softmax == "dense":
                osm = softmax_dense_masked(q_bh, k_bh, v_bh, T, N, cfg.chunk, cfg.anchors, cfg.scale)
            for t in range(T):
                R = read_state(F, G, t, T, cfg.chunk, cfg.anchors, anchor_read)
                o_lin = q_bh[t] @ R.T                      # o = R q per token
                Y[b, t, :, h, 1] = rms_gate(o_lin, inp["gate_lin"][b, t, :, h], cfg.rms_eps, wh)
                o = osm[t] if softmax == "dense" else softmax_frame(
                    q_bh[t], k_bh, v_bh, t, T, cfg.chunk, cfg.anchors, cfg.scale)
                Y[b, t, :, h, 0] = sigmoid(inp["gate_sm"][b, t, :, h]) * o
    if cfg.out_mode == 1:
        return Y.sum(axis=4)
    return Y


def hybrid_attn_rows(inp: dict, cfg: Cfg, rows, anchor_read: str = "text") -> np.ndarray:
    """The same core evaluated only at the listed (b, t, n, h) positions.
    Returns [len(rows), 2, d_v] (softmax slot, linear slot), unsummed."""
    rows = [tuple(int(x) for x in r) for r in rows]
    states = {}
    out = np.zeros((len(rows), 2, cfg.d_v))
    w = inp.get("rms_weight")
    for i, (b, t, n, h) in enumerate(rows):
        if (b, h) not in states:
            states[(b, h)] = head_states(inp, cfg, b, h)
        F, G = states[(b, h)]
        q = np.asarray(inp["q"][b, t, n, h], F64)
        R = read_state(F, G, t, cfg.T, cfg.chunk, cfg.anchors, anchor_read)
        out[i, 1] = rms_gate(R @ q, inp["gate_lin"][b, t, n, h], cfg.rms_eps, None if w is None else w[h])
        k_bh = inp["k"][b, :, :, h]
        v_bh = inp["v"][b, :, :, h]
        o = softmax_frame(q[None], k_bh, v_bh, t, cfg.T, cfg.chunk, cfg.anchors, cfg.scale)[0]
        out[i, 0] = sigmoid(inp["gate_sm"][b, t, n, h]) * o
    return out


def vda_intermediates(inp: dict, cfg: Cfg, b: int, h: int):
    """Per-frame maps (M_t, C_t), the text state S_x and the per-chunk read
    table R of one (batch, head), for checking a kernel stage by stage."""
    T = cfg.T
    Ms = np.zeros((T, cfg.d_k, cfg.d_k))
    Cs = np.zeros((T, cfg.d_v, cfg.d_k))
    anc = set(anchor_frames(T, cfg.anchors))
    for t in range(T):
        if t in anc:
            continue
        kk, vv, bb = inp["k"][b, t, :, h], inp["v"][b, t, :, h], inp["beta"][b, t, :, h]
        Ms[t], Cs[t] = frame_map(kk, vv, bb) if cfg.update == 0 else variant_frame_map(kk, vv, bb, cfg.update)
    F, G = head_states(inp, cfg, b, h)
    # the backward scan always starts from half the text state (the forward
    # one from fwd_init when that is given)
    return {"M": Ms, "C": Cs, "S_init": G[T], "F": F, "G": G,
            "R": read_table(F, G, T, cfg.chunk, cfg.anchors)}

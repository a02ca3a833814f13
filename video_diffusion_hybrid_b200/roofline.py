"""Algorithmic work of the hybrid attention core, for roofline fractions.

These are counts of what the method must compute or move at minimum
(independent of any kernel's blocking), used by the benchmark:

* softmax: 4 * d * (allowed query-key token pairs) per head -- QK^T and PV,
  one multiply-add (2 flops) each per pair and dimension;
* Gram/write: 2 * N * (d_k^2 + d_v d_k) per non-anchor frame-head;
* read: 2 * d_k * d_v per query token and head;
* bytes: each input read once and each output written once.
"""
from __future__ import annotations


def allowed_frame_pairs(T: int, chunk: int = 5, anchors: int = 4) -> int:
    """Number of (query frame, key frame) pairs on the softmax path."""
    total = 0
    for tq in range(T):
        if anchors and tq in (0, T - 1):
            total += T
            continue
        c = tq // chunk
        lo, hi = max(0, (c - 1) * chunk), min(T, (c + 2) * chunk)
        n = hi - lo
        if anchors:
            n += (1 if lo > 0 else 0) + (1 if hi < T and T - 1 >= hi else 0)
        total += n
    return total


def softmax_flops(B, T, N, H, d, chunk=5, anchors=4) -> float:
    return 4.0 * d * allowed_frame_pairs(T, chunk, anchors) * N * N * H * B


def gram_flops(B, T, N, H, d, anchors=4) -> float:
    frames = T - (2 if anchors and T >= 2 else 0)
    return 2.0 * N * (2 * d * d) * frames * H * B


def read_flops(B, T, N, H, d) -> float:
    return 2.0 * d * d * B * T * N * H


def softmax_bytes(B, T, N, H, d, elem=2, out_slot_bytes=None) -> float:
    """q, k, v, gate_sm read once; y softmax slot written once."""
    tok = B * T * N * H * d
    return tok * elem * 4 + tok * (out_slot_bytes or elem)


def written_frames(T: int, anchors: int = 4) -> int:
    return T - (2 if anchors and T >= 2 else 0)


def gram_bytes(B, T, N, H, d, anchors=4, elem=2) -> float:
    """Per-frame write: k, v (elem bytes) and beta (fp32) of the written frames
    read once; A_t, B_t (fp32 d x d) written once."""
    nw = written_frames(T, anchors)
    return nw * B * H * (N * (2 * d * elem + 4) + 2 * d * d * 4)


def sweep_flops(B, T, H, d, anchors=4, with_c=True) -> float:
    """SPD solve per written frame-head: d pivots of a d x d rank-one update
    (d^3 multiply-adds), plus C = B M (d^3 multiply-adds) where the scan
    needs C (the tensor-core scan forms (alpha S + B) M itself: with_c=False)."""
    return (4.0 if with_c else 2.0) * d ** 3 * written_frames(T, anchors) * B * H


def variant_map_flops(B, T, N, H, d, anchors=4, update=2) -> float:
    """The ablation writes' per-frame maps: every token updates each of the
    2d rows of the stacked [M'; C'] (d multiply-adds a row), and the
    token-wise rule first takes each row's dot product with the key (d more)."""
    per_token = (4.0 if update == 2 else 2.0) * 2 * d * d
    return per_token * N * written_frames(T, anchors) * B * H


def scan_bytes(B, T, H, d, chunk=5, anchors=4) -> float:
    """Both directions read every written frame's M_t (as its bf16 hi/lo
    split, 4 bytes an entry) and C_t (fp32); the chunk-boundary states (fp32,
    C + 1 per direction) are written once and the start state read once."""
    C = (T + chunk - 1) // chunk
    nw = written_frames(T, anchors)
    return B * H * (2 * nw * 2 * d * d * 4 + 2 * (C + 1) * d * d * 4 + 2 * d * d * 4)


def read_bytes(B, T, N, H, d, elem=2, y_elem=4) -> float:
    """q and gate_lin read once, the linear slot of y written once (the read
    table itself is a few MB and stays in L2)."""
    return B * T * N * H * d * (2 * elem + y_elem)


def fp32_simt_tflops(sm_mhz: float, sms: int = 148) -> float:
    """SIMT fp32 peak: 128 FMA lanes per SM per clock, 2 flops each."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12

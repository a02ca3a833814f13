"""The benchmark's algorithmic work counts (roofline.py) against independent
counts: the oracle's explicit frame mask for the softmax pairs, and sizes
worked out from the tensors' shapes for the byte counts.  Every roofline
fraction the benchmark reports divides one of these counts by a time, so a
wrong count would misstate every fraction."""
import numpy as np
import pytest

from oracle import vdn_oracle as O
from video_diffusion_hybrid_b200 import roofline as R


@pytest.mark.parametrize("T,chunk,anchors", [(2, 5, 4), (3, 5, 4), (7, 5, 0), (10, 5, 4), (23, 5, 4), (90, 5, 4),
                                             (180, 5, 4), (25, 5, 0)])
def test_allowed_frame_pairs_is_the_mask_count(T, chunk, anchors):
    # the oracle's boolean (query frame, key frame) mask, counted
    assert R.allowed_frame_pairs(T, chunk, anchors) == int(np.count_nonzero(O.frame_mask(T, chunk, anchors)))


def test_softmax_flops_at_768p():
    # 4 d flops per allowed token pair: QK^T and PV, one multiply-add each per dimension
    T, N, H, d = 90, 1008, 24, 128
    pairs = int(np.count_nonzero(O.frame_mask(T, 5, 4))) * N * N * H
    assert R.softmax_flops(1, T, N, H, d) == 4.0 * d * pairs
    # the density the pages print for this shape (19.98 %) sets the size: about 20.2 TFLOP
    assert R.softmax_flops(1, T, N, H, d) / (4.0 * d * (T * N) ** 2 * H) == pytest.approx(
        O.mask_density(T, 5, 4), rel=1e-12)
    assert R.softmax_flops(1, T, N, H, d) == pytest.approx(20.2e12, rel=2e-3)


def test_byte_counts_from_tensor_sizes():
    B, T, N, H, d = 1, 90, 1008, 24, 128
    tok = B * T * N * H
    written = T - 2  # the two anchor frames take no write
    # read: q and gate_lin in (bf16), y's linear slot out (bf16 here)
    assert R.read_bytes(B, T, N, H, d, elem=2, y_elem=2) == tok * d * 2 * 3
    # Gram: k and v (bf16) and beta (fp32) of the written frames in, A_t and B_t (fp32) out
    k_v_beta = written * N * H * (2 * d * 2 + 4)
    a_b = written * H * 2 * d * d * 4
    assert R.gram_bytes(B, T, N, H, d) == k_v_beta + a_b
    # scan: per direction, every written frame's M_t split (2 bf16 an entry) and B_t (fp32),
    # the C + 1 boundary states written (fp32) and the start state read (fp32)
    C = (T + 4) // 5
    per_dir = written * d * d * (4 + 4) + (C + 1) * d * d * 4 + d * d * 4
    assert R.scan_bytes(B, T, H, d) == H * 2 * per_dir


def test_sweep_flops_counts_the_inverse_and_the_product():
    # the inverse of a d x d SPD matrix by the sweep: d^3 multiply-adds; C = B M: d^3 more
    d, H, T = 128, 24, 90
    n = (T - 2) * H
    assert R.sweep_flops(1, T, H, d, with_c=False) == 2.0 * d ** 3 * n
    assert R.sweep_flops(1, T, H, d, with_c=True) == 4.0 * d ** 3 * n


def test_simt_peak_from_unit_counts():
    # 148 SMs x 128 FMA lanes x 2 flops x clock
    assert R.fp32_simt_tflops(1965.0) == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)

"""Pins of the oracle's Hadamard rotation (BitDecoding-FP4, "Outlier-Aware Key
Quantization": an orthogonal Hadamard rotation of K, the inverse on the query side).

Anchors: the Sylvester matrix from scipy, its closed-form identities (H H^T = n I, scores
scaled by n), exact integer cases, a hand-worked n = 4 example and the purpose of the
rotation (outlier channels spread out, smaller quantisation error)."""
import numpy as np
import pytest
import scipy.linalg

from oracle import attention as A
from oracle import formats as F
from oracle import rotate as R


def test_hand_worked_n4():
    # H_4 rows: [1 1 1 1], [1 -1 1 -1], [1 1 -1 -1], [1 -1 -1 1]
    x = np.array([[1.0, 2.0, 3.0, 4.0]], dtype=np.float32)
    assert np.array_equal(R.fwht_rows(x), np.array([[10.0, -2.0, -4.0, 0.0]], dtype=np.float32))


@pytest.mark.parametrize("n", [2, 8, 64, 128])
def test_matches_sylvester_matrix_on_integers(n):
    """Small integers: every butterfly sum is exact in FP32, so the result equals x @ H."""
    x = np.random.default_rng(n).integers(-50, 50, size=(7, n)).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    assert np.array_equal(R.fwht_rows(x).astype(np.float64), x.astype(np.float64) @ H)


def test_general_values_within_fp32_rounding_of_the_matrix_product():
    x = np.random.default_rng(3).normal(size=(33, 128)).astype(np.float32)
    H = scipy.linalg.hadamard(128).astype(np.float64)
    ref = x.astype(np.float64) @ H
    got = R.fwht_rows(x).astype(np.float64)
    # 7 stages, each one FP32 rounding of a partial sum bounded by sum |x|
    bound = 8 * np.finfo(np.float32).eps * np.abs(x).astype(np.float64).sum(axis=1, keepdims=True)
    assert np.all(np.abs(got - ref) <= bound)


def test_involution_and_score_scaling():
    """H H = n I (twice gives n x, exactly for integers) and (Q H)(K H)^T = n Q K^T."""
    x = np.random.default_rng(4).integers(-20, 20, size=(5, 64)).astype(np.float32)
    assert np.array_equal(R.fwht_rows(R.fwht_rows(x)), 64 * x)
    q = np.random.default_rng(5).normal(size=(6, 128))
    k = np.random.default_rng(6).normal(size=(9, 128))
    qr = R.fwht_rows(q).astype(np.float64)
    kr = R.fwht_rows(k).astype(np.float64)
    assert np.max(np.abs(qr @ kr.T - 128 * (q.astype(np.float32).astype(np.float64) @ k.astype(np.float32).astype(np.float64).T))) < 1e-2


def test_multiplier_applies_before_the_rotation():
    x = np.random.default_rng(7).normal(size=(4, 128)).astype(np.float32)
    mul = np.float32(2.0) ** np.random.default_rng(8).integers(-3, 4, size=128).astype(np.float32)
    assert np.array_equal(R.rotate_rows(x, mul), R.fwht_rows((x * mul).astype(np.float32)))


def test_rotation_spreads_outlier_channels_and_lowers_the_score_error():
    """K with 4 channels x20 (the causal GQA workload's outliers): after the rotation no
    channel stands out, and the MXFP4 (32-element blocks) quantisation error of the scores
    drops (the reason the pages give for the rotation).  With NVFP4's 16-element blocks the
    error is about the same either way, so it is not asserted."""
    rng = np.random.default_rng(9)
    S, d = 256, 128
    q = rng.normal(size=(S, d)).astype(np.float32)
    k = rng.normal(size=(S, d)).astype(np.float32)
    k[:, [3, 40, 77, 100]] *= 20.0
    exact = q.astype(np.float64) @ k.astype(np.float64).T

    def deq(x):
        p, s = F.quantize_rows(x, "mxfp4")
        return F.dequantize_rows(p, s, "mxfp4")
    plain = deq(q) @ deq(k).T
    rot = deq(R.fwht_rows(q)) @ deq(R.fwht_rows(k)).T / d
    assert np.abs(rot - exact).mean() < 0.85 * np.abs(plain - exact).mean()
    colmax = np.abs(R.fwht_rows(k)).max(axis=0) / np.sqrt(d)    # orthonormal scale
    assert colmax.max() < 0.3 * np.abs(k).max(axis=0).max()

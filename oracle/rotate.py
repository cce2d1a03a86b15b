"""Hadamard rotation of Q and K rows before quantisation (an ablation of Smooth-QK).

Test infrastructure (see the package header): never called by the CUDA path.

Source
------
* BitDecoding-FP4, "Outlier-Aware Key Quantization": an orthogonal rotation of the
  keys (a Hadamard transform, O(d log d)) spreads channel outliers across the head
  dimension before quantisation; the inverse rotation goes on the query side, so the
  attention scores are unchanged.  The pages give this as the alternative to the
  static smoothing of HiFA4 / BitDecoding.

Reading (the pages fix no normalisation or evaluation order): the rotation is the
unnormalised Sylvester Hadamard matrix H_n (H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]],
n = d a power of two), applied to each row of Q and of K (H is symmetric and
H H^T = n I, so (Q H)(K H)^T = n Q K^T: the attention call divides its score scale
by n, an exact power of two).  It is evaluated in IEEE FP32 by the fast Walsh-Hadamard
butterflies, stages h = 1, 2, 4, ..., n/2 in that order, each pair (a, b) of positions
(i, i + h) inside a block of 2h becoming (a + b, a - b); the Smooth-QK multiplier, when
given, is applied first (one FP32 multiply), then the rotation, then block quantisation.
"""
from __future__ import annotations

import numpy as np


def fwht_rows(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform of every row (last axis, a power of two) in
    FP32, by butterfly stages h = 1, 2, ..., n/2."""
    y = np.array(x, dtype=np.float32, copy=True)
    n = y.shape[-1]
    if n & (n - 1):
        raise ValueError("row length must be a power of two")
    lead = y.shape[:-1]
    h = 1
    while h < n:
        z = y.reshape(lead + (n // (2 * h), 2, h))
        a = z[..., 0, :].copy()
        b = z[..., 1, :].copy()
        z[..., 0, :] = a + b          # float32 + float32: one IEEE rounding
        z[..., 1, :] = a - b
        y = z.reshape(lead + (n,))
        h *= 2
    return y


def rotate_rows(x, mul=None) -> np.ndarray:
    """The rotated FP32 rows the quantiser sees: fwht(x * mul) (mul optional, one FP32
    multiply, broadcastable to x)."""
    x32 = np.asarray(x, dtype=np.float32)
    if mul is not None:
        x32 = (x32 * np.asarray(mul, dtype=np.float32)).astype(np.float32)
    return fwht_rows(x32)

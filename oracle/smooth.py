"""Calibration of the static per-channel Smooth-QK multipliers.

Test infrastructure (see the package header): never called by the CUDA path.

Sources
-------
* HiFA4, Abstract: Smooth-QK applies a calibration-static per-channel
  equivalent rescaling to Q and K after RoPE, moving quantisation difficulty
  from K to Q, with no per-tile online reduction at inference.
* BitDecoding-FP4, "Outlier-Aware Key Quantization": static smoothing
  estimates per-channel coefficients during a calibration phase and rescales
  keys per channel.

Reading (the pages give no formula): for kv-head h and channel c,
    r_c   = max_t |K_tc| / max_{t, q-heads of h} |Q_tc|      (FP32 division)
    lam_c = sqrt(r_c) rounded to the nearest power of two in the log domain
            (ties up), clamped to [2^-8, 2^8];
Q is multiplied by lam and K by 1/lam, both exact for powers of two, so
Q K^T is unchanged before quantisation.  Special cases: r = 0 -> 2^-8,
r = inf -> 2^8, r = NaN (both maxima zero) -> 1.
"""
from __future__ import annotations

import numpy as np


def nearest_pow2_exponent_of_sqrt(r) -> np.ndarray:
    """Integer e = round(log2(sqrt(r))) with ties up, for finite r > 0, from the exact
    binary exponent of r: r in [2^(2e-1), 2^(2e+1))."""
    r = np.asarray(r, dtype=np.float64)
    _, ex = np.frexp(r)
    E = ex - 1                      # floor(log2 r)
    return np.floor_divide(E + 1, 2)


def calibrate(q_cal, k_cal) -> np.ndarray:
    """q_cal [Hq, T, d], k_cal [Hkv, T, d] (bf16 values) -> lam [Hkv, d] float32."""
    q_cal = np.asarray(q_cal, dtype=np.float32)
    k_cal = np.asarray(k_cal, dtype=np.float32)
    Hq, Hkv = q_cal.shape[0], k_cal.shape[0]
    grp = Hq // Hkv
    qmax = np.abs(q_cal).reshape(Hkv, grp * q_cal.shape[1], -1).max(axis=1)   # [Hkv, d]
    kmax = np.abs(k_cal).max(axis=1)                                         # [Hkv, d]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (kmax / qmax).astype(np.float32)
    e = np.zeros(r.shape, dtype=np.int64)
    fin = np.isfinite(r) & (r > 0)
    e[fin] = nearest_pow2_exponent_of_sqrt(r[fin])
    e[r == 0] = -8
    e[np.isinf(r)] = 8
    e[np.isnan(r)] = 0
    e = np.clip(e, -8, 8)
    return np.exp2(e).astype(np.float32)

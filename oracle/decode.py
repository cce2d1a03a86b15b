"""Decode attention over an FP4 paged KV cache with a BF16 vertical-line set and window.

Test infrastructure (see the package header): never called by the CUDA path.

Sources
-------
* HyQuant (Hybrid-Precision Quantization for LLM Attention): keys are split
  into vertical-line positions, a recent sliding window and the quantised
  remainder; vertical lines and the window stay in FP16/BF16; in decode the
  cache is stored the same way and dequantisation is fused into the scan under
  a single softmax.  Keeping 5% of tokens in full precision adds about 15% of
  the non-window KV over strict 4-bit, so a vertical-line token replaces its
  4-bit copy rather than duplicating it.
* BitDecoding-FP4, "System-Level Optimization": the paged KV cache maps
  fixed-size token blocks to physical memory through a block table.

This is the plain definition: one softmax over the union of the three key
classes, each key counted once, in FP64.  The query and the probabilities are
not quantised in decode (the pages quantise only the cache here).  Excluded
slots of the FP4 region are zero-filled before quantisation (so they do not
enter any block maximum) and masked out of the softmax.
"""
from __future__ import annotations

import numpy as np

from . import formats


def quantize_fp4_region(k, v, hp_pos, fmt: str, g_k: float = 1.0, g_v: float = 1.0):
    """Dequantised FP4 keys/values of the non-window prefix of one (batch, kv-head).

    k, v [n_fp4, d] bf16 values; hp_pos are the vertical-line positions (zero-filled
    before quantisation).  K blocks run along d, V blocks along tokens (from token 0,
    so page boundaries are block boundaries)."""
    kz = np.array(k, dtype=np.float32, copy=True)
    vz = np.array(v, dtype=np.float32, copy=True)
    kz[hp_pos] = 0.0
    vz[hp_pos] = 0.0
    pk, sk = formats.quantize_rows(kz, fmt, 0.0, g_k)
    kh = formats.dequantize_rows(pk, sk, fmt, g_k)
    pv, sv = formats.quantize_cols_transposed(vz, fmt, 0.0, g_v)
    vh = formats.dequantize_rows(pv, sv, fmt, g_v).T[: v.shape[0]]
    return kh, vh


def attend(q, keys, values, sm_scale: float):
    """softmax(q keys^T * sm_scale) values in FP64; q [G, d], keys/values [N, d]."""
    s = (np.asarray(q, np.float64) @ np.asarray(keys, np.float64).T) * sm_scale
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ np.asarray(values, np.float64)) / p.sum(axis=1, keepdims=True)


def decode_group(q, k, v, hp_pos, window: int, fmt: str, g_k: float = 1.0, g_v: float = 1.0,
                 sm_scale: float | None = None, fp4_part=None):
    """Oracle decode output for the G q-heads of one (batch, kv-head).

    q [G, d]; k, v [L, d] bf16 values of every key position (the current token is the
    last); positions [L-window, L) form the BF16 window, hp_pos (within [0, L-window))
    the BF16 vertical-line set, the rest is FP4.  `fp4_part` may pass precomputed
    (k_hat, v_hat) of the FP4 region."""
    L, d = k.shape
    sm = 1.0 / np.sqrt(d) if sm_scale is None else sm_scale
    n_fp4 = L - window
    kh, vh = quantize_fp4_region(k[:n_fp4], v[:n_fp4], hp_pos, fmt, g_k, g_v) if fp4_part is None else fp4_part
    keep = np.ones(n_fp4, dtype=bool)
    keep[hp_pos] = False
    keys = np.concatenate([kh[keep], np.asarray(k[hp_pos], np.float64), np.asarray(k[n_fp4:], np.float64)])
    vals = np.concatenate([vh[keep], np.asarray(v[hp_pos], np.float64), np.asarray(v[n_fp4:], np.float64)])
    return attend(q, keys, vals, sm)

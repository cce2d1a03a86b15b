"""Hybrid-precision prefill: vertical-line and window keys in BF16, the rest in FP4, under
one online softmax.

Test infrastructure (see the package header): never called by the CUDA path.

Source
------
* HyQuant (Hybrid-Precision Quantization for LLM Attention), single body: the keys of
  each query are split into vertical-line positions, a recent sliding window and the
  quantised remainder; vertical lines and the window stay in full precision (FP16/BF16),
  the rest is 4-bit; the low-bit and the full-precision GEMMs share one FlashAttention-
  style kernel and one online softmax.  In the decode cache a vertical-line token replaces
  its 4-bit copy.

Readings (the pages give no tiling, order or mask rule):
* Causal, top-left aligned.  Query row i: window W_i = {j : i - W < j <= i}; vertical keys
  V_i = {v in V : v <= i - W} (vertical lines inside the window are window keys); FP4 keys
  F_i = {j <= i} minus W_i minus V.
* The full-precision part comes first: s_j = (q_i . k_j) * sm_scale on the bf16 values,
  m0 = max s_j, p_j = exp(s_j - m0) unquantised, l0 = sum p_j, o0 = sum p_j v_j.
* Then the FP4 key tiles (width 128, in key order) exactly as the prefill oracle
  (pre-normalisation quantisation of P against the running maximum, normaliser from P_hat),
  the running state starting at (m0, l0, o0); keys outside F_i are masked.
* The FP4 operands are quantised from Q, K and V with the vertical-line rows of K and V
  zeroed before quantisation (as the decode cache); the window keys keep their FP4 copies
  (they are FP4 keys of later rows).
"""
from __future__ import annotations

import numpy as np

from . import attention


def key_classes(S: int, window: int, vlines) -> tuple[np.ndarray, np.ndarray]:
    """Boolean [S, S] masks (rows = queries, cols = keys): full precision, FP4."""
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    visible = j <= i
    win = visible & (j > i - window)
    vl = np.zeros(S, dtype=bool)
    vl[np.asarray(vlines, dtype=np.int64)] = True
    full = win | (visible & vl[None, :])
    fp4 = visible & ~full
    return full, fp4


def full_precision_part(q, k, v, full_mask, sm_scale: float):
    """(m0, l0, o0) per row over the keys of `full_mask`, unquantised, FP64."""
    s = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) * sm_scale
    s = np.where(full_mask, s, -np.inf)
    m0 = s.max(axis=1)
    p = np.where(full_mask, np.exp(s - m0[:, None]), 0.0)
    return m0, p.sum(axis=1), p @ np.asarray(v, np.float64)


def hybrid_prefill_head(q, k, v, qhat, khat, vhat, vlines, window: int, fmt: str,
                        qmax_p: float = 0.0, sm_scale: float | None = None, rows=None):
    """One (batch, q-head): q, k, v bf16 values [S, d]; qhat, khat, vhat the dequantised FP4
    operands (K, V quantised with the vertical-line rows zeroed); returns out [R, d]."""
    S, d = q.shape
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    full, fp4 = key_classes(S, window, vlines)
    m0, l0, o0 = full_precision_part(q[rows], k, v, full[rows], sm)
    return attention.attention_pnq(qhat, khat, vhat, causal=True, fmt=fmt, qmax_p=qmax_p,
                                   sm_scale=sm, rows=rows, key_mask=fp4[rows], init=(m0, l0, o0))

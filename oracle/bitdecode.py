"""Decode with FP4 tensor-core products on both sides: a dual-residual FP4 query against the
FP4 paged cache, and the probabilities quantised before the PV product.

Test infrastructure (see the package header): never called by the CUDA path.

Sources
-------
* BitDecoding-FP4 (Algorithm-System Co-Design for Native FP4 KV Cache Decoding), "Error
  Sources": a query quantised to FP4 alongside the cache loses most of the logit accuracy;
  a dual-residual query - the query as the sum of two FP4 tensors, the second quantising
  the residual of the first - brings the logit error down (60 % to 1 % on the pages'
  measurement).  "System-Level Optimization": the softmax is transposed so that its
  normalisation runs along the MMA accumulation direction and P is quantised inside the
  softmax reduction; the query MMAs are stacked over the paged cache.

Readings (the pages give no formulas):
* q1 = NVFP4(q) (16-element blocks along d, UE4M3 scales, tensor scale 1), r = q - deq(q1)
  in FP32, q2 = NVFP4(r); the scores use deq(q1) + deq(q2) (the two products accumulate in
  FP32 on the GPU).
* The cache is the decode's paged NVFP4 cache holding every key (no BF16 set or window).
* Keys are scanned in tiles of 128 positions (two 64-token pages) in position order; P is
  quantised exactly as in the prefill (pre-normalisation quantisation of exp(s - m) against
  the running maximum, 16-key NVFP4 blocks with g_P = 1/(6*448), normaliser from P_hat).
* The scan of a sequence is split into contiguous ranges of `tiles_per_split` whole tiles
  (the last shorter); each range keeps its own running state and the ranges are merged
  exactly (log-sum-exp).  The range length is part of the definition, since each range
  restarts the running maximum.
"""
from __future__ import annotations

import numpy as np

from . import attention, formats


def dual_residual_query(q):
    """deq(q1) + deq(q2) for bf16-valued q [..., d] (FP64 result; q1, q2 NVFP4)."""
    q32 = np.asarray(q, dtype=np.float32)
    p1, s1 = formats.quantize_rows(q32, "nvfp4")
    d1 = formats.dequantize_rows(p1, s1, "nvfp4")
    r = (q32 - d1.astype(np.float32)).astype(np.float32)     # FP32 residual (deq(q1) is exact in FP32)
    p2, s2 = formats.quantize_rows(r, "nvfp4")
    return d1 + formats.dequantize_rows(p2, s2, "nvfp4"), (p1, s1, p2, s2)


def split_ranges(L: int, tiles_per_split: int, tile: int = attention.BC):
    """Key ranges [a, b) of the splits of an L-token scan."""
    n_tiles = -(-L // tile)
    per = max(1, int(tiles_per_split))
    return [(t0 * tile, min(L, (t0 + per) * tile)) for t0 in range(0, n_tiles, per)]


def decode_group_fp4q(q, k, v, tiles_per_split: int, sm_scale: float | None = None):
    """Decode output for the G q-heads of one (sequence, kv-head): q [G, d], k, v [L, d] the
    bf16 values of the cached keys; returns [G, d] (FP64)."""
    L, d = k.shape
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    qt, _ = dual_residual_query(q)
    pk, sk = formats.quantize_rows(np.asarray(k, np.float32), "nvfp4")
    kh = formats.dequantize_rows(pk, sk, "nvfp4")
    pv, sv = formats.quantize_cols_transposed(np.asarray(v, np.float32), "nvfp4")
    vh = formats.dequantize_rows(pv, sv, "nvfp4").T[:L]
    outs, lses = [], []
    for a, b in split_ranges(L, tiles_per_split):
        o, lse = attention.attention_pnq(qt, kh[a:b], vh[a:b], causal=False, fmt="nvfp4", sm_scale=sm,
                                         return_lse=True)
        outs.append(o)
        lses.append(lse)
    lse = np.stack(lses)                       # [splits, G]
    w = np.exp(lse - lse.max(axis=0))
    return np.einsum("sg,sgd->gd", w, np.stack(outs)) / w.sum(axis=0)[:, None]

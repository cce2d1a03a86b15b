"""Prefill attention: tiled online softmax with pre-normalisation quantisation.

Test infrastructure (see the package header): never called by the CUDA path.

Sources
-------
* HiFA4 (Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs), Abstract:
  QK^T and PV both run as 4-bit GEMMs inside FlashAttention with an online
  softmax state; P-Reordering accumulates the softmax normaliser from the same
  quantised weights P_hat that feed the PV GEMM (not from a higher-precision
  reconstruction).  The inconsistent alternative (normaliser from the
  unquantised exponentials) gives a coherent output-scaling error with net
  probability-mass loss per tile.
* MXAttention, Abstract: Pre-Normalization Quantization quantises the
  unnormalised softmax exponentials before the row-wise summation, which keeps
  the output normalised by construction.
* BitDecoding-FP4, "Underflow-Aware Probability Scaling": with E4M3 scales,
  small probabilities must not round to zero.  Reading: NVFP4 P uses the static
  FP32 tensor scale g_P = 1/(6*448), since P_tilde <= 1 by construction.

The algorithm, per (batch, q-head) and query row, exactly as executed here:

    s_j = (q_hat . k_hat_j) * sm_scale                          (FP64)
    m = -inf, l = 0, o = 0
    for each key tile T of width Bc = 128, in order, that holds a visible key:
        m_new   = max(m, max_{j in T} s_j)        (masked keys: s = -inf)
        p~_j    = exp(s_j - m_new)                (masked keys: 0)
        p^_j    = block-quantise(p~ rounded to FP32) per blk consecutive keys of T
        alpha   = exp(m - m_new)
        l = alpha*l + sum_j p^_j ;  o = alpha*o + sum_j p^_j v_hat_j ;  m = m_new
    out = o / l

Readings (silent or ambiguous on the pages): Bc = 128; the running maximum is
exact at every tile (no conditional rescale); P is quantised against the
current m_new; the P scale decision is taken in FP32 like the tensors';
sm_scale = 1/sqrt(d); masked keys are exact zeros inside their P blocks;
causal attention is top-left aligned (query i sees keys <= i).

Variant (an ablation, off by default): conditional rescaling with a threshold tau
(an integer number of binades), the FlashAttention-4 technique named in the
FLAMIA page's FlashAttention-4 abstract.  The reference m is kept while a tile's
maximum stays within tau binades above it, so p~ = exp(s - m) may reach 2^tau:

        tmax = max_{j in T} s_j
        if m = -inf or (tmax - m) * log2(e) > tau:  m_new = max(m, tmax)
        else:                                       m_new = m
        (then as above, against m_new)

The MXFP4 P scale absorbs p~ > 1 unchanged; the NVFP4 P tensor scale becomes
g_P * 2^tau so that UE4M3 still spans the block maxima.  tau = 0 is the exact
running maximum above.
"""
from __future__ import annotations

import numpy as np

from . import formats

BC = 128
G_P_NVFP4 = float(np.float32(1.0 / (6.0 * 448.0)))


def p_tensor_scale(fmt: str, tau: int = 0) -> float:
    """Second-level FP32 scale of P: g_P = fl32(1/(6*448)) for NVFP4, times 2^tau under
    conditional rescaling (exact: a power-of-two multiple); 1 for MXFP4."""
    return G_P_NVFP4 * 2.0 ** int(tau) if fmt == "nvfp4" else 1.0


def quantize_p(p32: np.ndarray, fmt: str, qmax_p: float = 0.0, tau: int = 0) -> np.ndarray:
    """FP64 dequantised P_hat of FP32 exponentials p32 [R, BC], blocks along keys."""
    blk = formats.block_size(fmt)
    R, W = p32.shape
    g = p_tensor_scale(fmt, tau)
    codes, s = formats.quantize_blocks(p32.reshape(R, W // blk, blk), fmt,
                                       qmax_p if fmt == "mxfp4" else 0.0, g)
    return formats.dequantize_blocks(codes, s, fmt, g).reshape(R, W)


def attention_pnq(qhat, khat, vhat, *, causal: bool, fmt: str, qmax_p: float = 0.0,
                  sm_scale: float | None = None, rows=None, consistent: bool = True,
                  return_weights: bool = False, return_lse: bool = False, return_eps: bool = False,
                  p_quantizer=None, rescale_tau: int = 0, key_mask=None, init=None):
    """Tiled PNQ attention for one (batch, head) on dequantised operands.

    qhat [Sq, d], khat/vhat [Sk, d] (FP64).  `rows` selects query rows (default all).
    consistent=False takes the normaliser from the unquantised exponentials
    (the HiFA4 'inconsistent' variant, a diagnostic).  Optional extras:
    the effective key weights (P_hat rescaled to the final maximum, divided by l),
    the log-sum-exp m + ln(l) and the per-tile mass ratio eps = sum p^ / sum p~ - 1.
    `p_quantizer(p32) -> p_hat` replaces the P quantiser (tests use the identity).
    `rescale_tau` > 0 selects conditional rescaling (see the module header).
    `key_mask` (bool [R, Sk], True = the key takes part) removes keys beyond the causal
    mask; `init` = (m, l, o) per row starts the online state from an earlier part of the
    same softmax (the full-precision keys of the hybrid prefill)."""
    tau = int(rescale_tau)
    if tau < 0 or tau != rescale_tau:
        raise ValueError("rescale_tau must be a non-negative integer")
    qhat = np.asarray(qhat, dtype=np.float64)
    khat = np.asarray(khat, dtype=np.float64)
    vhat = np.asarray(vhat, dtype=np.float64)
    Sq, d = qhat.shape
    Sk = khat.shape[0]
    rows = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    R = len(rows)
    S = (qhat[rows] @ khat.T) * sm
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    o = np.zeros((R, vhat.shape[1]))
    if init is not None:
        m = np.array(init[0], dtype=np.float64, copy=True)
        l = np.array(init[1], dtype=np.float64, copy=True)
        o = np.array(init[2], dtype=np.float64, copy=True)
    W = np.zeros((R, Sk)) if return_weights else None
    eps = []
    for t0 in range(0, Sk, BC):
        t1 = min(Sk, t0 + BC)
        s = S[:, t0:t1].copy()
        if causal:
            s[np.arange(t0, t1)[None, :] > rows[:, None]] = -np.inf
        if key_mask is not None:
            s[~np.asarray(key_mask)[:, t0:t1]] = -np.inf
        act = np.isfinite(s).any(axis=1)
        if not act.any():
            continue
        tmax = np.max(s, axis=1)                           # masked keys are -inf
        m_new = np.maximum(m, tmax)
        if tau > 0:
            with np.errstate(invalid="ignore"):
                grow = (tmax - m) * np.log2(np.e) > tau
            m_new = np.where(np.isneginf(m) | grow, m_new, m)
        with np.errstate(invalid="ignore"):
            p = np.where(np.isfinite(s), np.exp(s - m_new[:, None]), 0.0)
            alpha = np.where(act, np.exp(m - m_new), 1.0)
        pad = np.zeros((R, BC))
        pad[:, : t1 - t0] = p
        if p_quantizer is None:
            phat = quantize_p(pad.astype(np.float32), fmt, qmax_p, tau)[:, : t1 - t0]
        else:
            phat = np.asarray(p_quantizer(pad), dtype=np.float64)[:, : t1 - t0]
        phat[~act] = 0.0
        alpha = np.where(np.isneginf(m) & act, 0.0, alpha)
        denom_add = phat.sum(axis=1) if consistent else p.sum(axis=1)
        l = alpha * l + denom_add
        o = alpha[:, None] * o + phat @ vhat[t0:t1]
        if return_weights:
            W *= alpha[:, None]
            W[:, t0:t1] = phat
        if return_eps:
            with np.errstate(invalid="ignore", divide="ignore"):
                eps.append(phat[act].sum(axis=1) / p[act].sum(axis=1) - 1.0)
        m = m_new
    out = o / l[:, None]
    res = [out]
    if return_weights:
        res.append(W / l[:, None])
    if return_lse:
        res.append(m + np.log(l))
    if return_eps:
        res.append(np.concatenate(eps) if eps else np.zeros(0))
    return res[0] if len(res) == 1 else tuple(res)


def attention_plain(q, k, v, *, causal: bool, sm_scale: float | None = None, rows=None):
    """Unquantised softmax attention in FP64 (the BF16 reference of the inputs)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Sq, d = q.shape
    rows = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    s = (q[rows] @ k.T) * sm
    if causal:
        s[np.arange(k.shape[0])[None, :] > rows[:, None]] = -np.inf
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def quantize_qkv(q, k, v, fmt: str, qmax: float = 0.0, g_q: float = 1.0, g_k: float = 1.0,
                 g_v: float = 1.0, mul_q=None, mul_k=None):
    """Quantise bf16-valued Q [.., Sq, d], K, V [.., Sk, d] as the library does (Q, K blocks
    along d with optional smoothing multipliers; V blocks along tokens) and return the FP64
    dequantised tensors (V back in [.., Sk, d] orientation)."""
    pq, sq = formats.quantize_rows(q, fmt, qmax, g_q, mul_q)
    pk, sk = formats.quantize_rows(k, fmt, qmax, g_k, mul_k)
    pv, sv = formats.quantize_cols_transposed(v, fmt, qmax, g_v)
    qh = formats.dequantize_rows(pq, sq, fmt, g_q)
    kh = formats.dequantize_rows(pk, sk, fmt, g_k)
    vt = formats.dequantize_rows(pv, sv, fmt, g_v)
    vh = np.swapaxes(vt, -1, -2)[..., : v.shape[-2], :]
    return qh, kh, vh


def prefill(q, k, v, *, causal: bool, fmt: str, qmax: float = 0.0, qmax_p: float = 0.0,
            lam=None, sm_scale: float | None = None, rows=None, heads=None, return_lse: bool = False,
            rescale_tau: int = 0, consistent: bool = True):
    """Oracle output of the library's prefill pipeline on bf16-valued inputs.

    q [B, Hq, Sq, d], k/v [B, Hkv, Sk, d]; `lam` [Hkv, d] Smooth-QK multipliers
    (Q gets lam of its kv-head, K gets 1/lam).  `rows` samples query rows and `heads`
    a list of (b, h) pairs.  Returns {(b, h): out [R, d]} (and lse when asked)."""
    B, Hq, Sq, d = q.shape
    Hkv = k.shape[1]
    heads = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    res = {}
    cache = {}
    for (b, h) in heads:
        kvh = h * Hkv // Hq
        mq = None if lam is None else lam[kvh][None, :]
        mk = None if lam is None else (1.0 / lam[kvh].astype(np.float64)).astype(np.float32)[None, :]
        if (b, kvh) not in cache:
            _, kh, vh = quantize_qkv(q[b, h][:1], k[b, kvh], v[b, kvh], fmt, qmax, mul_k=mk)
            cache[(b, kvh)] = (kh, vh)
        kh, vh = cache[(b, kvh)]
        pq, sq = formats.quantize_rows(q[b, h], fmt, qmax, 1.0, mq)
        qh = formats.dequantize_rows(pq, sq, fmt)
        res[(b, h)] = attention_pnq(qh, kh, vh, causal=causal, fmt=fmt, qmax_p=qmax_p,
                                    sm_scale=sm_scale, rows=rows, return_lse=return_lse,
                                    rescale_tau=rescale_tau, consistent=consistent)
    return res

"""Pins of the oracle's hybrid-precision prefill (HyQuant: vertical-line and window keys
in full precision, the rest 4-bit, one online softmax).

Anchors: with the quantisers replaced by identities the split into parts is pure
bookkeeping (plain softmax attention); a window covering every key is plain attention on
the bf16 values; every visible key lands in exactly one class; the weights stay a convex
combination; a scalar brute-force restatement on a tiny case."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import formats as F
from oracle import hybrid as Hy


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).normal(size=shape) * scale).astype(np.float32)


def _vlines(S, seed, frac=0.05):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(S, max(1, int(frac * S)), replace=False))


def test_key_classes_partition_the_visible_keys():
    S, W = 300, 64
    vl = _vlines(S, 1)
    full, fp4 = Hy.key_classes(S, W, vl)
    vis = np.tril(np.ones((S, S), dtype=bool))
    assert np.array_equal(full | fp4, vis) and not np.any(full & fp4)
    assert np.all(full[np.arange(S), np.arange(S)])                  # a row sees itself in BF16
    i = 250
    assert np.array_equal(np.flatnonzero(full[i]), np.union1d(np.arange(i - W + 1, i + 1), vl[vl <= i]))


@pytest.mark.parametrize("S,W", [(260, 128), (700, 64)])
def test_identity_quantisers_give_plain_attention(S, W):
    q, k, v = _rand((S, 32), 2, 1.5), _rand((S, 32), 3, 1.5), _rand((S, 32), 4)
    vl = _vlines(S, 5)
    full, fp4 = Hy.key_classes(S, W, vl)
    m0, l0, o0 = Hy.full_precision_part(q, k, v, full, 1.0 / math.sqrt(32))
    out = A.attention_pnq(q, k, v, causal=True, fmt="nvfp4", key_mask=fp4, init=(m0, l0, o0),
                          p_quantizer=lambda p: p)
    ref = A.attention_plain(q, k, v, causal=True)
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_window_over_everything_is_plain_attention():
    S = 200
    q, k, v = _rand((S, 64), 6), _rand((S, 64), 7), _rand((S, 64), 8)
    vl = _vlines(S, 9)
    kz, vz = k.copy(), v.copy()
    kz[vl] = 0.0
    vz[vl] = 0.0
    qh, kh, vh = A.quantize_qkv(q, kz, vz, "mxfp4")
    out = Hy.hybrid_prefill_head(q, k, v, qh, kh, vh, vl, window=S, fmt="mxfp4")
    assert np.max(np.abs(out - A.attention_plain(q, k, v, causal=True))) <= 1e-12


def _scalar_hybrid(q, k, v, qh, kh, vh, vl, W, fmt, rows):
    """Brute-force restatement with scalar loops (tiny inputs only)."""
    S, d = q.shape
    sm = 1.0 / math.sqrt(d)
    blk = F.block_size(fmt)
    g = A.p_tensor_scale(fmt)
    vls = set(int(x) for x in vl)
    out = []
    for i in rows:
        full = [j for j in range(i + 1) if j > i - W or j in vls]
        s = {j: float(np.dot(q[i].astype(np.float64), k[j].astype(np.float64))) * sm for j in full}
        m = max(s.values())
        l = sum(math.exp(x - m) for x in s.values())
        o = sum(math.exp(s[j] - m) * v[j].astype(np.float64) for j in full)
        for t0 in range(0, i + 1, 128):
            keys = [j for j in range(t0, min(i + 1, t0 + 128)) if j not in s]
            if not keys:
                continue
            sc = {j: float(np.dot(qh[i], kh[j])) * sm for j in keys}
            m_new = max(m, max(sc.values()))
            pt = np.zeros(128, dtype=np.float32)
            for j in keys:
                pt[j - t0] = np.float32(math.exp(sc[j] - m_new))
            c, sb = F.quantize_blocks(pt.reshape(128 // blk, blk), fmt, 0.0, g)
            ph = F.dequantize_blocks(c, sb, fmt, g).reshape(128)
            a = math.exp(m - m_new)
            l = a * l + sum(ph[j - t0] for j in keys)
            o = a * o + sum(ph[j - t0] * vh[j] for j in keys)
            m = m_new
        out.append(o / l)
    return np.array(out)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_matches_scalar_bruteforce(fmt):
    S, d, W = 300, 32, 64
    q, k, v = _rand((S, d), 10, 1.5), _rand((S, d), 11, 1.5), _rand((S, d), 12)
    vl = _vlines(S, 13, 0.08)
    kz, vz = k.copy(), v.copy()
    kz[vl] = 0.0
    vz[vl] = 0.0
    qh, kh, vh = A.quantize_qkv(q, kz, vz, fmt)
    rows = np.array([0, 5, 63, 64, 130, 200, 299])
    out = Hy.hybrid_prefill_head(q, k, v, qh, kh, vh, vl, W, fmt, rows=rows)
    ref = _scalar_hybrid(q, k, v, qh, kh, vh, vl, W, fmt, rows)
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_output_is_a_convex_combination():
    """Every output coordinate lies between the smallest and largest value any visible key
    (bf16 V or FP4 V_hat) offers."""
    S, W = 400, 128
    q, k, v = _rand((S, 64), 14, 1.5), _rand((S, 64), 15, 1.5), _rand((S, 64), 16)
    vl = _vlines(S, 17)
    kz, vz = k.copy(), v.copy()
    kz[vl] = 0.0
    vz[vl] = 0.0
    qh, kh, vh = A.quantize_qkv(q, kz, vz, "nvfp4")
    out = Hy.hybrid_prefill_head(q, k, v, qh, kh, vh, vl, W, "nvfp4")
    lo = np.minimum.accumulate(np.minimum(v, vh), axis=0)
    hi = np.maximum.accumulate(np.maximum(v, vh), axis=0)
    assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)

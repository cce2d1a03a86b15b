"""Pins of the oracle's FP4 tensor-core decode (BitDecoding-FP4: dual-residual FP4 query,
FP4 probabilities, paged FP4 cache).

Anchors: a query already on the NVFP4 grid has a zero residual; the residual cuts the
logit error (the pages' reason for it); a scalar brute-force restatement of the split scan
and its log-sum-exp merge; one split equals the prefill oracle's PNQ loop on the same
operands; the output is a convex combination of the V_hat rows."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import bitdecode as BD
from oracle import formats as F


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).normal(size=shape) * scale).astype(np.float32)


def test_query_on_the_grid_has_no_residual():
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, size=(4, 128)).astype(np.uint8)
    codes[:, ::16] = 7                                        # every block holds a 6: scale 1.0
    scales = np.full((4, 8), 0x38, dtype=np.uint8)            # UE4M3 1.0
    q = F.dequantize_rows(F.pack_nibbles(codes), scales, "nvfp4").astype(np.float32)
    qt, (p1, s1, p2, s2) = BD.dual_residual_query(q)
    assert np.array_equal(qt, q.astype(np.float64))
    assert np.all(F.dequantize_rows(p2, s2, "nvfp4") == 0.0)


def test_residual_cuts_the_logit_error():
    q, k = _rand((8, 128), 2), _rand((500, 128), 3)
    exact = q.astype(np.float64) @ k.astype(np.float64).T
    p1, s1 = F.quantize_rows(q, "nvfp4")
    one = F.dequantize_rows(p1, s1, "nvfp4") @ k.astype(np.float64).T
    qt, _ = BD.dual_residual_query(q)
    two = qt @ k.astype(np.float64).T
    e1 = np.abs(one - exact).mean() / np.abs(exact).mean()
    e2 = np.abs(two - exact).mean() / np.abs(exact).mean()
    assert e2 < 0.15 * e1


def test_split_ranges():
    assert BD.split_ranges(1000, 3) == [(0, 384), (384, 768), (768, 1000)]
    assert BD.split_ranges(128, 4) == [(0, 128)]
    assert BD.split_ranges(300, 8) == [(0, 300)]
    assert BD.split_ranges(300, 1) == [(0, 128), (128, 256), (256, 300)]


def _scalar(q, k, v, tps):
    G, d = q.shape
    L = k.shape[0]
    sm = 1.0 / math.sqrt(d)
    qt, _ = BD.dual_residual_query(q)
    pk, sk = F.quantize_rows(k, "nvfp4")
    kh = F.dequantize_rows(pk, sk, "nvfp4")
    pv, sv = F.quantize_cols_transposed(v, "nvfp4")
    vh = F.dequantize_rows(pv, sv, "nvfp4").T[:L]
    g = A.p_tensor_scale("nvfp4")
    out = np.zeros((G, d))
    for gi in range(G):
        parts = []
        for a, b in BD.split_ranges(L, tps):
            m, l, o = -math.inf, 0.0, np.zeros(d)
            for t0 in range(a, b, 128):
                keys = list(range(t0, min(b, t0 + 128)))
                s = [float(np.dot(qt[gi], kh[j])) * sm for j in keys]
                mn = max(m, max(s))
                pt = np.zeros(128, dtype=np.float32)
                for i, x in enumerate(s):
                    pt[i] = np.float32(math.exp(x - mn))
                c, sb = F.quantize_blocks(pt.reshape(8, 16), "nvfp4", 0.0, g)
                ph = F.dequantize_blocks(c, sb, "nvfp4", g).reshape(128)
                al = math.exp(m - mn) if m != -math.inf else 0.0
                l = al * l + sum(ph[:len(keys)])
                o = al * o + sum(ph[i] * vh[j] for i, j in enumerate(keys))
                m = mn
            parts.append((m + math.log(l), o / l))
        M = max(x for x, _ in parts)
        wsum = sum(math.exp(x - M) for x, _ in parts)
        out[gi] = sum(math.exp(x - M) * o for x, o in parts) / wsum
    return out


@pytest.mark.parametrize("L,tps", [(300, 2), (520, 1), (200, 4)])
def test_matches_scalar_bruteforce(L, tps):
    q, k, v = _rand((4, 128), 4, 1.5), _rand((L, 128), 5, 1.5), _rand((L, 128), 6)
    got = BD.decode_group_fp4q(q, k, v, tps)
    assert np.max(np.abs(got - _scalar(q, k, v, tps))) <= 1e-12


def test_one_split_is_the_prefill_loop_and_output_is_convex():
    L = 700
    q, k, v = _rand((4, 128), 7, 1.5), _rand((L, 128), 8, 1.5), _rand((L, 128), 9)
    got = BD.decode_group_fp4q(q, k, v, 100)
    qt, _ = BD.dual_residual_query(q)
    kh = F.dequantize_rows(*F.quantize_rows(k, "nvfp4"), "nvfp4")
    vh = F.dequantize_rows(*F.quantize_cols_transposed(v, "nvfp4"), "nvfp4").T[:L]
    ref = A.attention_pnq(qt, kh, vh, causal=False, fmt="nvfp4")
    assert np.max(np.abs(got - ref)) <= 1e-12
    assert np.all(got >= vh.min(axis=0) - 1e-12) and np.all(got <= vh.max(axis=0) + 1e-12)

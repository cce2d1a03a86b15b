"""Pins of the oracle's attention, decode, smoothing and identification functions.

Anchors: closed forms, invariants that hold by construction, special cases
that reduce to plain softmax attention, and a scalar brute-force restatement of
the tiled loop on tiny inputs.
"""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import decode as D
from oracle import formats as F
from oracle import hyquant as H
from oracle import smooth as SM


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).normal(size=shape) * scale).astype(np.float32)


# ----------------------------------------------------------------------------- tiled loop
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [64, 200, 256])
def test_tiled_loop_identity_quantizer_is_softmax(causal, S):
    q, k, v = _rand((S, 32), 1), _rand((S, 32), 2, 2.0), _rand((S, 32), 3)
    out = A.attention_pnq(q, k, v, causal=causal, fmt="nvfp4", p_quantizer=lambda p: p)
    ref = A.attention_plain(q, k, v, causal=causal)
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_attention_plain_closed_forms():
    """The unquantised reference against closed forms: zero queries weight every visible key
    equally (the output is the mean of all values, or under the causal mask the mean of the
    prefix); two keys whose scores differ by delta get the logistic weights 1 / (1 + e^-delta)
    and 1 / (1 + e^delta); sm_scale multiplies delta."""
    rng = np.random.default_rng(17)
    S, d = 7, 4
    q = np.zeros((S, d))
    k, v = rng.normal(size=(S, d)), rng.normal(size=(S, d))
    assert np.max(np.abs(A.attention_plain(q, k, v, causal=False) - v.mean(axis=0))) <= 1e-15
    out = A.attention_plain(q, k, v, causal=True)
    for i in range(S):
        assert np.max(np.abs(out[i] - v[: i + 1].mean(axis=0))) <= 1e-15
    q2 = np.array([[1.0, 0.0, 0.0, 0.0]])
    k2 = np.array([[3.0, 0.0, 0.0, 0.0], [0.4, 0.0, 0.0, 0.0]])
    v2 = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    for sm in (None, 0.3):
        delta = (3.0 - 0.4) * (0.5 if sm is None else sm)          # 1 / sqrt(4) by default
        w0 = 1.0 / (1.0 + math.exp(-delta))
        got = A.attention_plain(q2, k2, v2, causal=False, sm_scale=sm)[0]
        assert abs(got[0] - w0) <= 1e-15 and abs(got[1] - (1.0 - w0)) <= 1e-15 and got[2] == got[3] == 0.0


def _scalar_pnq(q, k, v, causal, fmt, qmax_p=0.0, tau=0, stats=None):
    """Brute-force restatement with scalar Python loops (tiny inputs only).  tau > 0: the
    reference maximum moves only when a tile's maximum exceeds it by more than tau binades
    (then p~ may exceed 1, and NVFP4 P takes the tensor scale g_P * 2^tau)."""
    Sq, d = q.shape
    Sk = k.shape[0]
    sm = 1.0 / math.sqrt(d)
    blk = F.block_size(fmt)
    g = np.float32(1.0 / (6.0 * 448.0)) * 2.0 ** tau if fmt == "nvfp4" else 1.0
    out = np.zeros((Sq, v.shape[1]))
    for i in range(Sq):
        m, l, o = -math.inf, 0.0, np.zeros(v.shape[1])
        for t0 in range(0, Sk, 128):
            keys = [j for j in range(t0, min(Sk, t0 + 128)) if not (causal and j > i)]
            if not keys:
                continue
            s = {j: float(np.dot(q[i].astype(np.float64), k[j].astype(np.float64))) * sm for j in keys}
            tmax = max(s.values())
            if m == -math.inf or (tmax - m) / math.log(2.0) > tau:
                m_new = max(m, tmax)
            else:
                m_new = m
            ptil = np.zeros(128, dtype=np.float32)
            for j in keys:
                ptil[j - t0] = np.float32(math.exp(s[j] - m_new))
            if stats is not None:
                stats["max_ptilde"] = max(stats.get("max_ptilde", 0.0), float(ptil.max()))
            c, sb = F.quantize_blocks(ptil.reshape(128 // blk, blk), fmt, qmax_p if fmt == "mxfp4" else 0.0, g)
            phat = F.dequantize_blocks(c, sb, fmt, g).reshape(128)
            alpha = math.exp(m - m_new) if m != -math.inf else 0.0
            l = alpha * l + sum(phat[j - t0] for j in keys)
            o = alpha * o + sum(phat[j - t0] * v[j].astype(np.float64) for j in keys)
            m = m_new
        out[i] = o / l
    return out


@pytest.mark.parametrize("fmt,causal,qmax_p", [("nvfp4", True, 0.0), ("mxfp4", False, 0.0),
                                               ("mxfp4", True, 7.25)])
def test_tiled_pnq_matches_scalar_bruteforce(fmt, causal, qmax_p):
    S = 150                                       # two key tiles, the second ragged
    q, k, v = _rand((S, 16), 4, 2.0), _rand((S, 16), 5, 2.0), _rand((S, 16), 6)
    rows = np.array([0, 1, 63, 127, 128, 129, 149])
    out = A.attention_pnq(q, k, v, causal=causal, fmt=fmt, qmax_p=qmax_p, rows=rows)
    ref = _scalar_pnq(q[rows] if not causal else q, k, v, causal, fmt, qmax_p)
    ref = ref if not causal else ref[rows]
    assert np.max(np.abs(out - ref)) <= 1e-12


# ----------------------------------------------------------------------------- PNQ invariants
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("causal", [False, True])
def test_pnq_weights_are_convex(fmt, causal):
    S = 300
    q, k, v = _rand((S, 64), 7, 1.5), _rand((S, 64), 8, 1.5), _rand((S, 64), 9)
    out, w = A.attention_pnq(q, k, v, causal=causal, fmt=fmt, return_weights=True)
    assert np.all(w >= 0)
    assert np.max(np.abs(w.sum(axis=1) - 1.0)) <= 1e-12
    assert np.max(np.abs(w @ v.astype(np.float64) - out)) <= 1e-12
    if causal:
        assert np.all(w[np.triu_indices(S, 1)] == 0)
    lo = np.min(v, axis=0) if not causal else None
    if lo is not None:
        assert np.all(out >= lo - 1e-12) and np.all(out <= np.max(v, axis=0) + 1e-12)


def test_constant_v_is_preserved_only_with_consistent_normaliser():
    S = 384
    q, k = _rand((S, 64), 10, 2.0), _rand((S, 64), 11, 2.0)
    v = np.ones((S, 64), dtype=np.float32)
    _, _, vh = A.quantize_qkv(q, k, v, "nvfp4")
    assert np.all(vh == 1.03125)                  # 1.0 under NVFP4: scale 0.171875, code 6
    out = A.attention_pnq(q, k, vh, causal=True, fmt="nvfp4")
    assert np.max(np.abs(out - 1.03125)) <= 1e-12
    bad = A.attention_pnq(q, k, vh, causal=True, fmt="nvfp4", consistent=False)
    assert np.max(np.abs(bad - 1.03125)) > 1e-3


def test_inconsistent_normaliser_loses_mass():
    """HiFA4: the normaliser from unquantised exponentials overstates the mass of P_hat."""
    S = 1024
    q, k, v = _rand((S, 64), 12, 1.5), _rand((S, 64), 13, 1.5), _rand((S, 64), 14)
    _, eps = A.attention_pnq(q, k, v, causal=False, fmt="nvfp4", consistent=False,
                             rows=np.arange(0, S, 8), return_eps=True)
    assert np.median(eps) < 0


# ----------------------------------------------------------------------------- closed forms
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_zero_query_gives_mean_of_values(fmt):
    S = 260
    q = np.zeros((S, 32), dtype=np.float32)
    k, v = _rand((S, 32), 15), _rand((S, 32), 16)
    out = A.attention_pnq(q, k, v, causal=False, fmt=fmt)
    assert np.max(np.abs(out - v.astype(np.float64).mean(axis=0))) <= 1e-12
    outc = A.attention_pnq(q, k, v, causal=True, fmt=fmt)
    pref = np.cumsum(v.astype(np.float64), axis=0) / np.arange(1, S + 1)[:, None]
    assert np.max(np.abs(outc - pref)) <= 1e-12


def test_first_causal_row_and_single_key():
    q, k, v = _rand((130, 32), 17), _rand((130, 32), 18), _rand((130, 32), 19)
    out = A.attention_pnq(q, k, v, causal=True, fmt="nvfp4", rows=[0])
    assert np.max(np.abs(out[0] - v[0])) <= 1e-12
    out1 = A.attention_pnq(q[:5], k[:1], v[:1], causal=False, fmt="mxfp4")
    assert np.max(np.abs(out1 - v[0])) <= 1e-12


def test_quantized_attention_is_close_to_unquantized():
    S = 256
    q, k, v = _rand((S, 64), 20), _rand((S, 64), 21), _rand((S, 64), 22)
    qh, kh, vh = A.quantize_qkv(q, k, v, "nvfp4")
    out = A.attention_pnq(qh, kh, vh, causal=True, fmt="nvfp4")
    ref = A.attention_plain(q, k, v, causal=True)
    rel = np.abs(out - ref).sum() / np.abs(ref).sum()
    assert 1e-3 < rel < 0.2


def test_lse_of_a_single_tile():
    S = 100
    q, k, v = _rand((S, 32), 23), _rand((S, 32), 24), _rand((S, 32), 25)
    _, lse = A.attention_pnq(q, k, v, causal=False, fmt="nvfp4", return_lse=True)
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(32)
    m = s.max(axis=1)
    p = np.exp(s - m[:, None])
    ph = A.quantize_p(np.pad(p, ((0, 0), (0, 28))).astype(np.float32), "nvfp4")[:, :S]
    assert np.max(np.abs(lse - (m + np.log(ph.sum(axis=1))))) <= 1e-12


# ----------------------------------------------------------------------------- decode
def test_decode_without_hybrid_parts_is_quantized_attention():
    L, d = 320, 32
    q, k, v = _rand((4, d), 26), _rand((L, d), 27), _rand((L, d), 28)
    out = D.decode_group(q, k, v, np.zeros(0, dtype=np.int64), 0, "nvfp4")
    kh, vh = D.quantize_fp4_region(k, v, np.zeros(0, dtype=np.int64), "nvfp4")
    ref = np.stack([A.attention_pnq(q[i:i + 1], kh, vh, causal=False, fmt="nvfp4",
                                    p_quantizer=lambda p: p)[0] for i in range(4)])
    assert np.max(np.abs(out - ref)) <= 1e-12
    # the FP4 region quantises exactly like the tensor quantiser (K along d, V along tokens)
    kh2 = F.dequantize_rows(*F.quantize_rows(k, "nvfp4"), "nvfp4")
    assert np.array_equal(kh, kh2)


def test_decode_all_full_precision_is_plain_attention():
    L, d, W = 256, 32, 64
    q, k, v = _rand((4, d), 29), _rand((L, d), 30), _rand((L, d), 31)
    hp = np.arange(L - W)
    out = D.decode_group(q, k, v, hp, W, "nvfp4")
    ref = A.attention_plain(q, k, v, causal=False)
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_decode_key_classes_each_count_once():
    L, d, W = 256, 32, 32
    q, k, v = _rand((2, d), 32), _rand((L, d), 33), _rand((L, d), 34)
    hp = np.array([3, 70, 150])
    out = D.decode_group(q, k, v, hp, W, "mxfp4")
    kh, vh = D.quantize_fp4_region(k[:L - W], v[:L - W], hp, "mxfp4")
    keep = np.setdiff1d(np.arange(L - W), hp)
    keys = np.concatenate([kh[keep], k[hp], k[L - W:]])
    vals = np.concatenate([vh[keep], v[hp], v[L - W:]])
    assert len(keys) == L
    assert np.max(np.abs(out - A.attention_plain(q, keys, vals, causal=False))) <= 1e-12
    # zero-filling excluded slots keeps them out of the V block maxima
    v2 = v.copy()
    v2[hp] = 1e4
    _, vh2 = D.quantize_fp4_region(k[:L - W], v2[:L - W], hp, "mxfp4")
    assert np.array_equal(vh2[keep], vh[keep])


# ----------------------------------------------------------------------------- smoothing
def test_smoothing_is_exact_and_nearest_power_of_two():
    rng = np.random.default_rng(35)
    qc = rng.normal(size=(8, 64, 32)).astype(np.float32)
    kc = rng.normal(size=(2, 64, 32)).astype(np.float32)
    kc[:, :, 5] *= 20
    lam = SM.calibrate(qc, kc)
    assert lam.shape == (2, 32)
    assert np.all(np.log2(lam) == np.round(np.log2(lam)))
    # independent evaluation through log2/sqrt, away from ties
    qmax = np.abs(qc).reshape(2, 4 * 64, 32).max(axis=1)
    kmax = np.abs(kc).max(axis=1)
    r = (kmax / qmax).astype(np.float32)
    e = np.log2(np.sqrt(r.astype(np.float64)))
    safe = np.abs(e - np.floor(e) - 0.5) > 1e-6
    assert np.array_equal(np.log2(lam)[safe], np.clip(np.round(e), -8, 8)[safe])
    assert np.all(lam[:, 5] >= 4)                           # the outlier channel moves to Q
    # exact invariance of Q K^T
    for h in range(2):
        qq = qc[4 * h].astype(np.float64)
        kk = kc[h].astype(np.float64)
        lhs = (qq * lam[h]) @ (kk / lam[h]).T
        assert np.array_equal(lhs, qq @ kk.T)


def test_smoothing_ties_and_edges():
    assert SM.nearest_pow2_exponent_of_sqrt(np.array([2.0, 0.5, 8.0, 1.0, 1.99, 0.26])).tolist() == [1, 0, 2, 0, 0, -1]
    qc = np.zeros((1, 4, 3), dtype=np.float32)
    kc = np.zeros((1, 4, 3), dtype=np.float32)
    qc[0, 0, 0] = 1.0
    kc[0, 0, 1] = 1.0
    lam = SM.calibrate(qc, kc)
    assert lam.tolist() == [[2.0 ** -8, 2.0 ** 8, 1.0]]


# ----------------------------------------------------------------------------- identification
def test_vertical_lines_recover_planted_positions():
    rng = np.random.default_rng(36)
    N, d = 2000, 64
    u = rng.normal(size=d)
    u /= np.linalg.norm(u)
    k = rng.normal(size=(N, d))
    planted = np.sort(rng.choice(N, 100, replace=False))
    k[planted] += 6.0 * u
    q = rng.normal(size=(64, d)) + 3.0 * u
    sel = H.select_vertical_lines(q, k, 0.05)
    assert len(sel) == 100
    assert len(np.intersect1d(sel, planted)) >= 95


def test_column_mass_invariants_and_brute_force():
    """Each observation query's probabilities sum to 1, so the masses sum to Nq; all-zero
    queries give the uniform mass Nq/N; a scalar loop with math.exp agrees on a tiny case."""
    import math
    rng = np.random.default_rng(37)
    q = rng.normal(size=(48, 32))
    k = rng.normal(size=(300, 32)) * 1.7
    m = H.column_mass(q, k)
    assert np.all(m >= 0.0)
    assert abs(m.sum() - 48.0) < 1e-10
    mz = H.column_mass(np.zeros((7, 32)), k)
    assert np.max(np.abs(mz - 7.0 / 300.0)) < 1e-15
    qs, ks = rng.normal(size=(3, 4)), rng.normal(size=(5, 4))
    ref = [0.0] * 5
    for i in range(3):
        sc = [sum(qs[i][c] * ks[j][c] for c in range(4)) / 2.0 for j in range(5)]
        mx = max(sc)
        e = [math.exp(x - mx) for x in sc]
        tot = sum(e)
        for j in range(5):
            ref[j] += e[j] / tot
    assert np.max(np.abs(H.column_mass(qs, ks) - np.array(ref))) < 1e-13


def test_vertical_line_count_and_ties():
    """n = ceil(rho * N) (0.05 * 32640 -> 1632 exactly, 0.05 * 101 -> 6); equal masses are
    taken lowest position first; the result is sorted."""
    k = np.random.default_rng(38).normal(size=(32640, 8))
    sel = H.select_vertical_lines(np.zeros((4, 8)), k, 0.05)
    assert len(sel) == 1632 and np.array_equal(sel, np.arange(1632))
    k2 = np.random.default_rng(39).normal(size=(101, 8))
    sel2 = H.select_vertical_lines(np.random.default_rng(40).normal(size=(5, 8)), k2, 0.05)
    assert len(sel2) == 6 and np.all(np.diff(sel2) > 0)
    mass = H.column_mass(np.random.default_rng(40).normal(size=(5, 8)), k2)
    assert mass[sel2].min() >= np.sort(mass)[-6]


# ----------------------------------------------------------------------------- conditional rescale
@pytest.mark.parametrize("causal", [False, True])
def test_conditional_rescale_identity_quantizer_is_softmax(causal):
    """A stale reference maximum only changes the bookkeeping: with an identity P quantiser
    the result is still plain softmax attention."""
    S = 520
    q, k, v = _rand((S, 32), 41, 2.0), _rand((S, 32), 42, 2.0), _rand((S, 32), 43)
    out = A.attention_pnq(q, k, v, causal=causal, fmt="mxfp4", p_quantizer=lambda p: p, rescale_tau=8)
    ref = A.attention_plain(q, k, v, causal=causal)
    assert np.max(np.abs(out - ref)) <= 1e-12


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_conditional_rescale_matches_scalar_bruteforce(fmt):
    """Keys whose scores grow along the sequence: the second tile's maximum exceeds the
    first's, by less than tau = 8 binades, so p~ above 1 is quantised (checked)."""
    S, d = 256, 16
    q = _rand((S, d), 44, 1.0)
    k = _rand((S, d), 45, 1.0) * np.linspace(0.5, 1.5, S, dtype=np.float32)[:, None]
    v = _rand((S, d), 46)
    rows = np.array([5, 130, 200, 255])
    out = A.attention_pnq(q, k, v, causal=False, fmt=fmt, rows=rows, rescale_tau=8)
    st = {}
    ref = _scalar_pnq(q[rows], k, v, False, fmt, tau=8, stats=st)
    assert np.max(np.abs(out - ref)) <= 1e-12
    assert st["max_ptilde"] > 1.0
    exact = _scalar_pnq(q[rows], k, v, False, fmt, tau=0)
    assert np.max(np.abs(exact - ref)) > 0.0        # the variant changes P_hat


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_conditional_rescale_weights_are_convex(fmt):
    S = 300
    q, k, v = _rand((S, 64), 47, 1.5), _rand((S, 64), 48, 1.5), _rand((S, 64), 49)
    out, w = A.attention_pnq(q, k, v, causal=True, fmt=fmt, return_weights=True, rescale_tau=8)
    assert np.all(w >= 0)
    assert np.max(np.abs(w.sum(axis=1) - 1.0)) <= 1e-12
    assert np.max(np.abs(w @ v.astype(np.float64) - out)) <= 1e-12


def test_conditional_rescale_rejects_fractional_tau():
    q = _rand((8, 16), 50)
    with pytest.raises(ValueError):
        A.attention_pnq(q, q, q, causal=False, fmt="nvfp4", rescale_tau=2.5)

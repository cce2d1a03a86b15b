"""Pins of the oracle's format codecs against facts fixed by the definitions.

Each test compares the oracle with an independent construction (nearest-value
search, hand-worked golden cases, exhaustive round trips), never with itself.
"""
import os

import numpy as np
import pytest

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


# ----------------------------------------------------------------------------- E2M1
def test_e2m1_value_set_golden():
    for code, val in _load("e2m1_value_set.txt"):
        v = F.e2m1_decode(np.uint8(int(code)))
        assert float(v) == float(val)
        assert np.signbit(v) == val.startswith("-")


def _e2m1_nearest(a):
    """Independent encoder: nearest grid value, ties to the even code, saturating."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    d = np.abs(a[:, None].astype(np.float64) - grid[None, :])
    best = np.argmin(d, axis=1)                       # first minimum = lower code on a tie
    nxt = np.minimum(best + 1, 7)
    tie = (d[np.arange(len(a)), nxt] == d[np.arange(len(a)), best]) & (nxt != best)
    best = np.where(tie & (best % 2 == 1), nxt, best)
    best = np.where(a.astype(np.float64) >= 6.0, 7, best)     # saturation
    return best.astype(np.uint8)


def test_e2m1_exhaustive_decision_range():
    """Every FP32 magnitude in [2^-3, 2^3) (where all rounding decisions sit)."""
    for ex in range(-3, 3):
        base = np.uint32((ex + 127) << 23)
        for lo in range(0, 1 << 23, 1 << 21):
            u = base + np.arange(lo, lo + (1 << 21), dtype=np.uint32)
            a = u.view(np.float32)
            assert np.array_equal(F.e2m1_encode(a), _e2m1_nearest(a))


def test_e2m1_outside_range_and_sign():
    rng = np.random.default_rng(0)
    small = rng.uniform(0, 0.125, 100000).astype(np.float32)
    big = np.exp2(rng.uniform(3, 100, 100000)).astype(np.float32)
    for a in (small, big):
        assert np.array_equal(F.e2m1_encode(a), _e2m1_nearest(a))
    assert F.e2m1_encode(np.float32(np.inf)) == 7
    # the sign bit is kept on zero results
    assert F.e2m1_encode(np.float32(-0.0)) == 0x8
    assert F.e2m1_encode(np.float32(-0.1)) == 0x8
    assert F.e2m1_encode(np.float32(-5.5)) == 0xF
    vals = rng.normal(0, 3, 100000).astype(np.float32)
    assert np.array_equal(F.e2m1_encode(vals) & 7, _e2m1_nearest(np.abs(vals)))
    assert np.array_equal(F.e2m1_encode(vals) >> 3, np.signbit(vals).astype(np.uint8))


def test_e2m1_tie_points():
    # midpoint: (code on the tie, code just above, code just below)
    ties = {0.25: (0, 1, 0), 0.75: (2, 2, 1), 1.25: (2, 3, 2), 1.75: (4, 4, 3),
            2.5: (4, 5, 4), 3.5: (6, 6, 5), 5.0: (6, 7, 6)}
    for t, (c, up, dn) in ties.items():
        assert F.e2m1_encode(np.float32(t)) == c
        assert F.e2m1_encode(np.nextafter(np.float32(t), np.float32(10))) == up
        assert F.e2m1_encode(np.nextafter(np.float32(t), np.float32(0))) == dn


# ----------------------------------------------------------------------------- UE4M3
def _ue4m3_table():
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


def _ue4m3_nearest(t):
    tab = _ue4m3_table()                                 # 127 values, increasing
    t = np.asarray(t, dtype=np.float64)
    hi = np.clip(np.searchsorted(tab, t, side="left"), 1, len(tab) - 1)
    lo = hi - 1
    dl, dh = t - tab[lo], tab[hi] - t
    pick = np.where(dh < dl, hi, lo)
    tie = dh == dl
    pick = np.where(tie, np.where(hi % 2 == 0, hi, lo), pick)
    pick = np.where(t >= tab[-1], len(tab) - 1, pick)
    pick = np.where(t <= 0, 0, pick)
    return pick.astype(np.uint8)


def test_ue4m3_table_and_max():
    assert np.allclose(F.ue4m3_decode(np.arange(0x7F)), _ue4m3_table(), rtol=0, atol=0)
    assert F.ue4m3_decode(0x7E) == 448.0
    assert F.ue4m3_decode(0x01) == 2.0 ** -9
    assert F.ue4m3_encode(1e30) == 0x7E
    assert F.ue4m3_encode(2.0 ** -10) == 0          # tie between 0 and 2^-9 -> even (0)
    assert F.ue4m3_encode(np.nextafter(2.0 ** -10, 1.0)) == 1


def test_ue4m3_dense_sweep():
    """Every FP32 pattern near each rounding midpoint plus a dense stride over [2^-12, 2^10)."""
    tab = _ue4m3_table()
    mids = (tab[:-1] + tab[1:]) / 2
    pts = [np.float32(x) for x in np.concatenate([tab, mids])]
    probe = []
    for p in pts:
        u = np.array([p], dtype=np.float32).view(np.uint32)[0]
        probe.append((np.arange(-64, 65, dtype=np.int64) + int(u)).astype(np.uint32))
    probe = np.concatenate(probe).view(np.float32)
    probe = probe[(probe >= 0) & np.isfinite(probe)]
    stride = (np.arange(((127 - 12) << 23), ((127 + 10) << 23), 977, dtype=np.int64)
              .astype(np.uint32).view(np.float32))
    for t in (probe, stride):
        assert np.array_equal(F.ue4m3_encode(t), _ue4m3_nearest(t))


# ----------------------------------------------------------------------------- UE8M0 / MX rules
def test_ue8m0_bytes_roundtrip():
    for b in range(0, 255):
        val = F.ue8m0_decode(b)
        assert val == 2.0 ** (b - 127)
    # a block whose maximum is exactly 4 * 2^e (code 6 at scale 2^e) maps back to byte e+127
    for e in range(-125, 126):
        amax = np.float32(np.ldexp(4.0, e)) if abs(e) < 120 else None
        if amax is None or not np.isfinite(amax) or amax == 0:
            continue
        assert F.mx_exponent(amax) == e


def test_mx_rules_golden():
    for amax, e_ocp, e_uos, c_ocp, c_uos in _load("mx_scale_rules.txt"):
        a = np.float32(float(amax))
        eo = int(F.mx_exponent(a, 0.0))
        eu = int(F.mx_exponent(a, 7.25))
        assert eo == int(e_ocp), amax
        assert eu == int(e_uos), amax
        assert F.e2m1_encode(np.ldexp(np.float64(a), -eo)) == int(c_ocp)
        assert F.e2m1_encode(np.ldexp(np.float64(a), -eu)) == int(c_uos)


def test_mx_uos_is_smallest_exponent():
    rng = np.random.default_rng(1)
    amax = np.exp2(rng.uniform(-30, 30, 20000)).astype(np.float32)
    for qmax in (6.0, 7.25, 8.0):
        e = F.mx_exponent(amax, qmax)
        assert np.all(amax <= np.ldexp(qmax, e))
        assert np.all(amax > np.ldexp(qmax, e - 1))
    e = F.mx_exponent(amax, 0.0)
    assert np.all(amax < np.ldexp(8.0, e)) and np.all(amax >= np.ldexp(8.0, e - 1))
    assert F.mx_exponent(np.float32(0.0)) == -127


def test_nvfp4_golden():
    for amax, g, sb, sv, code, deq in _load("nvfp4_cases.txt"):
        x = np.zeros((1, 16), dtype=np.float32)
        x[0, 3] = np.float32(float(amax))
        codes, s = F.quantize_blocks(x, "nvfp4", 0.0, float(g))
        assert int(s[0]) == int(sb, 16), amax
        assert float(F.ue4m3_decode(s[0])) == float(sv)
        assert int(codes[0, 3]) == int(code)
        assert F.dequantize_blocks(codes, s, "nvfp4", float(g))[0, 3] == pytest.approx(float(deq), rel=1e-7)


# ----------------------------------------------------------------------------- round trips
@pytest.mark.parametrize("qmax", [0.0, 6.0, 7.25])
def test_mxfp4_roundtrip_all_scales_and_codes(qmax):
    e = np.arange(-120, 121)
    codes = np.arange(16, dtype=np.uint8)
    vals = F.e2m1_decode(codes)
    x = np.zeros((len(e), 2, 32), dtype=np.float64)
    x[:, 0, :16] = vals[None, :] * np.exp2(e)[:, None]
    x[:, 0, 16] = 6.0 * np.exp2(e)                       # the block maximum 6 * 2^e
    x[:, 1, :16] = vals[None, :] * np.exp2(e)[:, None]
    x[:, 1, 16] = -6.0 * np.exp2(e)
    c, s = F.quantize_blocks(x.astype(np.float32), "mxfp4", qmax)
    assert np.all(s == (e + 127)[:, None])
    assert np.array_equal(c[:, 0, :16], np.broadcast_to(codes, (len(e), 16)))
    back = F.dequantize_blocks(c, s, "mxfp4")
    assert np.array_equal(back, x)


@pytest.mark.parametrize("g", [1.0, 0.5, 3.0])
def test_nvfp4_roundtrip_all_scales_and_codes(g):
    sbytes = np.arange(1, 0x7F, dtype=np.uint8)          # the 126 finite non-zero UE4M3 values
    sv = F.ue4m3_decode(sbytes) * g
    codes = np.arange(16, dtype=np.uint8)
    x = np.zeros((len(sbytes), 16), dtype=np.float64)
    x[:, :15] = F.e2m1_decode(codes[:15])[None, :] * sv[:, None]
    x[:, 15] = -6.0 * sv
    c, s = F.quantize_blocks(x.astype(np.float32), "nvfp4", 0.0, g)
    assert np.array_equal(s, sbytes)
    assert np.array_equal(c[:, :15], np.broadcast_to(codes[:15], (len(sbytes), 15)))
    assert np.all(c[:, 15] == 0xF)
    assert np.array_equal(F.dequantize_blocks(c, s, "nvfp4", g), x)


def test_pack_order_and_layouts():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert F.pack_nibbles(codes).tolist() == [[0x21, 0x43]]
    assert np.array_equal(F.unpack_nibbles(F.pack_nibbles(codes)), codes)
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 64)).astype(np.float32)
    p, s = F.quantize_rows(x, "nvfp4")
    assert p.shape == (5, 32) and s.shape == (5, 4)
    # transposed quantisation = row quantisation of the transpose (with zero padding)
    v = rng.normal(size=(40, 16)).astype(np.float32)
    pt, st = F.quantize_cols_transposed(v, "mxfp4")
    vt = np.zeros((16, 64), dtype=np.float32)
    vt[:, :40] = v.T
    p2, s2 = F.quantize_rows(vt, "mxfp4")
    assert np.array_equal(pt, p2) and np.array_equal(st, s2)


def test_quantization_error_bound():
    """|x - x_hat| <= half the local grid step * scale, except for clipped values (|y| > 6)."""
    rng = np.random.default_rng(3)
    x = rng.normal(size=(4096, 16)).astype(np.float32)
    c, s = F.quantize_blocks(x, "nvfp4")
    xh = F.dequantize_blocks(c, s, "nvfp4")
    sc = F.ue4m3_decode(s)[:, None]
    y = np.abs(x) / sc
    step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    ok = y <= 6.0
    assert np.all(np.abs(x - xh)[ok] <= 0.5 * step[ok] * sc.repeat(16, 1)[ok] * (1 + 1e-6))


def test_smoothing_multiplier_enters_before_amax():
    x = np.ones((1, 16), dtype=np.float32)
    mul = np.full((1, 16), 4.0, dtype=np.float32)
    p1, s1 = F.quantize_rows(x * 4.0, "nvfp4")
    p2, s2 = F.quantize_rows(x, "nvfp4", mul=mul)
    assert np.array_equal(p1, p2) and np.array_equal(s1, s2)


def test_transposed_quantisation_hand_worked():
    """quantize_cols_transposed against bytes worked out by hand (NVFP4, blocks of 16 tokens,
    one block per channel and half of the 32 tokens):
      channel 0, tokens 0..3 = 6, 3, -1.5, 0.5: amax 6 -> t = 6 / 6 = 1 -> UE4M3 0x38 (exponent
        field 7), codes 7 (6), 5 (3), 8|3 (-1.5), 1 (0.5) -> bytes 0x57, 0x1B (low nibble first);
      channel 1, tokens 0..3 = 2, 1, 0.5, -2: t = 2 / 6 rounds to 1.375 * 2^-2 = 0.34375 ->
        UE4M3 0x2B; y = 5.818, 2.909, 1.455, -5.818 round to 6, 3, 1.5, -6 -> codes 7, 5, 3,
        8|7 -> bytes 0x57, 0xF3;
      every other token is 0, so the second block of each channel has scale byte 0."""
    v = np.zeros((32, 2), dtype=np.float32)
    v[:4, 0] = [6.0, 3.0, -1.5, 0.5]
    v[:4, 1] = [2.0, 1.0, 0.5, -2.0]
    p, s = F.quantize_cols_transposed(v, "nvfp4")
    assert p.shape == (2, 16) and s.shape == (2, 2)
    expect_p = np.zeros((2, 16), dtype=np.uint8)
    expect_p[0, :2] = [0x57, 0x1B]
    expect_p[1, :2] = [0x57, 0xF3]
    assert p.tolist() == expect_p.tolist()
    assert s.tolist() == [[0x38, 0x00], [0x2B, 0x00]]
    # MXFP4 (blocks of 32 tokens, OCP rule): amax 6 -> e = floor(log2 6) - 2 = 0 -> E8M0 127,
    # the values are their own codes; a channel of zeros gets the smallest exponent (E8M0 0)
    pm, sm = F.quantize_cols_transposed(v[:, :1] * np.float32(1.0), "mxfp4")
    assert pm.shape == (1, 16) and sm.tolist() == [[127]]
    assert pm[0, :2].tolist() == [0x57, 0x1B] and not pm[0, 2:].any()

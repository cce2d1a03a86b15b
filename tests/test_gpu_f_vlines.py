"""Vertical-line identification on the GPU against the oracle (HyQuant column mass):
masses element by element, the selected set a valid top-n of the oracle's masses within
the masses' error band, positions / exclusion mask / gathered BF16 rows exact, the count
rule, planted heavy hitters, and the full-size decode configuration on sampled groups."""
import math

import numpy as np
import pytest

import synth
from oracle import hyquant as H

pytestmark = pytest.mark.gpu


def _bf16(a):
    return synth.round_to_bf16(np.asarray(a, dtype=np.float32))


def _run(q_obs, k, v, n_prefix, rho=0.05):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(torch.bfloat16)
    npf = torch.tensor(n_prefix, dtype=torch.int32, device=dev)
    res = fa4q.select_vertical_lines(t(q_obs), t(k), t(v), npf, rho=rho)
    torch.cuda.synchronize()
    return {n: (x.float().cpu().numpy() if x.dtype == torch.bfloat16 else x.cpu().numpy()) for n, x in res.items()}


def _check_group(res, b, h, q_obs, k, v, n, rho, G):
    R = q_obs.shape[2] * G
    qo = q_obs[b, h * G:(h + 1) * G].reshape(R, -1)
    ref = H.column_mass(qo, k[b, h, :n])
    got = res["mass"][b, h]
    err = np.abs(got[:n] - ref)
    assert err.max() <= 1e-4 * ref.max() + 1e-7, f"mass err {err.max():.3e} (max {ref.max():.3e})"
    assert np.all(got[n:] == 0.0)
    assert abs(got[:n].sum() - R) <= 1e-3 * R
    cnt = int(math.ceil(rho * n - 1e-9))
    assert int(res["counts"][b, h]) == cnt
    pos = res["positions"][b, h, :cnt]
    assert np.all(np.diff(pos) > 0) and pos.min() >= 0 and pos.max() < n
    # valid top-cnt of the oracle's masses within the error band of the GPU masses
    band = 2.0 * err.max() + 1e-12
    thr = np.sort(ref)[-cnt]
    assert ref[pos].min() >= thr - band
    rest = np.setdiff1d(np.arange(n), pos)
    if len(rest):
        assert ref[rest].max() <= thr + band
    # exclusion words and gathered rows are exact
    words = res["excl"][b, h].view(np.uint64)
    bits = np.zeros(len(words) * 64, dtype=bool)
    bits[pos] = True
    expect = np.packbits(bits.reshape(-1, 64)[:, ::-1], axis=1).view(">u8").ravel().astype(np.uint64)
    assert np.array_equal(words, expect)
    assert np.array_equal(res["hp_k"][b, h, :cnt], k[b, h, pos])
    assert np.array_equal(res["hp_v"][b, h, :cnt], v[b, h, pos])
    return len(np.intersect1d(pos, np.sort(np.argsort(-ref, kind="stable")[:cnt]))) / max(cnt, 1)


@pytest.mark.parametrize("d,Hq,Hkv,n_obs,L,n_prefix", [
    (64, 4, 2, 16, 1000, [872, 500]),
    (128, 8, 2, 8, 2100, [2100, 1]),
    (128, 4, 4, 64, 777, [650, 0]),
])
def test_select_vertical_lines_small(d, Hq, Hkv, n_obs, L, n_prefix):
    rng = np.random.default_rng(d + L)
    B = len(n_prefix)
    q_obs = _bf16(rng.normal(size=(B, Hq, n_obs, d)))
    k = _bf16(rng.normal(size=(B, Hkv, L, d)) * 1.3)
    v = _bf16(rng.normal(size=(B, Hkv, L, d)))
    res = _run(q_obs, k, v, n_prefix)
    for b in range(B):
        for h in range(Hkv):
            if n_prefix[b] == 0:
                assert int(res["counts"][b, h]) == 0 and np.all(res["mass"][b, h] == 0.0)
                assert np.all(res["excl"][b, h] == 0)
                continue
            _check_group(res, b, h, q_obs, k, v, n_prefix[b], 0.05, Hq // Hkv)


def test_select_vertical_lines_recovers_planted():
    rng = np.random.default_rng(41)
    B, Hq, Hkv, n_obs, L, d = 1, 4, 1, 16, 3000, 128
    u = rng.normal(size=d)
    u /= np.linalg.norm(u)
    planted = np.sort(rng.choice(2800, 140, replace=False))
    k = rng.normal(size=(B, Hkv, L, d))
    k[0, 0, planted] += 6.0 * u          # the oracle recovers 137 of the 140 on these inputs
    q_obs = _bf16(rng.normal(size=(B, Hq, n_obs, d)) + 3.0 * u)
    k, v = _bf16(k), _bf16(rng.normal(size=(B, Hkv, L, d)))
    res = _run(q_obs, k, v, [2800])
    assert int(res["counts"][0, 0]) == 140
    assert len(np.intersect1d(res["positions"][0, 0, :140], planted)) >= 133
    _check_group(res, 0, 0, q_obs, k, v, 2800, 0.05, Hq)


def test_select_vertical_lines_decode_workload_sampled():
    """The decode configuration (32 sequences, 32/8 heads, 32768 keys, 64 observation queries
    per q-head, 5% of the 32640-token prefix) in one call; three groups checked in full."""
    w = synth.WORKLOADS[4]
    B, Hq, Hkv, d, L = w.B, w.Hq, w.Hkv, w.d, w.L
    q_obs = np.stack([synth.decode_observation_queries(w, b) for b in range(B)])
    k = np.stack([np.stack([synth.decode_kv_slice(w, "k", b, h) for h in range(Hkv)]) for b in range(B)])
    v = np.stack([np.stack([synth.decode_kv_slice(w, "v", b, h) for h in range(Hkv)]) for b in range(B)])
    res = _run(q_obs, k, v, [w.fp4_len] * B, rho=w.hp_frac)
    assert np.all(res["counts"] == w.n_hp)
    overlaps = [_check_group(res, b, h, q_obs, k, v, w.fp4_len, w.hp_frac, Hq // Hkv)
                for (b, h) in [(0, 0), (17, 5), (31, 7)]]
    assert min(overlaps) >= 0.9, overlaps


def test_identify_quantize_decode_pipeline():
    """Identification -> page quantisation with its exclusion mask -> decode with its BF16
    rows, against the oracle's hybrid decode over the positions the GPU selected (the
    selection itself is checked above; here every later step must agree on it)."""
    import dataclasses
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    from oracle import decode as OD
    from fa4q_testlib import assert_close
    w = dataclasses.replace(synth.WORKLOADS[4], B=3, L=2200)
    dev = torch.device("cuda:0")
    B, Hq, Hkv, d, L, W, P = w.B, w.Hq, w.Hkv, w.d, w.L, w.window, w.n_pages
    host = {(b, h): (synth.decode_kv_slice(w, "k", b, h), synth.decode_kv_slice(w, "v", b, h))
            for b in range(B) for h in range(Hkv)}
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(torch.bfloat16)
    tK = bf(np.stack([np.stack([host[(b, h)][0] for h in range(Hkv)]) for b in range(B)]))
    tV = bf(np.stack([np.stack([host[(b, h)][1] for h in range(Hkv)]) for b in range(B)]))
    Q = np.stack([synth.decode_query(w, b) for b in range(B)])
    q_obs = bf(np.stack([synth.decode_observation_queries(w, b) for b in range(B)]))
    fp4_len = torch.full((B,), w.fp4_len, dtype=torch.int32, device=dev)
    sel = fa4q.select_vertical_lines(q_obs, tK, tV, fp4_len, rho=w.hp_frac)
    excl = sel["excl"][:, :, :P].contiguous()           # the cache's pages only
    table = torch.from_numpy(synth.decode_block_table(w).astype(np.int32)).to(dev)
    kp, ks, vp, vs = fa4q.quantize_kv_pages(tK, tV, fp4_len, excl, table, B * P)
    wl = torch.full((B,), W, dtype=torch.int32, device=dev)
    out = fa4q.decode(bf(Q), kp, ks, vp, vs, table, fp4_len, excl, sel["hp_k"], sel["hp_v"], sel["counts"],
                      tK[:, :, w.fp4_len:].contiguous(), tV[:, :, w.fp4_len:].contiguous(), wl)
    out = out.float().cpu().numpy()
    assert fa4q.device_status()[0] == 0
    pos, cnt = sel["positions"].cpu().numpy(), sel["counts"].cpu().numpy()
    G = Hq // Hkv
    gs, rs = [], []
    for b in range(B):
        for h in range(Hkv):
            kk, vv = host[(b, h)]
            ref = OD.decode_group(Q[b, h * G:(h + 1) * G], kk, vv, pos[b, h, :cnt[b, h]], W, "nvfp4")
            gs.append(out[b, h * G:(h + 1) * G])
            rs.append(synth.round_to_bf16(np.asarray(ref, dtype=np.float32)))
    assert_close(np.stack(gs), np.stack(rs), what="identify+decode")

"""fa4q_attn_fwd_hybrid (HyQuant hybrid-precision prefill: window and vertical-line keys in
BF16, the rest FP4, one online softmax) against the oracle's hybrid prefill, element by
element; max-abs <= 2e-2, mean-rel <= 2e-3 (the BF16 part's probabilities enter its PV
tiles rounded to bf16)."""
import numpy as np
import pytest

import synth
from oracle import attention as OA
from oracle import hybrid as OH
from fa4q_testlib import assert_close, to_dev_bf16

pytestmark = pytest.mark.gpu


def _rand(shape, seed, scale=1.0):
    return synth.round_to_bf16(np.random.default_rng(seed).normal(size=shape).astype(np.float32)
                               * np.float32(scale))


def _vlines(S, n, seed):
    return np.sort(np.random.default_rng(seed).choice(S, n, replace=False)).astype(np.int32)


def run_hybrid(q, k, v, vls, window, fmt, qmax_p=0.0, out_fp32=True):
    """q [B,Hq,S,d], k/v [B,Hkv,S,d] bf16 values; vls[b][h] vertical-line positions or None."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    B, Hq, S, d = q.shape
    Hkv = k.shape[1]
    kz, vz = k.copy(), v.copy()
    max_vl = 0 if vls is None else max(1, max(len(vls[b][h]) for b in range(B) for h in range(Hkv)))
    if vls is not None:
        pos = np.zeros((B, Hkv, max_vl), np.int32)
        cnt = np.zeros((B, Hkv), np.int32)
        vk = np.zeros((B, Hkv, max_vl, d), np.float32)
        vv = np.zeros((B, Hkv, max_vl, d), np.float32)
        words = (S + 63) // 64
        ex = np.zeros((B, Hkv, words), np.uint64)
        for b in range(B):
            for h in range(Hkv):
                p = vls[b][h]
                pos[b, h, :len(p)] = p
                cnt[b, h] = len(p)
                vk[b, h, :len(p)] = k[b, h, p]
                vv[b, h, :len(p)] = v[b, h, p]
                for x in p:
                    ex[b, h, x // 64] |= np.uint64(1) << np.uint64(x % 64)
                kz[b, h, p] = 0.0
                vz[b, h, p] = 0.0
        t_pos = torch.from_numpy(pos).to(dev)
        t_cnt = torch.from_numpy(cnt).to(dev)
        t_vk, t_vv = to_dev_bf16(vk, dev), to_dev_bf16(vv, dev)
        t_ex = torch.from_numpy(ex.view(np.int64)).to(dev)
    else:
        t_pos = t_cnt = t_vk = t_vv = t_ex = None
    tq, tk, tv = to_dev_bf16(q, dev), to_dev_bf16(k, dev), to_dev_bf16(v, dev)
    pq, sq = fa4q.quantize(tq, fmt, fa4q.FA4Q_AXIS_INNER)
    pk, sk = fa4q.quantize(to_dev_bf16(kz, dev), fmt, fa4q.FA4Q_AXIS_INNER)
    pv, sv = fa4q.quantize(to_dev_bf16(vz, dev), fmt, fa4q.FA4Q_AXIS_OUTER)
    out = fa4q.attn_fwd_hybrid(pq, sq, pk, sk, pv, sv, tq, tk, tv, t_pos, t_cnt, t_vk, t_vv, t_ex,
                               B=B, Hq=Hq, Hkv=Hkv, S=S, d=d, window=window, fmt=fmt, qmax_p=qmax_p,
                               out_fp32=out_fp32)
    torch.cuda.synchronize()
    code, detail = fa4q.device_status()
    assert code == 0, f"device status {code} detail {detail:#x}"
    return out.float().cpu().numpy(), kz, vz


def oracle_hybrid(q, k, v, kz, vz, vls, window, fmt, qmax_p=0.0, rows=None, heads=None):
    B, Hq, S, d = q.shape
    Hkv = k.shape[1]
    res = {}
    for (b, h) in (heads or [(b, h) for b in range(B) for h in range(Hq)]):
        hk = h * Hkv // Hq
        qh, kh, vh = OA.quantize_qkv(q[b, h], kz[b, hk], vz[b, hk], fmt)
        vl = np.zeros(0, np.int64) if vls is None else vls[b][hk]
        res[(b, h)] = OH.hybrid_prefill_head(q[b, h], k[b, hk], v[b, hk], qh, kh, vh, vl, window, fmt,
                                             qmax_p=qmax_p, rows=rows)
    return res


@pytest.mark.parametrize("fmt,S,Hq,Hkv,window,frac", [
    ("nvfp4", 384, 2, 1, 128, 0.05),
    ("mxfp4", 520, 4, 2, 128, 0.05),
    ("nvfp4", 300, 2, 2, 64, 0.10),
    ("mxfp4", 200, 2, 1, 128, 0.0),     # window only
    ("nvfp4", 100, 2, 1, 128, 0.05),    # every key inside the window: no FP4 key at all
])
def test_hybrid_prefill(fmt, S, Hq, Hkv, window, frac):
    d = 128
    q = _rand((1, Hq, S, d), S + 1, 1.5)
    k = _rand((1, Hkv, S, d), S + 2, 1.5)
    v = _rand((1, Hkv, S, d), S + 3)
    n = int(frac * S)
    vls = None if n == 0 else [[_vlines(S, n, 10 * h + 4) for h in range(Hkv)]]
    got, kz, vz = run_hybrid(q, k, v, vls, window, fmt)
    ref = oracle_hybrid(q, k, v, kz, vz, vls, window, fmt)
    assert_close(np.stack([got[0, h] for h in range(Hq)]), np.stack([ref[(0, h)] for h in range(Hq)]),
                 what=f"hybrid {fmt} S={S} W={window}")


def test_hybrid_full_size_sampled_rows():
    """The causal GQA NVFP4 shape at S = 4096 (32/8 heads) with 5% vertical lines per kv-head
    and a 128-token window, sampled rows of three heads."""
    w = synth.WORKLOADS[3]
    S, d = 4096, 128
    q, k, v = synth.prefill_inputs(w, S=S)
    vls = [[_vlines(S, int(0.05 * S), 100 + h) for h in range(w.Hkv)]]
    got, kz, vz = run_hybrid(q, k, v, vls, 128, w.fmt)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, 255, 2048, S - 129, S - 1],
                                     np.random.default_rng(5).choice(S, 20, replace=False)]))
    heads = [(0, 0), (0, 13), (0, w.Hq - 1)]
    ref = oracle_hybrid(q, k, v, kz, vz, vls, 128, w.fmt, rows=rows, heads=heads)
    assert_close(np.stack([got[0, h][rows] for (_, h) in heads]), np.stack([ref[hh] for hh in heads]),
                 what="hybrid full size")

"""fa4q_attn_fwd against the oracle's tiled PNQ attention (element by element).

Tolerance (stated for the path): max-abs <= 2e-2 and mean-rel <= 2e-3, mean-rel being
sum|gpu - oracle| / sum|oracle| over the checked elements."""
import numpy as np
import pytest

import synth
from oracle import attention as OA
from oracle import smooth as OS
from fa4q_testlib import assert_close, to_dev_bf16

pytestmark = pytest.mark.gpu


def run_prefill(q, k, v, fmt, causal, qmax=0.0, qmax_p=0.0, lam=None, out_fp32=True, want_lse=False,
                tau=0, l_from_ptilde=False):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    B, Hq, S, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    mq = mk = None
    if lam is not None:
        mq = torch.from_numpy(lam).to(dev)
        mk = torch.from_numpy((1.0 / lam.astype(np.float64)).astype(np.float32)).to(dev)
    pq, sq = fa4q.quantize(to_dev_bf16(q, dev), fmt, fa4q.FA4Q_AXIS_INNER, qmax, 1.0, mq, Hq, Hq // Hkv)
    pk, sk = fa4q.quantize(to_dev_bf16(k, dev), fmt, fa4q.FA4Q_AXIS_INNER, qmax, 1.0, mk, Hkv, 1)
    pv, sv = fa4q.quantize(to_dev_bf16(v, dev), fmt, fa4q.FA4Q_AXIS_OUTER, qmax)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev) if want_lse else None
    out = fa4q.attn_fwd(pq, sq, pk, sk, pv, sv, B=B, Hq=Hq, Hkv=Hkv, S_q=S, S_k=Sk, d=d, fmt=fmt,
                        causal=causal, qmax_p=qmax_p, out_fp32=out_fp32, lse=lse, rescale_tau=tau,
                        l_from_ptilde=l_from_ptilde)
    torch.cuda.synchronize()
    code, detail = fa4q.device_status()
    assert code == 0, f"device status {code} detail {detail:#x}"
    o = out.float().cpu().numpy()
    return (o, lse.cpu().numpy()) if want_lse else o


def _rand(shape, seed, scale=1.0):
    return synth.round_to_bf16(np.random.default_rng(seed).normal(size=shape).astype(np.float32)
                               * np.float32(scale))


def check(q, k, v, fmt, causal, qmax=0.0, qmax_p=0.0, lam=None, rows=None, heads=None, what="",
          tau=0):
    got = run_prefill(q, k, v, fmt, causal, qmax, qmax_p, lam, tau=tau)
    ref = OA.prefill(q, k, v, causal=causal, fmt=fmt, qmax=qmax, qmax_p=qmax_p, lam=lam, rows=rows,
                     heads=heads, rescale_tau=tau)
    gs, rs = [], []
    for (b, h), r in ref.items():
        gs.append(got[b, h] if rows is None else got[b, h][rows])
        rs.append(r)
    return assert_close(np.stack(gs), np.stack(rs), what=what)


def test_tiny_noncausal_workload():
    w = synth.WORKLOADS[1]
    q, k, v = synth.prefill_inputs(w)
    check(q, k, v, "nvfp4", False, what="tiny")


@pytest.mark.parametrize("fmt,causal,d,S,Hq,Hkv,B,qmax", [
    ("nvfp4", True, 128, 384, 4, 2, 1, 0.0),
    ("mxfp4", True, 128, 256, 2, 2, 1, 7.25),
    ("nvfp4", False, 64, 200, 2, 1, 2, 0.0),
    ("mxfp4", True, 128, 333, 4, 4, 1, 0.0),
    ("mxfp4", False, 64, 300, 2, 2, 1, 0.0),
    ("nvfp4", True, 64, 129, 2, 2, 1, 0.0),
    ("nvfp4", False, 128, 1, 1, 1, 1, 0.0),
    ("nvfp4", True, 128, 1, 1, 1, 1, 0.0),
])
def test_prefill_shapes(fmt, causal, d, S, Hq, Hkv, B, qmax):
    q = _rand((B, Hq, S, d), S + d, 1.5)
    k = _rand((B, Hkv, S, d), S + d + 1, 1.5)
    v = _rand((B, Hkv, S, d), S + d + 2)
    check(q, k, v, fmt, causal, qmax, qmax, what=f"{fmt} causal={causal} d={d} S={S}")


def test_noncausal_unequal_lengths():
    q = _rand((1, 2, 256, 128), 7)
    k = _rand((1, 2, 520, 128), 8)
    v = _rand((1, 2, 520, 128), 9)
    check(q, k, v, "nvfp4", False, what="Sq != Sk")


def test_bf16_output_and_lse():
    q = _rand((1, 2, 256, 128), 10, 2.0)
    k = _rand((1, 2, 256, 128), 11, 2.0)
    v = _rand((1, 2, 256, 128), 12)
    for fmt in ("nvfp4", "mxfp4"):
        o16 = run_prefill(q, k, v, fmt, True, out_fp32=False)
        _, lse = run_prefill(q, k, v, fmt, True, want_lse=True)
        ref = OA.prefill(q, k, v, causal=True, fmt=fmt, return_lse=True)
        for (b, h), (r, rl) in ref.items():
            r16 = synth.round_to_bf16(r.astype(np.float32))
            assert_close(o16[b, h], r16, what=f"bf16 out {fmt}")
            assert np.max(np.abs(lse[b, h] - rl)) <= 1e-3


def test_smoothed_mxfp4_gqa_recipe():
    w = synth.WORKLOADS[2]
    q, k, v = synth.prefill_inputs(w, S=512)
    qc, kc = synth.calibration_inputs(w)
    lam = OS.calibrate(qc, kc)
    check(q, k, v, "mxfp4", True, lam=lam, what="smoothed")


@pytest.mark.parametrize("fmt,causal,S,Hq,Hkv,B", [
    ("mxfp4", True, 1000, 40, 8, 1),     # 320 items of 1..8 key tiles, several per CTA
    ("nvfp4", False, 200, 80, 16, 2),    # 320 items of 2 key tiles (ragged last tile)
])
def test_prefill_persistent_many_short_items(fmt, causal, S, Hq, Hkv, B):
    """More work items than SMs, all short: the kernel runs persistently (one CTA per SM
    walking the longest-first item list), so CTAs carry their barrier phases, Q slots and
    accumulators from one item to the next; heads spread over the list are checked."""
    d = 128
    q = _rand((B, Hq, S, d), S + 7, 1.5)
    k = _rand((B, Hkv, S, d), S + 8, 1.5)
    v = _rand((B, Hkv, S, d), S + 9)
    heads = [(0, 0), (0, 1), (B - 1, Hq // 2), (B - 1, Hq - 3), (B - 1, Hq - 1)]
    check(q, k, v, fmt, causal, heads=heads, what=f"persistent {fmt} causal={causal}")


def _rows(S, n_rand, seed):
    base = [0, 1, 127, 128, 129, S // 2, S - 129, S - 128, S - 1]
    rnd = np.random.default_rng(seed).choice(S, n_rand, replace=False)
    return np.unique(np.concatenate([base, rnd]))


@pytest.mark.parametrize("wid", [2, 3, 5])
def test_full_size_workloads_sampled_rows(wid):
    """The full-size workloads in the benchmark's launch configuration; the oracle checks
    sampled rows (rows are independent) of a few heads."""
    w = synth.WORKLOADS[wid]
    q, k, v = synth.prefill_inputs(w)
    lam = None
    if w.smooth:
        lam = OS.calibrate(*synth.calibration_inputs(w))
    rows = _rows(w.S, 23, wid)
    heads = [(0, 0), (0, w.Hq // 2 + 1), (0, w.Hq - 1)]
    check(q, k, v, w.fmt, w.causal, w.qmax, w.qmax_p, lam, rows=rows, heads=heads, what=w.name)


@pytest.mark.parametrize("fmt,causal,S,Hq,Hkv,tau", [
    ("mxfp4", True, 700, 4, 2, 8),       # holds keys equal to a kept reference (E2M1 tie 0.25)
    ("mxfp4", False, 450, 2, 2, 4),
    ("mxfp4", False, 300, 2, 1, 1),
    ("mxfp4", True, 129, 2, 2, 8),
])
def test_conditional_rescale(fmt, causal, S, Hq, Hkv, tau):
    """fa4q_attn_fwd_ex (reference maximum kept within tau binades) against the oracle's
    conditional-rescale variant; keys grow along the sequence so the reference is often
    kept while later tiles exceed it.  (NVFP4 with tau > 0 is refused on the host.)"""
    d = 128
    q = _rand((1, Hq, S, d), S + tau, 1.5)
    k = _rand((1, Hkv, S, d), S + tau + 1, 1.5) * np.linspace(0.6, 1.4, S, dtype=np.float32)[:, None]
    k = synth.round_to_bf16(k.astype(np.float32))
    v = _rand((1, Hkv, S, d), S + tau + 2)
    check(q, k, v, fmt, causal, tau=tau, what=f"rescale tau={tau} {fmt} causal={causal}")


def test_conditional_rescale_full_size_sampled_rows():
    """The causal GQA MXFP4 workload (the benchmark's) with tau = 8, sampled rows."""
    w = synth.WORKLOADS[2]
    q, k, v = synth.prefill_inputs(w)
    lam = OS.calibrate(*synth.calibration_inputs(w))
    rows = _rows(w.S, 23, 8)
    heads = [(0, 0), (0, w.Hq - 1)]
    check(q, k, v, w.fmt, w.causal, w.qmax, w.qmax_p, lam, rows=rows, heads=heads, what="tau=8 w2", tau=8)


@pytest.mark.parametrize("fmt,causal,S,Hq,Hkv", [
    ("nvfp4", False, 384, 2, 2),
    ("mxfp4", True, 520, 4, 2),
    ("nvfp4", True, 300, 2, 1),
])
def test_inconsistent_normaliser(fmt, causal, S, Hq, Hkv):
    """l_from_ptilde: normaliser from the unquantised exponentials (the HiFA4 baseline)
    against the oracle's inconsistent variant; and, from the two GPU outputs, the
    coherent per-row scaling sum P_hat / sum P~ with net mass loss (median below 1)."""
    d = 128
    q = _rand((1, Hq, S, d), S + 31, 1.5)
    k = _rand((1, Hkv, S, d), S + 32, 1.5)
    v = _rand((1, Hkv, S, d), S + 33)
    got = run_prefill(q, k, v, fmt, causal, l_from_ptilde=True)
    ref = OA.prefill(q, k, v, causal=causal, fmt=fmt, consistent=False)
    assert_close(np.stack([got[0, h] for h in range(Hq)]), np.stack([ref[(0, h)] for h in range(Hq)]),
                 what=f"inconsistent normaliser {fmt}")
    con = run_prefill(q, k, v, fmt, causal)
    rows = np.abs(con).min(axis=-1) > 1e-3              # rows without near-zero entries
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = got / con                               # per row: sum P_hat / sum P~ (used on `rows`)
    r = ratio[..., 0][rows]
    assert np.max(np.abs(ratio[rows] - r[:, None])) <= 1e-4     # one factor per row
    assert np.median(r) < 1.0                            # net mass loss

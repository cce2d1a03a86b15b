"""Error of the method against unquantised attention on the synthetic workloads, from the
oracle alone.

Test infrastructure like the rest of this package; run by hand:
    python -m oracle.report_accuracy [--rows 64] [--heads 2] [--groups 2]

Prefill workloads: for a fixed sample of (head, query row) pairs, the oracle's output of the
library's pipeline (block quantisation of Q, K, V, FP4 products, PNQ with the normaliser from
P_hat) against plain FP64 softmax attention on the same bf16 inputs; the inconsistent
normaliser (the HiFA4 baseline, from the unquantised exponentials) beside it.  Decode
workload: a few (sequence, kv-head) groups; the hybrid-cache decode (FP4 remainder, BF16
vertical lines and window) and the FP4 tensor-core decode (dual-residual query, all keys FP4)
against plain attention over every key.  mean_rel = sum|x - ref| / sum|ref| over the sample.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

from . import attention as OA
from . import bitdecode as BD
from . import decode as OD
from . import smooth as OS


def _err(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.abs(x - ref).max()), float(np.abs(x - ref).sum() / np.abs(ref).sum())


def prefill_rows(w, n_rows: int, n_heads: int, seed: int = 0):
    import synth
    q, k, v = synth.prefill_inputs(w)
    lam = OS.calibrate(*synth.calibration_inputs(w)) if w.smooth else None
    rng = np.random.default_rng(seed)
    heads = sorted(rng.choice(w.Hq, n_heads, replace=False).tolist())
    rows = np.sort(rng.choice(w.S, min(n_rows, w.S), replace=False))
    got, inc, ref = [], [], []
    for h in heads:
        kw = dict(causal=w.causal, fmt=w.fmt, qmax=w.qmax, qmax_p=w.qmax_p, lam=lam, rows=rows, heads=[(0, h)])
        got.append(OA.prefill(q, k, v, **kw)[(0, h)])
        inc.append(OA.prefill(q, k, v, consistent=False, **kw)[(0, h)])
        hk = h // (w.Hq // w.Hkv)
        ref.append(OA.attention_plain(q[0, h], k[0, hk], v[0, hk], causal=w.causal, rows=rows))
    return _err(np.stack(got), np.stack(ref)), _err(np.stack(inc), np.stack(ref)), len(heads) * len(rows)


def decode_groups(dw, n_groups: int):
    import synth
    G = dw.Hq // dw.Hkv
    tiles = (dw.n_pages + 1) // 2
    s = max(1, min(-(-1184 // (dw.B * dw.Hkv)), tiles))
    tps = -(-tiles // s)
    hyb, fp4q, ref = [], [], []
    for gi in range(n_groups):
        b, h = gi % dw.B, (gi * 3) % dw.Hkv
        q = synth.decode_query(dw, b)[h * G:(h + 1) * G]
        k = synth.decode_kv_slice(dw, "k", b, h)
        v = synth.decode_kv_slice(dw, "v", b, h)
        hp = synth.decode_hp_positions(dw, b, h)
        hyb.append(OD.decode_group(q, k, v, hp, dw.window, "nvfp4"))
        fp4q.append(BD.decode_group_fp4q(q, k, v, tps))
        ref.append(OA.attention_plain(q, k, v, causal=False))
    return _err(np.stack(hyb), np.stack(ref)), _err(np.stack(fp4q), np.stack(ref))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=64)
    ap.add_argument("--heads", type=int, default=2)
    ap.add_argument("--groups", type=int, default=2)
    ap.add_argument("--workloads", default="1,2,3,5")
    args = ap.parse_args()
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    print("| workload | sample | method vs unquantised: max-abs / mean-rel | "
          "inconsistent normaliser: max-abs / mean-rel |")
    print("|---|---|---|---|")
    for wid in [int(x) for x in args.workloads.split(",")]:
        w = synth.WORKLOADS[wid]
        (ma, mr), (ia, ir), n = prefill_rows(w, args.rows, args.heads)
        print(f"| {w.name} | {n} rows | {ma:.3g} / {mr:.3g} | {ia:.3g} / {ir:.3g} |")
    dw = synth.WORKLOADS[4]
    (ha, hr), (fa, fr) = decode_groups(dw, args.groups)
    G = dw.Hq // dw.Hkv
    print(f"| {dw.name}: hybrid-cache decode | {args.groups * G} q-heads | {ha:.3g} / {hr:.3g} | - |")
    print(f"| {dw.name}: FP4 tensor-core decode (all keys FP4) | {args.groups * G} q-heads | "
          f"{fa:.3g} / {fr:.3g} | - |")


if __name__ == "__main__":
    main()

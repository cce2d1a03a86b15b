"""The accuracy report bench.py adds beside the CPU baseline: on the oracle's sampled rows,
GPU vs oracle and each vs unquantised attention.  Checked on the CPU with a stand-in for the
GPU's bf16 output (the oracle's own output rounded to bf16, then a perturbed copy)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _full_oracle(w):
    import synth
    from oracle import attention as OA
    q, k, v = synth.prefill_inputs(w)
    ref = OA.prefill(q, k, v, causal=w.causal, fmt=w.fmt, qmax=w.qmax, qmax_p=w.qmax_p)
    out = np.zeros((w.B, w.Hq, w.S, w.d))
    for (b, h), r in ref.items():
        out[b, h] = r
    return out


def test_accuracy_report_fields_and_identities():
    import bench
    import synth
    w = synth.WORKLOADS[1]                      # B=1, H=2, S=128, d=64, NVFP4, non-causal
    exact = _full_oracle(w)
    out = synth.round_to_bf16(exact.astype(np.float32)).astype(np.float64)   # a bf16 output
    acc = {}
    bench.oracle_prefill_sample(w, 0.5, gpu_out=out, accuracy=acc)
    assert acc["rows"] > 0
    # the report rounds the oracle to bf16 before comparing: an exact bf16 result reads 0
    assert acc["gpu_vs_oracle"]["max_abs"] == 0.0 and acc["gpu_vs_oracle"]["mean_rel"] == 0.0
    # against unquantised attention the two differ by at most the bf16 rounding
    rnd = np.abs(out - exact).max()
    assert abs(acc["gpu_vs_unquantized"]["max_abs"] - acc["oracle_vs_unquantized"]["max_abs"]) <= rnd + 1e-12
    # 4-bit operands and probabilities: a few percent from unquantised attention
    assert 1e-3 < acc["oracle_vs_unquantized"]["mean_rel"] < 0.3
    # a perturbed "GPU" output: its distance to the oracle is reported, and by the triangle
    # inequality its error vs unquantised differs from the oracle's by at most that much
    rng = np.random.default_rng(1)
    noisy = out + rng.normal(scale=1e-3, size=out.shape)
    acc2 = {}
    bench.oracle_prefill_sample(w, 0.5, gpu_out=noisy, accuracy=acc2)
    d_go = acc2["gpu_vs_oracle"]["max_abs"]
    assert 0 < d_go < 1e-2
    assert abs(acc2["gpu_vs_unquantized"]["max_abs"] - acc2["oracle_vs_unquantized"]["max_abs"]) <= d_go + 1e-12


def test_no_report_without_gpu_output():
    import bench
    import synth
    acc = {}
    bench.oracle_prefill_sample(synth.WORKLOADS[1], 0.2, accuracy=acc)
    assert acc == {}

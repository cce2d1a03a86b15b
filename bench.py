"""Benchmark of the fused 4-bit microscaled FlashAttention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 5|2|3] [--no-sub] [--no-decode] [--no-cpu-baseline]

One step = one pass of the prefill hot path over one synthetic batch: block quantisation of
Q, K (with the calibrated per-channel multipliers where the workload smooths) and V
(transposed), then the fused FP4 attention kernel.  The headline workload is the largest
single-GPU prefill: non-causal MXFP4 with the scale bound Qmax = 7.25 (B=1, H=40, S=32768,
d=128, 1% of tokens x8).  Inputs are resident in HBM; L2 (126 MB) is flushed by a 256 MB
write before every timed step.  The metric is prefill TFLOP/s (4*B*Hq*S^2*d, halved for
causal).  The two other prefill workloads (causal GQA MXFP4 + Smooth-QK at S=4096, causal
GQA NVFP4 at S=16384) are timed the same way and reported under "prefill_workloads".  The
decode path (batch 32, 32/8 heads, 32768 keys, NVFP4 pages + 5% BF16 vertical lines +
128-token BF16 window) is timed in the same run and reported under "decode" (us/step,
GB/s), and the FP4 tensor-core decode (dual-residual query) on the same shape under
"decode_fp4q".

N > 1 (torchrun): every rank runs its own independent batch (weak scaling, no collective on
the data path); the step time is the max over ranks.  `--impl reference` times the CPU oracle
on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "FP4 attention prefill TFLOPS & 32K decode µs/step; % of FP4 tensor / HBM roofline"
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture
# of each roofline kernel (summaries and commands in profiles/).  A figure is reported only
# while the kernel's sources hash to the ones it was taken on; any change makes it null.
# Each capture ran a smaller batch of the same kernel (fewer heads, fewer sequences), so
# that it stays small; the traffic is stored per unit (query head, sequence) and scaled to
# the timed batch, the operand reads growing in proportion to the units.
NCU_TRAFFIC = {
    # profiles/attn_fwd_noncausal_mxfp4_uos_s32768.md: 107,980,544 + 89,369,088 B for 16 of the
    # 40 heads (the output write-back that stays in L2 at the end of the launch is not in it)
    "attn_fwd": {"sources": ("attn_fwd.cu", "fa4q_common.cuh"), "workload": "noncausal_mxfp4_uos_h40_s32768",
                 "sha256": "de54c21559c148c16d65baacc7df36b6f7fab41261fa03952cb237cee838653d",
                 "bytes_per_unit": (107980544 + 89369088) / 16},
    # profiles/decode_split_paged_nvfp4_b8_l32k.md: 358,902,272 + 8,193,536 B for 8 sequences
    "decode": {"sources": ("decode.cu", "fa4q_common.cuh"), "workload": None,
               "sha256": "ba940cd89265356d949f7a42e68a6b04591dda9da095edeabffefb29fc940c4f",
               "bytes_per_unit": (358902272 + 8193536) / 8},
    # profiles/decode_fp4q_paged_nvfp4_b8_l32k.md: 302,323,968 + 4,372,992 B for 8 sequences
    "decode_fp4q": {"sources": ("decode_tc.cu", "fa4q_common.cuh"), "workload": None,
                    "sha256": "67d20327f671a0249d5eeebd7395234a3a23deb9e11d7f9fc995909bfe115a1d",
                    "bytes_per_unit": (302323968 + 4372992) / 8},
}


def max_over_ranks(values, dev=None):
    """Element-wise maximum of per-rank timings over all ranks (the list itself with one rank).
    NCCL reduces device tensors, gloo host tensors; every rank must call it in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    on_dev = dist.get_backend() == "nccl"
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=dev if on_dev else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def world_size() -> int:
    import torch.distributed as dist
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


def job_rate(units_per_rank: float, ms: float, world: int) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time, per second."""
    return world * units_per_rank / (ms * 1e-3)


def sources_sha256(names) -> str:
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "microscaled_fp4_flashattention_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kernel: str, units: int, workload: str | None = None):
    """DRAM bytes of one launch over `units` heads or sequences, or None when the kernel
    changed since the capture or the capture was of another workload."""
    e = NCU_TRAFFIC[kernel]
    if e["sha256"] is None or sources_sha256(e["sources"]) != e["sha256"]:
        return None
    if e["workload"] is not None and workload != e["workload"]:
        return None
    return int(round(e["bytes_per_unit"] * units))


# ------------------------------------------------------------------------------ helpers
def load_sm_max_mhz() -> float:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p)).get("sm_max_mhz", 1965.0))
    return 1965.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


# ------------------------------------------------------------------------------ prefill workload
class PrefillRun:
    """Device-resident inputs and outputs of one prefill batch, and the step itself."""

    def __init__(self, w, dev, fa4q, seed_offset: int = 0):
        import torch
        self.w, self.dev, self.fa4q = w, dev, fa4q
        q, k, v = synth.prefill_inputs(w) if seed_offset == 0 else self._shifted(w, seed_offset)
        self.host = (q, k, v)
        self.flops = w.flops
        self.q = torch.from_numpy(q).to(dev).to(torch.bfloat16)
        self.k = torch.from_numpy(k).to(dev).to(torch.bfloat16)
        self.v = torch.from_numpy(v).to(dev).to(torch.bfloat16)
        self.mq = self.mk = None
        if w.smooth:
            qc, kc = synth.calibration_inputs(w)
            self.mq, self.mk = fa4q.smooth_calibrate(torch.from_numpy(qc).to(dev).to(torch.bfloat16),
                                                     torch.from_numpy(kc).to(dev).to(torch.bfloat16))
        self.out = torch.empty((w.B, w.Hq, w.S, w.d), dtype=torch.bfloat16, device=dev)
        self.qkv = fa4q.quantize_qkv(self.q, self.k, self.v, w.fmt, w.qmax, mul_q=self.mq, mul_k=self.mk)
        self.launches_per_step = 2

    @staticmethod
    def _shifted(w, off):
        import dataclasses
        ww = dataclasses.replace(w, wid=w.wid + 100 * off)
        return synth.prefill_inputs(ww)

    def step(self, attn_events=None, q=None, k=None, v=None):
        fa4q, w = self.fa4q, self.w
        q = self.q if q is None else q
        k = self.k if k is None else k
        v = self.v if v is None else v
        # quantise Q, K (with the smoothing multipliers) and V in one launch, then attention
        pq, sq, pk, sk, pv, sv = fa4q.quantize_qkv(q, k, v, w.fmt, w.qmax, mul_q=self.mq, mul_k=self.mk,
                                                   out=self.qkv)
        if attn_events is not None:
            attn_events[0].record()
        fa4q.attn_fwd(pq, sq, pk, sk, pv, sv, B=w.B, Hq=w.Hq, Hkv=w.Hkv, S_q=w.S, S_k=w.S, d=w.d,
                      fmt=w.fmt, causal=w.causal, qmax_p=w.qmax_p, out=self.out)
        if attn_events is not None:
            attn_events[1].record()
        return self.out


def hybrid_bench(run, w, dev, fa4q, flush, barrier, steps):
    """Time fa4q_attn_fwd_hybrid (one kernel: BF16 window / vertical-line tiles, then the FP4
    tiles, one online softmax) on the prefill batch; FLOPs counted as the causal total."""
    import torch
    if not w.causal or w.d != 128:
        return None
    B, Hq, Hkv, S, d = w.B, w.Hq, w.Hkv, w.S, w.d
    n_vl, W = int(0.05 * S), 128
    rng = synth.generator(w.wid, 5, 7)
    pos = np.stack([np.stack([np.sort(rng.choice(S, n_vl, replace=False)) for _ in range(Hkv)])
                    for _ in range(B)]).astype(np.int32)
    t_pos = torch.from_numpy(pos).to(dev)
    t_cnt = torch.full((B, Hkv), n_vl, dtype=torch.int32, device=dev)
    idx = t_pos.long()[..., None].expand(-1, -1, -1, d)
    vk = torch.gather(run.k, 2, idx).contiguous()
    vv = torch.gather(run.v, 2, idx).contiguous()
    ex = np.zeros((B, Hkv, (S + 63) // 64), np.uint64)
    for b in range(B):
        for h in range(Hkv):
            np.bitwise_or.at(ex[b, h], pos[b, h] // 64, np.uint64(1) << (pos[b, h] % 64).astype(np.uint64))
    t_ex = torch.from_numpy(ex.view(np.int64)).to(dev)
    kz, vz = run.k.clone(), run.v.clone()
    kz.scatter_(2, idx, 0.0)
    vz.scatter_(2, idx, 0.0)
    pq, sq, pk, sk, pv, sv = fa4q.quantize_qkv(run.q, kz, vz, w.fmt, w.qmax, mul_q=run.mq, mul_k=run.mk)
    out = torch.empty_like(run.out)
    call = lambda: fa4q.attn_fwd_hybrid(pq, sq, pk, sk, pv, sv, run.q, run.k, run.v, t_pos, t_cnt, vk, vv, t_ex,
                                        B=B, Hq=Hq, Hkv=Hkv, S=S, d=d, window=W, fmt=w.fmt, qmax_p=w.qmax_p,
                                        out=out)
    for _ in range(3):
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        ev[i][0].record()
        call()
        ev[i][1].record()
    barrier()
    ms, = max_over_ranks([float(np.mean([a.elapsed_time(b) for a, b in ev]))], dev)
    return {"kernels": "attn_fwd_kernel<HYB> (tcgen05: BF16 kind::f16 tiles, then FP4 block-scaled tiles)",
            "ms": ms, "TFLOP/s": run.flops / (ms * 1e-3) / 1e12, "window": W, "vertical_lines_per_kv_head": n_vl,
            "note": "FLOPs of the whole causal attention (both parts); seeded random vertical-line positions"}


# ------------------------------------------------------------------------------ decode workload
class DecodeRun:
    def __init__(self, dw, dev, fa4q):
        import torch
        self.dw, self.dev, self.fa4q = dw, dev, fa4q
        B, Hq, Hkv, d, L, W = dw.B, dw.Hq, dw.Hkv, dw.d, dw.L, dw.window
        n_fp4, P, n_hp = dw.fp4_len, dw.n_pages, dw.n_hp
        tK = torch.empty((B, Hkv, L, d), dtype=torch.bfloat16, device=dev)
        tV = torch.empty((B, Hkv, L, d), dtype=torch.bfloat16, device=dev)
        for b in range(B):
            for h in range(Hkv):
                tK[b, h] = torch.from_numpy(synth.decode_kv_slice(dw, "k", b, h)).to(dev).to(torch.bfloat16)
                tV[b, h] = torch.from_numpy(synth.decode_kv_slice(dw, "v", b, h)).to(dev).to(torch.bfloat16)
        Q = np.stack([synth.decode_query(dw, b) for b in range(B)])
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).to(dev)
        self.table = i32(synth.decode_block_table(dw))
        self.fp4_len = i32(np.full(B, n_fp4))
        # vertical-line tokens: top 5% of the non-window prefix by column mass from 64
        # observation queries per q-head (GPU identification), then the FP4 pages without them
        self.q_obs = torch.from_numpy(np.stack([synth.decode_observation_queries(dw, b) for b in range(B)])
                                      ).to(dev).to(torch.bfloat16)
        self.tK, self.tV = tK, tV
        sel = fa4q.select_vertical_lines(self.q_obs, tK, tV, self.fp4_len, rho=dw.hp_frac)
        assert int(sel["counts"].min()) == int(sel["counts"].max()) == n_hp
        self.excl = sel["excl"][:, :, :P].contiguous()
        self.kp, self.ks, self.vp, self.vs = fa4q.quantize_kv_pages(tK, tV, self.fp4_len, self.excl,
                                                                    self.table, B * P)
        self.hpk, self.hpv, self.hpc = sel["hp_k"], sel["hp_v"], sel["counts"]
        self.wk, self.wv = tK[:, :, n_fp4:].contiguous(), tV[:, :, n_fp4:].contiguous()
        self.wl = i32(np.full(B, W))
        self.q = torch.from_numpy(Q).to(dev).to(torch.bfloat16)
        self.out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(fa4q.decode_workspace_size(B, Hq, Hkv, d, P), dtype=torch.uint8, device=dev)
        blk = 16
        self.bytes = (2 * B * Hkv * P * 64 * (d // 2 + d // blk)          # FP4 K and V^T pages + scales
                      + 2 * B * Hkv * n_hp * d * 2 + 2 * B * Hkv * W * d * 2  # BF16 set and window
                      + B * Hkv * P * 8 + B * P * 4                      # exclusion masks, block table
                      + 2 * B * Hq * d * 2 + B * 4 * 2 + B * Hkv * 4)     # q, out, lengths, counts

    def step(self):
        fa4q = self.fa4q
        return fa4q.decode(self.q, self.kp, self.ks, self.vp, self.vs, self.table, self.fp4_len, self.excl,
                           self.hpk, self.hpv, self.hpc, self.wk, self.wv, self.wl, out=self.out,
                           workspace=self.ws)


def decode_bench(args, dev, fa4q, line, hbm_gbs, peak_kind, barrier):
    """Time the decode over the paged hybrid cache; adds line["decode"]."""
    import torch
    dw = synth.WORKLOADS[4]
    if args.decode_batch:
        import dataclasses
        dw = dataclasses.replace(dw, B=args.decode_batch)
    drun = DecodeRun(dw, dev, fa4q)
    for _ in range(max(3, args.warmup)):
        drun.step()
    barrier()
    dsteps = max(20, args.steps)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dsampler = ClockSampler(dev.index)
    with dsampler:
        t_end = time.time() + 1.0
        while time.time() < t_end:
            for _ in range(20):
                drun.step()
            torch.cuda.synchronize()
        d0.record()
        for _ in range(dsteps):
            drun.step()
        d1.record()
        barrier()
    d_ms, = max_over_ranks([d0.elapsed_time(d1) / dsteps], dev)
    world = world_size()
    gbs = job_rate(drun.bytes, d_ms, world) / 1e9
    # vertical-line identification (column mass + selection + mask + row gather); the method
    # refreshes it every 64 decoded tokens, so it is reported beside the step, not in it
    ws = torch.empty(fa4q.vlines_workspace_size(dw.B, dw.Hq, dw.Hkv, drun.q_obs.shape[2], dw.L),
                     dtype=torch.uint8, device=dev)
    ident = lambda: fa4q.select_vertical_lines(drun.q_obs, drun.tK, drun.tV, drun.fp4_len, rho=dw.hp_frac,
                                                workspace=ws)
    for _ in range(2):
        ident()
    i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    i0.record()
    for _ in range(5):
        ident()
    i1.record()
    torch.cuda.synchronize()
    id_ms, = max_over_ranks([i0.elapsed_time(i1) / 5], dev)
    line["decode"] = {"workload": dw.name, "us_per_step": d_ms * 1e3, "higher_is_better": False,
                      "GBps": gbs, "bytes_per_step": drun.bytes, "gpu_launches": 2 * dsteps,
                      "roofline": {"kernel": "decode_split_kernel+decode_combine_kernel", "bound": "hbm",
                                   "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                                   "traffic": ncu_traffic("decode", dw.B), "peak_source": f"{peak_kind} hbm copy"},
                      "identify": {"ms": id_ms, "every_tokens": 64, "us_per_step_amortized": id_ms * 1e3 / 64,
                                   "share_of_decode_step": (id_ms / 64) / (d_ms + id_ms / 64),
                                   "what": "column mass of 64 observation queries x 4 q-heads over the 32640-token "
                                           "prefix, top-5% selection, exclusion mask, BF16 row gather (all 32 x 8 groups)"},
                      "l2": "working set 1.4 GB > L2", "clocks": dsampler.summary()}


def decode_fp4q_bench(args, dev, fa4q, line, hbm_gbs, peak_kind, barrier):
    """Time the FP4 tensor-core decode (dual-residual query, all-FP4 paged cache) on the
    decode workload's shape; adds line["decode_fp4q"]."""
    import torch
    dw = synth.WORKLOADS[4]
    if args.decode_batch:
        import dataclasses
        dw = dataclasses.replace(dw, B=args.decode_batch)
    B, Hq, Hkv, d, L = dw.B, dw.Hq, dw.Hkv, dw.d, dw.L
    P = (L + 63) // 64
    gen = torch.Generator(device=dev)
    gen.manual_seed(4242)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).to(dev)
    table = i32(np.random.default_rng(4242).permutation(B * P).reshape(B, P))
    lens = i32(np.full(B, L))
    # quantise the cache one sequence at a time (a BF16 copy of the whole cache is 4 GB)
    kp = torch.empty((B * P, Hkv, 64, d // 2), dtype=torch.uint8, device=dev)
    vp = torch.empty((B * P, Hkv, d, 32), dtype=torch.uint8, device=dev)
    ks = vs = None
    for b in range(B):
        k = (torch.randn((1, Hkv, L, d), generator=gen, device=dev) * 1.5).to(torch.bfloat16)
        v = torch.randn((1, Hkv, L, d), generator=gen, device=dev).to(torch.bfloat16)
        tb = torch.arange(P, dtype=torch.int32, device=dev).view(1, P)
        kpb, ksb, vpb, vsb = fa4q.quantize_kv_pages(k, v, lens[b:b + 1], None, tb, P)
        if ks is None:
            ks = torch.empty((B * P,) + tuple(ksb.shape[1:]), dtype=ksb.dtype, device=dev)
            vs = torch.empty((B * P,) + tuple(vsb.shape[1:]), dtype=vsb.dtype, device=dev)
        rows = table[b].long()
        kp[rows], vp[rows], ks[rows], vs[rows] = kpb, vpb, ksb, vsb
        del k, v
    q = (torch.randn((B, Hq, d), generator=gen, device=dev) * 1.5).to(torch.bfloat16)
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    tps = args.fp4q_tiles_per_split
    splits = -(-((P + 1) // 2) // tps)
    ws = torch.empty(int(fa4q.lib().fa4q_decode_fp4q_workspace_size(B, Hq, Hkv, d, P, tps)),
                     dtype=torch.uint8, device=dev)
    step = lambda: fa4q.decode_fp4q(q, kp, ks, vp, vs, table, lens, B * P, out=out, workspace=ws,
                                    tiles_per_split=tps)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert fa4q.device_status()[0] == 0
    nbytes = (2 * B * Hkv * P * 64 * (d // 2 + d // 16)   # FP4 K and V^T pages + UE4M3 scales
              + B * P * 4 + B * 4 + 2 * B * Hq * d * 2)   # block table, lengths, q, out
    dsteps = max(20, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    with sampler:
        t_end = time.time() + 1.0
        while time.time() < t_end:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        e0.record()
        for _ in range(dsteps):
            step()
        e1.record()
        barrier()
    ms, = max_over_ranks([e0.elapsed_time(e1) / dsteps], dev)
    gbs = job_rate(nbytes, ms, world_size()) / 1e9
    line["decode_fp4q"] = {
        "workload": f"{dw.name} shape, all {L} keys FP4 (NVFP4 pages)", "us_per_step": ms * 1e3,
        "higher_is_better": False, "GBps": gbs, "bytes_per_step": nbytes, "gpu_launches": 3 * dsteps,
        "splits": splits, "tiles_per_split": tps,
        "roofline": {"kernel": "decode_tc_kernel+dec_query_kernel+decode_combine_kernel", "bound": "hbm",
                     "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                     "traffic": ncu_traffic("decode_fp4q", dw.B),
                     "peak_source": f"{peak_kind} hbm copy"},
        "note": "dual-residual NVFP4 query and PNQ probabilities on the block-scaled tensor cores "
                "(BitDecoding-FP4); seeded gaussian cache, not the hybrid cache of line['decode']",
        "l2": "working set 1.2 GB > L2", "clocks": sampler.summary()}
    del kp, vp, ks, vs, ws


# ------------------------------------------------------------------------------ CPU oracle timing
def oracle_prefill_sample(w, budget_s: float, host=None, gpu_out=None, accuracy=None):
    """Time the oracle on sampled (head, row) work of workload w for about budget_s seconds;
    returns (TFLOP/s, description, seconds).

    With gpu_out (the GPU's output [B, Hq, S, d] for the same inputs, batch 0 used) and a dict
    `accuracy`, the sampled rows also give the accuracy report (untimed): GPU vs oracle, and
    GPU and oracle each vs unquantised FP64 softmax attention on the bf16 inputs (sums of
    absolute differences over sums of absolute reference values, and maxima)."""
    from oracle import attention as OA
    from oracle import smooth as OS
    q, k, v = host if host is not None else synth.prefill_inputs(w)
    lam = OS.calibrate(*synth.calibration_inputs(w)) if w.smooth else None
    rng = np.random.default_rng(0)
    done_flops, t_used, n_rows, heads_used = 0.0, 0.0, 0, 0
    sums = np.zeros(5)    # sums of |g-o|, |o|, |g-u|, |o-u|, |u| over the reported rows
    maxs = np.zeros(3)    # max |g-o|, |g-u|, |o-u|
    acc_rows = 0
    R = 64
    while t_used < budget_s and heads_used < w.Hq:
        h = int(rng.integers(w.Hq))
        rows = np.sort(rng.choice(w.S, R, replace=False))
        t0 = time.perf_counter()
        res = OA.prefill(q, k, v, causal=w.causal, fmt=w.fmt, qmax=w.qmax, qmax_p=w.qmax_p, lam=lam, rows=rows,
                         heads=[(0, h)])
        dt = time.perf_counter() - t0
        if gpu_out is not None and accuracy is not None and heads_used < 6:   # bounded extra host time
            sel = slice(0, 256)                  # at most 256 rows per head (bounded host memory)
            o = np.asarray(res[(0, h)], dtype=np.float64)[sel]
            hk = h // (w.Hq // w.Hkv)
            u = OA.attention_plain(q[0, h], k[0, hk], v[0, hk], causal=w.causal, rows=rows[sel])
            g = np.asarray(gpu_out[0, h][rows[sel]], dtype=np.float64)
            ob = synth.round_to_bf16(o.astype(np.float32)).astype(np.float64)   # the GPU output is bf16
            sums += [np.abs(g - ob).sum(), np.abs(ob).sum(), np.abs(g - u).sum(), np.abs(o - u).sum(),
                     np.abs(u).sum()]
            acc_rows += len(rows[sel])
            maxs = np.maximum(maxs, [np.abs(g - ob).max(), np.abs(g - u).max(), np.abs(o - u).max()])
        keys = (rows + 1) if w.causal else np.full(R, w.S)
        done_flops += float(4.0 * w.d * keys.sum())
        t_used += dt
        n_rows += R
        heads_used += 1
        if dt < budget_s / 8:
            R = min(w.S, R * 2)
    desc = f"{n_rows} query rows over {heads_used} heads of {w.name} (all keys per row, oracle as is)"
    if gpu_out is not None and accuracy is not None and sums[1] > 0:
        accuracy.update({
            "rows": acc_rows, "what": "query rows of the first sampled heads of the cpu_baseline sample; "
                                      "mean_rel = sum|x - ref| / sum|ref|; the bf16 GPU output is compared "
                                      "with the oracle rounded to bf16",
            "gpu_vs_oracle": {"max_abs": float(maxs[0]), "mean_rel": float(sums[0] / sums[1])},
            "gpu_vs_unquantized": {"max_abs": float(maxs[1]), "mean_rel": float(sums[2] / sums[4])},
            "oracle_vs_unquantized": {"max_abs": float(maxs[2]), "mean_rel": float(sums[3] / sums[4])}})
    return done_flops / t_used / 1e12, desc, t_used


# ------------------------------------------------------------------------------ prefill timing
def time_prefill(run, flush, steps, barrier, gpu_index, soak_s, dev):
    """Time `steps` prefill steps (L2 flushed by an untimed write before each) and, inside
    each, the attention kernel alone (CUDA events on the launching stream).  Clocks are
    sampled during a soak of back-to-back steps and the timed loop.  Returns (mean step ms,
    mean attention ms, clock summary), the times as the max over ranks."""
    import torch
    for _ in range(3):
        run.step()
    barrier()
    sampler = ClockSampler(gpu_index)
    with sampler:
        t_end = time.time() + soak_s
        while time.time() < t_end:
            for _ in range(20):
                run.step()
            torch.cuda.synchronize()
        barrier()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        aev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(float(i))                      # evict L2 (untimed)
            ev[i][0].record()
            run.step(attn_events=aev[i])
            ev[i][1].record()
        barrier()
    t_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    a_ms = float(np.mean([a.elapsed_time(b) for a, b in aev]))
    t_ms, a_ms = max_over_ranks([t_ms, a_ms], dev)
    return t_ms, a_ms, sampler.summary()


def attn_roofline(w, flops, a_ms, fp4_peak, peak_src, world):
    """Roofline record of the attention kernel: algorithmic FLOPs per launch over its mean
    launch time, against the FP4 dense peak; `traffic` from the ncu capture of this
    workload when the kernel is unchanged since, else null."""
    achieved = flops / (a_ms * 1e-3) / 1e12
    sm_mhz = load_sm_max_mhz()
    # exponential ceiling: every score needs one 2^x; six of every eight run on MUFU at
    # 16 per clock per SM (the FMA pipe takes the other two), 4*d FLOPs per score
    exp_peak = 16.0 / (6.0 / 8.0) * 4 * w.d * 148 * sm_mhz * 1e6 / 1e12
    return {"kernel": "attn_fwd_kernel", "bound": "tensor", "achieved": achieved, "peak": fp4_peak,
            "unit": "TFLOP/s", "frac": achieved / fp4_peak,
            "traffic": ncu_traffic("attn_fwd", w.B * w.Hq, workload=w.name),
            "traffic_note": "dram read + write per launch, scaled by heads from a 16-head ncu capture of the "
                            "same kernel; the part of the bf16 output (B*Hq*S*d*2 B) still in L2 when the "
                            "launch ends is written back later and falls outside the figure",
            "peak_source": peak_src, "ms_per_launch": a_ms, "launches_per_step": 1,
            "exp_ceiling": {"peak": exp_peak, "unit": "TFLOP/s", "frac": achieved / exp_peak,
                            "what": "MUFU ex2 at 16/clk/SM for 6 of 8 exponentials, 148 SMs at "
                                    f"{sm_mhz:.0f} MHz, 4*d FLOPs per score"}}


# ------------------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=5, choices=[2, 3, 5])
    ap.add_argument("--no-sub", action="store_true", help="skip the other prefill workloads")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true", help="time only the decode path")
    ap.add_argument("--decode-fp4q-only", action="store_true",
                    help="time only the FP4 tensor-core decode (dual-residual query)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="decode batch (0 = the workload's 32); smaller batches are for profiling")
    ap.add_argument("--fp4q-tiles-per-split", type=int, default=32,
                    help="range length of the FP4 tensor-core decode (part of its result)")
    ap.add_argument("--prefill-heads", type=int, default=0,
                    help="query heads of the prefill batch (0 = the workload's; the group ratio is kept); "
                         "fewer heads are for profiling and never the headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--soak-s", type=float, default=2.0)
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = synth.WORKLOADS[args.workload]
    if args.prefill_heads > 0 and args.prefill_heads != w.Hq:
        import dataclasses
        g = w.Hq // w.Hkv
        if args.prefill_heads % g:
            ap.error(f"--prefill-heads must be a multiple of the group size {g}")
        w = dataclasses.replace(w, name=f"{w.name}_heads{args.prefill_heads}", Hq=args.prefill_heads,
                                Hkv=args.prefill_heads // g)

    if args.impl == "reference":
        if rank != 0:
            return
        steps, warm = max(1, args.steps), max(0, args.warmup)
        per_step = 2.5
        for _ in range(warm):
            oracle_prefill_sample(w, per_step / 4)
        tf, desc, secs = [], None, 0.0
        for _ in range(steps):
            v, desc, s = oracle_prefill_sample(w, per_step)
            tf.append(v)
            secs += s
        value = statistics.mean(tf)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": steps, "warmup": warm, "ms_per_step": 1e3 * secs / steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": w.fmt, "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "d": w.d,
                           "causal": w.causal, "fmt": w.fmt},
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_kind = load_peaks()

    if args.decode_only or args.decode_fp4q_only:
        line = {"metric": METRIC, "n_gpus": world}
        bench_fn = decode_fp4q_bench if args.decode_fp4q_only else decode_bench
        bench_fn(args, dev, fa4q, line, hbm_gbs, peak_kind, barrier=lambda: torch.cuda.synchronize())
        print(json.dumps(line))
        return
    run = PrefillRun(w, dev, fa4q, seed_offset=rank)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(3, args.warmup)):
        run.step()
    barrier()
    gpu_index = dev.index if world == 1 else local_rank
    t_ms, a_ms, clocks = time_prefill(run, flush, args.steps, barrier, gpu_index, args.soak_s, dev)
    value = job_rate(run.flops, t_ms, world) / 1e12

    # ablation beside the headline: conditional rescaling (reference maximum kept within 8
    # binades, fa4q_attn_fwd_ex; MXFP4 only), the attention kernel alone on the same operands
    tau_ms = None
    if w.fmt == "mxfp4":
        pq, sq, pk, sk, pv, sv = run.qkv
        tau_run = lambda: fa4q.attn_fwd(pq, sq, pk, sk, pv, sv, B=w.B, Hq=w.Hq, Hkv=w.Hkv, S_q=w.S, S_k=w.S,
                                        d=w.d, fmt=w.fmt, causal=w.causal, qmax_p=w.qmax_p, out=run.out,
                                        rescale_tau=8)
        for _ in range(3):
            tau_run()
        tev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(float(i))
            tev[i][0].record()
            tau_run()
            tev[i][1].record()
        barrier()
        tau_ms, = max_over_ranks([float(np.mean([a.elapsed_time(b) for a, b in tev]))], dev)

    # end to end through the public API: pinned host inputs -> device, quantise, attend, output -> host
    q_h = torch.from_numpy(run.host[0]).to(torch.bfloat16).pin_memory()
    k_h = torch.from_numpy(run.host[1]).to(torch.bfloat16).pin_memory()
    v_h = torch.from_numpy(run.host[2]).to(torch.bfloat16).pin_memory()
    o_h = torch.empty(run.out.shape, dtype=torch.bfloat16).pin_memory()
    qd, kd, vd = torch.empty_like(run.q), torch.empty_like(run.k), torch.empty_like(run.v)

    def e2e_step():
        qd.copy_(q_h, non_blocking=True)
        kd.copy_(k_h, non_blocking=True)
        vd.copy_(v_h, non_blocking=True)
        out = run.step(q=qd, k=kd, v=vd)
        o_h.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(5, args.steps // 2)
    e0.record()
    for _ in range(e_steps):
        e2e_step()
    e1.record()
    barrier()
    e_ms, = max_over_ranks([e0.elapsed_time(e1) / e_steps], dev)
    h2d = (q_h.numel() + k_h.numel() + v_h.numel()) * 2
    d2h = o_h.numel() * 2
    del q_h, k_h, v_h, o_h, qd, kd, vd

    fp4_peak = bf16_tf * FP4_PER_BF16
    peak_src = f"{peak_kind} bf16 burst {bf16_tf:.1f} TFLOP/s x {FP4_PER_BF16:g} (nominal FP4/BF16)"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": t_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.fmt, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "d": w.d, "causal": w.causal,
                   "fmt": w.fmt, "smooth": w.smooth, "qmax": w.qmax, "qmax_p": w.qmax_p,
                   "parallelism": f"replicas x{world}",
                   "step": "quantize Q,K,V + fused FP4 attention",
                   "l2": "flushed before each timed step (256 MB write, untimed)"},
        "gpu_launches": run.launches_per_step * args.steps,
        "e2e": {"value": job_rate(run.flops, e_ms, world) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e_ms},
        "roofline": attn_roofline(w, run.flops, a_ms, fp4_peak, peak_src, world),
        "clocks": clocks,
    }
    # ablation beside the headline: Hadamard-rotated Q and K (fa4q_quantize_rotated, the
    # alternative to Smooth-QK) against the plain inner quantisation of the same tensors
    def time_q(fn, reps=10):
        for _ in range(2):
            fn()
        e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps):
            flush.fill_(float(i))
            e[i][0].record()
            fn()
            e[i][1].record()
        barrier()
        return max_over_ranks([float(np.mean([a.elapsed_time(b) for a, b in e]))], dev)[0]
    rot_ms = time_q(lambda: (fa4q.quantize_rotated(run.q, w.fmt, w.qmax), fa4q.quantize_rotated(run.k, w.fmt, w.qmax)))
    inn_ms = time_q(lambda: (fa4q.quantize(run.q, w.fmt, fa4q.FA4Q_AXIS_INNER, w.qmax),
                             fa4q.quantize(run.k, w.fmt, fa4q.FA4Q_AXIS_INNER, w.qmax)))
    qk_elems = run.q.numel() + run.k.numel()
    qk_bytes = qk_elems * 2 + qk_elems // 2 + qk_elems // (32 if w.fmt == "mxfp4" else 16)
    line["ablation_hadamard"] = {
        "kernel": "quant_rotated_kernel (Q and K, two launches)", "ms": rot_ms,
        "GBps": qk_bytes / (rot_ms * 1e-3) / 1e9, "plain_inner_ms": inn_ms,
        "plain_inner_GBps": qk_bytes / (inn_ms * 1e-3) / 1e9,
        "note": "Walsh-Hadamard rotation of every Q/K row fused into the quantiser; not on the headline path"}
    if tau_ms is not None:
        line["ablation_rescale_tau8"] = {
            "kernel": "attn_fwd_kernel via fa4q_attn_fwd_ex(rescale_tau=8)", "ms_per_launch": tau_ms,
            "TFLOP/s": run.flops / (tau_ms * 1e-3) / 1e12,
            "frac_of_fp4_peak": run.flops / (tau_ms * 1e-3) / 1e12 / fp4_peak,
            "note": "P quantised against a reference maximum kept within 8 binades "
                    "(FlashAttention-4 conditional rescaling); not the headline reading"}

    # the GPU's output of this batch, for the accuracy report beside the CPU baseline
    gpu_out = (run.out.float().cpu().numpy() if rank == 0 and world == 1 and not args.no_cpu_baseline
               else None)
    # the other prefill workloads, each timed as the headline (its own clocks); the hybrid
    # prefill (HyQuant) runs beside the causal MXFP4 one, on the same inputs
    if not args.no_sub:
        del run
        torch.cuda.empty_cache()
        subs = {}
        for wid in (5, 2, 3):
            if wid == args.workload:
                continue
            ws_ = synth.WORKLOADS[wid]
            r2 = PrefillRun(ws_, dev, fa4q, seed_offset=rank)
            ts, as_, cl = time_prefill(r2, flush, args.steps, barrier, gpu_index, min(1.0, args.soak_s), dev)
            subs[ws_.name] = {
                "ms_per_step": ts, "TFLOP/s": job_rate(r2.flops, ts, world) / 1e12,
                "config": {"B": ws_.B, "Hq": ws_.Hq, "Hkv": ws_.Hkv, "S": ws_.S, "d": ws_.d, "causal": ws_.causal,
                           "fmt": ws_.fmt, "smooth": ws_.smooth, "qmax": ws_.qmax, "qmax_p": ws_.qmax_p},
                "gpu_launches": r2.launches_per_step * args.steps,
                "roofline": attn_roofline(ws_, r2.flops, as_, fp4_peak, peak_src, world), "clocks": cl}
            if ws_.causal and ws_.fmt == "mxfp4":
                hy = hybrid_bench(r2, ws_, dev, fa4q, flush, barrier, args.steps)
                # against the plain attention kernel on the same inputs (same FLOP count)
                hy["vs_plain_attention"] = as_ / hy["ms"]
                line["hybrid_prefill"] = dict(workload=ws_.name, **hy)
            del r2
            torch.cuda.empty_cache()
        line["prefill_workloads"] = subs
    if not args.no_decode:
        if args.no_sub:
            del run
        del flush
        torch.cuda.empty_cache()
        decode_bench(args, dev, fa4q, line, hbm_gbs, peak_kind, barrier)
        torch.cuda.empty_cache()
        decode_fp4q_bench(args, dev, fa4q, line, hbm_gbs, peak_kind, barrier)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        acc = {}
        v, desc, _ = oracle_prefill_sample(w, 12.0, gpu_out=gpu_out, accuracy=acc)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                "sample": desc}
        if acc:
            line["accuracy"] = acc
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

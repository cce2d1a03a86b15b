"""fa4q_decode_fp4q (BitDecoding-FP4: dual-residual FP4 query and FP4 probabilities on the
tensor cores, all-FP4 paged cache) against the oracle, element by element: the bf16 output
against the FP64 oracle rounded to bf16, max-abs <= 2e-2, mean-rel <= 2e-3.  The range
length tiles_per_split is part of the definition and is passed to both sides."""
import numpy as np
import pytest

import synth
from oracle import bitdecode as BD
from fa4q_testlib import assert_close, bf16_ref, to_dev_bf16

pytestmark = pytest.mark.gpu


def _run(B, Hq, Hkv, L, seed, tps=32, lens=None, shuffle=True):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    d = 128
    rng = np.random.default_rng(seed)
    k = synth.round_to_bf16(rng.normal(size=(B, Hkv, L, d)).astype(np.float32) * np.float32(1.5))
    v = synth.round_to_bf16(rng.normal(size=(B, Hkv, L, d)).astype(np.float32))
    q = synth.round_to_bf16(rng.normal(size=(B, Hq, d)).astype(np.float32) * np.float32(1.5))
    P = (L + 63) // 64
    n_phys = B * P
    table = (rng.permutation(n_phys) if shuffle else np.arange(n_phys)).reshape(B, P).astype(np.int32)
    lens = np.full(B, L, np.int32) if lens is None else np.asarray(lens, np.int32)
    t_len = torch.from_numpy(lens).to(dev)
    t_table = torch.from_numpy(table).to(dev)
    kp, ks, vp, vs = fa4q.quantize_kv_pages(to_dev_bf16(k, dev), to_dev_bf16(v, dev), t_len, None, t_table, n_phys)
    out = fa4q.decode_fp4q(to_dev_bf16(q, dev), kp, ks, vp, vs, t_table, t_len, n_phys, tiles_per_split=tps)
    torch.cuda.synchronize()
    assert fa4q.device_status()[0] == 0
    got = out.float().cpu().numpy()
    G = Hq // Hkv
    gs, rs = [], []
    for b in range(B):
        for h in range(Hkv):
            n = int(lens[b])
            rs.append(BD.decode_group_fp4q(q[b, h * G:(h + 1) * G], k[b, h, :n], v[b, h, :n], tps))
            gs.append(got[b, h * G:(h + 1) * G])
    return np.stack(gs), np.stack(rs)


@pytest.mark.parametrize("B,Hq,Hkv,L,tps", [
    (2, 8, 2, 700, 32),      # odd page count: the last page pair holds one page
    (2, 8, 2, 1024, 3),
    (1, 4, 1, 4160, 32),     # 33 tiles: a second range of one tile
    (1, 8, 1, 300, 1),       # G = 8; one tile per range
    (1, 16, 1, 520, 2),      # G = 16: every column of the 16-head MMA tile
    (2, 6, 2, 1100, 2),      # G = 3: padded heads inside the 4-head instantiation
    (1, 2, 2, 130, 32),      # MHA; a last tile with 2 keys
    (1, 4, 1, 9000, 64),     # a range longer than the block-table window of 16 tiles
])
def test_decode_fp4q(B, Hq, Hkv, L, tps):
    got, ref = _run(B, Hq, Hkv, L, L + Hq, tps)
    assert_close(got, bf16_ref(ref), what=f"decode_fp4q L={L} T={tps}")


def test_decode_fp4q_ragged_lengths_and_empty_splits():
    """Sequences of different lengths in one batch: the short one's later ranges are empty."""
    got, ref = _run(3, 8, 2, 2000, 7, tps=4, lens=[2000, 700, 64])
    assert_close(got, bf16_ref(ref), what="ragged")


def test_decode_fp4q_result_does_not_depend_on_the_batch():
    """The same sequence decoded alone and as one of a batch of 32 (other sequences random,
    its pages elsewhere in the cache) gives bit-identical output: the range length is fixed
    by the call, never derived from the batch or head counts."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    Hq, Hkv, d, L = 8, 2, 128, 3000
    P = (L + 63) // 64
    rng = np.random.default_rng(3000)
    outs = []
    k1 = rng.normal(size=(Hkv, L, d)).astype(np.float32)
    v1 = rng.normal(size=(Hkv, L, d)).astype(np.float32)
    q1 = rng.normal(size=(Hq, d)).astype(np.float32)
    for B in (1, 32):
        k = rng.normal(size=(B, Hkv, L, d)).astype(np.float32)
        v = rng.normal(size=(B, Hkv, L, d)).astype(np.float32)
        q = rng.normal(size=(B, Hq, d)).astype(np.float32)
        k[B - 1], v[B - 1], q[B - 1] = k1, v1, q1
        table = rng.permutation(B * P).reshape(B, P).astype(np.int32)
        t_len = torch.full((B,), L, dtype=torch.int32, device=dev)
        t_table = torch.from_numpy(table).to(dev)
        kp, ks, vp, vs = fa4q.quantize_kv_pages(to_dev_bf16(k, dev), to_dev_bf16(v, dev), t_len, None, t_table, B * P)
        out = fa4q.decode_fp4q(to_dev_bf16(q, dev), kp, ks, vp, vs, t_table, t_len, B * P, tiles_per_split=8)
        outs.append(out[B - 1].float().cpu().numpy())
    assert fa4q.device_status()[0] == 0
    assert np.array_equal(outs[0], outs[1])


def test_decode_fp4q_full_size_sampled_groups():
    """Batch 32, 32/8 heads, 32768 keys (the decode workload's shape, every key FP4)."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dw = synth.WORKLOADS[4]
    dev = torch.device("cuda:0")
    B, Hq, Hkv, d, L = dw.B, dw.Hq, dw.Hkv, dw.d, dw.L
    P = (L + 63) // 64
    tK = torch.empty((B, Hkv, L, d), dtype=torch.bfloat16, device=dev)
    tV = torch.empty((B, Hkv, L, d), dtype=torch.bfloat16, device=dev)
    host = {}
    for b in range(B):
        for h in range(Hkv):
            kk, vv = synth.decode_kv_slice(dw, "k", b, h), synth.decode_kv_slice(dw, "v", b, h)
            tK[b, h] = torch.from_numpy(kk).to(dev).to(torch.bfloat16)
            tV[b, h] = torch.from_numpy(vv).to(dev).to(torch.bfloat16)
            if (b, h) in [(0, 0), (17, 3), (31, 7)]:
                host[(b, h)] = (kk, vv)
    Q = np.stack([synth.decode_query(dw, b) for b in range(B)])
    table = torch.from_numpy(synth.decode_block_table(dw, n_pages=P).astype(np.int32)).to(dev)
    t_len = torch.full((B,), L, dtype=torch.int32, device=dev)
    kp, ks, vp, vs = fa4q.quantize_kv_pages(tK, tV, t_len, None, table, B * P)
    tps = 32
    out = fa4q.decode_fp4q(to_dev_bf16(Q, dev), kp, ks, vp, vs, table, t_len, B * P,
                           tiles_per_split=tps).float().cpu().numpy()
    assert fa4q.device_status()[0] == 0
    G = Hq // Hkv
    gs, rs = [], []
    for (b, h), (kk, vv) in host.items():
        rs.append(BD.decode_group_fp4q(Q[b, h * G:(h + 1) * G], kk, vv, tps))
        gs.append(out[b, h * G:(h + 1) * G])
    assert_close(np.stack(gs), bf16_ref(np.stack(rs)), what="decode_fp4q full size")

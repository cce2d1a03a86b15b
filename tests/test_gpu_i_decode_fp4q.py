"""fa4q_decode_fp4q (BitDecoding-FP4: dual-residual FP4 query and FP4 probabilities on the
tensor cores, all-FP4 paged cache) against the oracle, element by element; max-abs <= 2e-2,
mean-rel <= 5e-3 (the output is bf16, as fa4q_decode's)."""
import numpy as np
import pytest

import synth
from oracle import bitdecode as BD
from fa4q_testlib import assert_close, to_dev_bf16

pytestmark = pytest.mark.gpu


def _run(B, Hq, Hkv, L, seed, num_splits=0, lens=None, shuffle=True):
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
    out = fa4q.decode_fp4q(to_dev_bf16(q, dev), kp, ks, vp, vs, t_table, t_len, n_phys, num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa4q.device_status()[0] == 0
    _, tps = fa4q.decode_fp4q_plan(B, Hq, Hkv, P, num_splits)
    got = out.float().cpu().numpy()
    G = Hq // Hkv
    gs, rs = [], []
    for b in range(B):
        for h in range(Hkv):
            n = int(lens[b])
            rs.append(BD.decode_group_fp4q(q[b, h * G:(h + 1) * G], k[b, h, :n], v[b, h, :n], tps))
            gs.append(got[b, h * G:(h + 1) * G])
    return np.stack(gs), np.stack(rs)


@pytest.mark.parametrize("B,Hq,Hkv,L,splits", [
    (2, 8, 2, 700, 0),       # odd page count: the last page pair holds one page
    (2, 8, 2, 1024, 3),
    (1, 4, 1, 4160, 0),
    (1, 8, 1, 300, 1),       # G = 8
    (1, 16, 1, 520, 0),      # G = 16: every column of the 16-head MMA tile
    (2, 6, 2, 1100, 2),      # G = 3: padded heads inside the 4-head instantiation
    (1, 2, 2, 130, 0),       # MHA; a last tile with 2 keys
])
def test_decode_fp4q(B, Hq, Hkv, L, splits):
    got, ref = _run(B, Hq, Hkv, L, L + Hq, splits)
    assert_close(got, ref, mean_rel=5e-3, what=f"decode_fp4q L={L}")


def test_decode_fp4q_ragged_lengths_and_empty_splits():
    """Sequences of different lengths in one batch: the short one's later splits are empty."""
    got, ref = _run(3, 8, 2, 2000, 7, num_splits=4, lens=[2000, 700, 64])
    assert_close(got, ref, mean_rel=5e-3, what="ragged")


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
    out = fa4q.decode_fp4q(to_dev_bf16(Q, dev), kp, ks, vp, vs, table, t_len, B * P).float().cpu().numpy()
    assert fa4q.device_status()[0] == 0
    _, tps = fa4q.decode_fp4q_plan(B, Hq, Hkv, P)
    G = Hq // Hkv
    gs, rs = [], []
    for (b, h), (kk, vv) in host.items():
        rs.append(BD.decode_group_fp4q(Q[b, h * G:(h + 1) * G], kk, vv, tps))
        gs.append(out[b, h * G:(h + 1) * G])
    assert_close(np.stack(gs), np.stack(rs), mean_rel=5e-3, what="decode_fp4q full size")

"""fa4q_quantize_kv_pages + fa4q_decode against the oracle's hybrid decode.

The query and the probabilities are FP16 inside the tensor-core tiles and the output is
bf16: outputs are compared with the FP64 oracle rounded to bf16, at max-abs <= 2e-2 and
mean-rel <= 2e-3 (the attention tolerance)."""
import numpy as np
import pytest

import synth
from oracle import decode as OD
from fa4q_testlib import assert_close, bf16_ref

pytestmark = pytest.mark.gpu


def build_cache(dw, dev, with_hp=True, with_win=True, slices=None, fmt="nvfp4", kv_scale=1.0):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    B, Hq, Hkv, d, L, W = dw.B, dw.Hq, dw.Hkv, dw.d, dw.L, dw.window
    n_fp4, P = dw.fp4_len, dw.n_pages
    tK = torch.empty((B, Hkv, L, d), dtype=torch.bfloat16, device=dev)
    tV = torch.empty((B, Hkv, L, d), dtype=torch.bfloat16, device=dev)
    host = {}
    for b in range(B):
        for h in range(Hkv):
            kk = synth.decode_kv_slice(dw, "k", b, h) * np.float32(kv_scale)
            vv = synth.decode_kv_slice(dw, "v", b, h) * np.float32(kv_scale)
            tK[b, h] = torch.from_numpy(kk).to(dev).to(torch.bfloat16)
            tV[b, h] = torch.from_numpy(vv).to(dev).to(torch.bfloat16)
            if slices is None or (b, h) in slices:
                host[(b, h)] = (kk, vv)
    Q = np.stack([synth.decode_query(dw, b) for b in range(B)])
    n_hp = dw.n_hp if with_hp else 0
    hp = [[synth.decode_hp_positions(dw, b, h, n_hp=n_hp) if n_hp else np.zeros(0, np.int64)
           for h in range(Hkv)] for b in range(B)]
    excl = np.zeros((B, Hkv, P), dtype=np.uint64)
    for b in range(B):
        for h in range(Hkv):
            for pos in hp[b][h]:
                excl[b, h, pos // 64] |= np.uint64(1) << np.uint64(pos % 64)
    table = synth.decode_block_table(dw)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).to(dev)
    fp4_len = i32(np.full(B, n_fp4))
    t_excl = torch.from_numpy(excl.view(np.int64)).to(dev)
    t_table = i32(table)
    kp, ks, vp, vs = fa4q.quantize_kv_pages(tK, tV, fp4_len, t_excl, t_table, B * P, fmt=fmt)
    if n_hp:
        idx = torch.from_numpy(np.stack([np.stack(r) for r in hp])).to(dev)
        hpk = torch.gather(tK[:, :, :n_fp4], 2, idx[..., None].expand(-1, -1, -1, d)).contiguous()
        hpv = torch.gather(tV[:, :, :n_fp4], 2, idx[..., None].expand(-1, -1, -1, d)).contiguous()
        hpc = i32(np.full((B, Hkv), n_hp))
    else:
        hpk = hpv = hpc = None
    if with_win:
        wk, wv, wl = tK[:, :, n_fp4:].contiguous(), tV[:, :, n_fp4:].contiguous(), i32(np.full(B, W))
    else:
        wk = wv = wl = None
    tq = torch.from_numpy(Q).to(dev).to(torch.bfloat16)
    args = (tq, kp, ks, vp, vs, t_table, fp4_len, t_excl, hpk, hpv, hpc, wk, wv, wl)
    return args, Q, hp, host


def oracle_group(dw, Q, hp, host, b, h, with_win=True, fmt="nvfp4"):
    kk, vv = host[(b, h)]
    G = dw.Hq // dw.Hkv
    W = dw.window if with_win else 0
    L = dw.L if with_win else dw.fp4_len
    return OD.decode_group(Q[b, h * G:(h + 1) * G], kk[:L], vv[:L], hp[b][h], W, fmt)


def _check(dw, with_hp=True, with_win=True, slices=None, num_splits=0, fmt="nvfp4", kv_scale=1.0):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    args, Q, hp, host = build_cache(dw, dev, with_hp, with_win, slices, fmt=fmt, kv_scale=kv_scale)
    out = fa4q.decode(*args, fmt=fmt, num_splits=num_splits).float().cpu().numpy()
    assert fa4q.device_status()[0] == 0
    G = dw.Hq // dw.Hkv
    gs, rs = [], []
    for (b, h) in (slices or [(b, h) for b in range(dw.B) for h in range(dw.Hkv)]):
        gs.append(out[b, h * G:(h + 1) * G])
        rs.append(oracle_group(dw, Q, hp, host, b, h, with_win, fmt))
    return assert_close(np.stack(gs), bf16_ref(np.stack(rs)), what=dw.name)


@pytest.mark.parametrize("L,splits", [(700, 0), (700, 3), (1000, 1), (4160, 0)])
def test_decode_small(L, splits):
    dw = synth.DecodeWorkload(91, f"decode_L{L}", B=2, Hq=8, Hkv=2, d=128, L=L)
    _check(dw, num_splits=splits)


def test_decode_without_hybrid_parts():
    dw = synth.DecodeWorkload(92, "decode_fp4_only", B=2, Hq=4, Hkv=2, d=128, L=900, window=0)
    _check(dw, with_hp=False, with_win=False)


def test_decode_mha_and_gqa8():
    _check(synth.DecodeWorkload(93, "decode_mha", B=1, Hq=2, Hkv=2, d=128, L=600))
    _check(synth.DecodeWorkload(94, "decode_g8", B=1, Hq=16, Hkv=2, d=128, L=600))


def test_full_size_decode_sampled_groups():
    """Batch 32, 32/8 heads, 32768 keys; sampled (sequence, kv-head) groups vs the oracle."""
    dw = synth.WORKLOADS[4]
    _check(dw, slices=[(0, 0), (13, 5), (31, 7)])


@pytest.mark.parametrize("L,splits", [(700, 0), (4160, 3)])
def test_decode_mxfp4_pages(L, splits):
    """MXFP4 pages (32-element blocks, E8M0 scales) against the oracle's MXFP4 decode."""
    dw = synth.DecodeWorkload(97, f"decode_mx_L{L}", B=2, Hq=8, Hkv=2, d=128, L=L)
    _check(dw, num_splits=splits, fmt="mxfp4")


@pytest.mark.parametrize("kv_scale", [2.0 ** -24, 2.0 ** 20])
def test_decode_mxfp4_extreme_block_exponents(kv_scale):
    """K and V scaled so far that their E8M0 block scales leave FP16's range: the pages'
    exponents are applied in FP32, so the output still matches the oracle relative to V's
    magnitude.  FP4 pages only (the BF16 vertical-line and window rows enter the tensor-core
    tiles through FP16 and are limited to its range)."""
    dw = synth.DecodeWorkload(98, "decode_mx_scaled", B=1, Hq=4, Hkv=1, d=128, L=900, window=0)
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    args, Q, hp, host = build_cache(dw, dev, with_hp=False, with_win=False, fmt="mxfp4", kv_scale=kv_scale)
    out = fa4q.decode(*args, fmt="mxfp4").float().cpu().numpy()
    assert fa4q.device_status()[0] == 0
    ref = oracle_group(dw, Q, hp, host, 0, 0, with_win=False, fmt="mxfp4")
    assert_close(out[0] / kv_scale, bf16_ref(ref) / kv_scale, what=f"mx decode x{kv_scale}")


def test_full_size_decode_mxfp4_sampled_groups():
    """The batch-32 / 32768-key decode with MXFP4 pages, sampled groups vs the oracle."""
    dw = synth.WORKLOADS[4]
    _check(dw, slices=[(0, 0), (31, 7)], fmt="mxfp4")

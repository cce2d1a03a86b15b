"""fa4q_quantize_rotated (Hadamard-rotated rows, the outlier-spreading alternative to
Smooth-QK) against the oracle: packed nibbles and scale bytes bit for bit, and the fused
attention on rotated Q, K against the oracle's PNQ attention on the same operands."""
import numpy as np
import pytest

import synth
from oracle import attention as OA
from oracle import formats as F
from oracle import rotate as OR
from fa4q_testlib import assert_close, tile_sf, to_dev_bf16

pytestmark = pytest.mark.gpu


def _outliers(shape, seed, scale=1.0):
    """Gaussians with four channels x20 (the causal GQA workload's K outliers) and a few
    all-zero rows."""
    rng = np.random.default_rng(seed)
    x = rng.normal(size=shape).astype(np.float32) * np.float32(scale)
    x[..., [3, 17, 40, shape[-1] - 5]] *= np.float32(20.0)
    x.reshape(-1, shape[-1])[::53] = 0.0
    return synth.round_to_bf16(x)


@pytest.mark.parametrize("fmt,qmax,g", [("nvfp4", 0.0, 1.0), ("nvfp4", 6.5, 0.37),
                                        ("mxfp4", 0.0, 1.0), ("mxfp4", 7.25, 1.0)])
@pytest.mark.parametrize("d,tiled", [(128, True), (128, False), (64, True), (64, False)])
def test_rotated_bit_exact(fmt, qmax, g, d, tiled):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    blk = F.block_size(fmt)
    x = _outliers((3, 200, d), d + int(qmax * 4) + tiled, 2.0 ** 10)
    p, s = fa4q.quantize_rotated(to_dev_bf16(x, dev), fmt, qmax, g,
                                 sf_layout=fa4q.FA4Q_SF_TILED if tiled else fa4q.FA4Q_SF_ROWMAJOR)
    p, s = p.cpu().numpy(), s.cpu().numpy()
    for gi in range(3):
        rp, rs = F.quantize_rows(OR.rotate_rows(x[gi]), fmt, qmax, g)
        assert np.array_equal(p[gi], rp), f"packed mismatch in group {gi}"
        assert np.array_equal(s[gi], tile_sf(rs, 200, d, blk) if tiled else rs), f"scales group {gi}"


def test_rotated_with_smoothing_multiplier():
    """The Smooth-QK multiplier (per kv-head, q-heads grouped) is applied before the rotation."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    Hq, ratio, S, d = 4, 2, 150, 128
    x = _outliers((Hq, S, d), 5)
    mul = np.float32(2.0) ** np.random.default_rng(6).integers(-4, 5, size=(Hq // ratio, d)).astype(np.float32)
    tm = torch.from_numpy(mul).to(dev)
    p, s = fa4q.quantize_rotated(to_dev_bf16(x, dev), "mxfp4", smooth_mul=tm, smooth_heads=Hq,
                                 smooth_ratio=ratio)
    p, s = p.cpu().numpy(), s.cpu().numpy()
    for h in range(Hq):
        rp, rs = F.quantize_rows(OR.rotate_rows(x[h], mul[h // ratio]), "mxfp4")
        assert np.array_equal(p[h], rp)
        assert np.array_equal(s[h], tile_sf(rs, S, d, 32))


@pytest.mark.parametrize("fmt,causal", [("mxfp4", True), ("nvfp4", False)])
def test_attention_on_rotated_q_k(fmt, causal):
    """Q and K rotated, V not; the score scale divided by d (H H^T = d I)."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    Hq, Hkv, S, d = 4, 2, 300, 128
    q = _outliers((1, Hq, S, d), 7, 1.5)
    k = _outliers((1, Hkv, S, d), 8, 1.5)
    v = synth.round_to_bf16(np.random.default_rng(9).normal(size=(1, Hkv, S, d)).astype(np.float32))
    sm = 1.0 / (d * np.sqrt(d))
    pq, sq = fa4q.quantize_rotated(to_dev_bf16(q, dev), fmt)
    pk, sk = fa4q.quantize_rotated(to_dev_bf16(k, dev), fmt)
    pv, sv = fa4q.quantize(to_dev_bf16(v, dev), fmt, fa4q.FA4Q_AXIS_OUTER)
    out = fa4q.attn_fwd(pq, sq, pk, sk, pv, sv, B=1, Hq=Hq, Hkv=Hkv, S_q=S, S_k=S, d=d, fmt=fmt,
                        causal=causal, sm_scale=float(np.float32(sm)), out_fp32=True)
    torch.cuda.synchronize()
    assert fa4q.device_status()[0] == 0
    got = out.cpu().numpy()
    gs, rs = [], []
    for h in range(Hq):
        kvh = h * Hkv // Hq
        qh = F.dequantize_rows(*F.quantize_rows(OR.rotate_rows(q[0, h]), fmt), fmt)
        kh = F.dequantize_rows(*F.quantize_rows(OR.rotate_rows(k[0, kvh]), fmt), fmt)
        pvo, svo = F.quantize_cols_transposed(v[0, kvh], fmt)
        vh = F.dequantize_rows(pvo, svo, fmt).T[:S]
        rs.append(OA.attention_pnq(qh, kh, vh, causal=causal, fmt=fmt, sm_scale=float(np.float32(sm))))
        gs.append(got[0, h])
    assert_close(np.stack(gs), np.stack(rs), what=f"rotated {fmt}")

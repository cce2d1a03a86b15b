"""fa4q_quantize against the oracle quantiser: packed nibbles and scale bytes bit for bit."""
import numpy as np
import pytest

import synth
from oracle import formats as F
from oracle import smooth as OS
from fa4q_testlib import tile_sf, untile_sf, to_dev_bf16

pytestmark = pytest.mark.gpu


def _wide(shape, seed, blk):
    """Gaussians with a per-block dynamic range of 2^-40..2^40, zero blocks and tiny blocks."""
    rng = np.random.default_rng(seed)
    x = rng.normal(size=shape).astype(np.float32)
    nb = shape[-1] // blk
    scale = np.exp2(rng.uniform(-40, 40, size=shape[:-1] + (nb, 1))).astype(np.float32)
    x = (x.reshape(shape[:-1] + (nb, blk)) * scale).reshape(shape)
    flat = x.reshape(-1, blk)
    flat[::97] = 0.0
    flat[5::89] *= np.float32(2.0 ** -100)
    flat[7::61] = np.abs(flat[7::61])
    return synth.round_to_bf16(x)


def _run_inner(x, fmt, qmax=0.0, g=1.0, mul=None, heads=1, ratio=1, tiled=True):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    tx = to_dev_bf16(x, dev)
    tm = None if mul is None else torch.from_numpy(np.ascontiguousarray(mul, dtype=np.float32)).to(dev)
    p, s = fa4q.quantize(tx, fmt, fa4q.FA4Q_AXIS_INNER, qmax, g, tm, heads, ratio,
                         fa4q.FA4Q_SF_TILED if tiled else fa4q.FA4Q_SF_ROWMAJOR)
    return p.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("fmt,qmax,g", [("nvfp4", 0.0, 1.0), ("nvfp4", 6.5, 0.37),
                                        ("mxfp4", 0.0, 1.0), ("mxfp4", 7.25, 1.0)])
@pytest.mark.parametrize("tiled", [False, True])
def test_inner_bit_exact(fmt, qmax, g, tiled):
    blk = F.block_size(fmt)
    x = _wide((3, 200, 128), 1 + int(qmax * 4) + tiled, blk)
    p, s = _run_inner(x, fmt, qmax, g, tiled=tiled)
    for gi in range(3):
        rp, rs = F.quantize_rows(x[gi], fmt, qmax, g)
        assert np.array_equal(p[gi], rp), f"packed mismatch in group {gi}"
        if tiled:
            assert np.array_equal(s[gi], tile_sf(rs, 200, 128, blk)), f"tiled scales group {gi}"
        else:
            assert np.array_equal(s[gi], rs), f"scales group {gi}"


@pytest.mark.parametrize("fmt,cols", [("nvfp4", 48), ("nvfp4", 80), ("mxfp4", 96)])
def test_inner_odd_blocks_per_row(fmt, cols):
    """Row-major scales with an odd number of blocks per row: a work unit of two slots then
    spans the end of one row and the start of the next, and an odd slot count ends in a
    single slot."""
    x = _wide((3, 51, cols), 5 + cols, F.block_size(fmt))
    p, s = _run_inner(x, fmt, tiled=False)
    for gi in range(3):
        rp, rs = F.quantize_rows(x[gi], fmt)
        assert np.array_equal(p[gi], rp), f"packed mismatch in group {gi}"
        assert np.array_equal(s[gi], rs), f"scales group {gi}"


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_inner_head_dim_64(fmt):
    blk = F.block_size(fmt)
    x = _wide((2, 130, 64), 11, blk)
    p, s = _run_inner(x, fmt)
    for gi in range(2):
        rp, rs = F.quantize_rows(x[gi], fmt)
        assert np.array_equal(p[gi], rp)
        assert np.array_equal(untile_sf(s[gi], 130, 64, blk), rs)
        assert np.array_equal(s[gi], tile_sf(rs, 130, 64, blk))


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("S,d", [(200, 128), (130, 64), (4096, 128)])
@pytest.mark.parametrize("tiled", [False, True])
def test_outer_transposed_bit_exact(fmt, S, d, tiled):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    blk = F.block_size(fmt)
    x = synth.round_to_bf16(np.random.default_rng(S + d).normal(size=(2, S, d)).astype(np.float32)
                            * np.float32(3.0))
    x[0, :17] = 0.0
    dev = torch.device("cuda:0")
    p, s = fa4q.quantize(to_dev_bf16(x, dev), fmt, fa4q.FA4Q_AXIS_OUTER,
                         sf_layout=fa4q.FA4Q_SF_TILED if tiled else fa4q.FA4Q_SF_ROWMAJOR)
    p, s = p.cpu().numpy(), s.cpu().numpy()
    S_pad = -(-S // 32) * 32
    for gi in range(2):
        rp, rs = F.quantize_cols_transposed(x[gi], fmt)
        assert np.array_equal(p[gi], rp)
        if tiled:
            assert np.array_equal(s[gi], tile_sf(rs, d, S_pad, blk))
        else:
            assert np.array_equal(s[gi], rs)


def test_smoothing_multiplier_and_calibration():
    """Smooth-QK on the causal GQA workload recipe: GPU calibration bit-exact with the oracle's,
    then Q*lambda and K/lambda quantised bit-exact."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    w = synth.WORKLOADS[2]
    qc, kc = synth.calibration_inputs(w)
    lam = OS.calibrate(qc, kc)
    dev = torch.device("cuda:0")
    mq, mk = fa4q.smooth_calibrate(to_dev_bf16(qc, dev), to_dev_bf16(kc, dev))
    assert np.array_equal(mq.cpu().numpy(), lam)
    assert np.array_equal(mk.cpu().numpy(), (1.0 / lam.astype(np.float64)).astype(np.float32))
    assert (lam > 1).any()
    q, k, _ = synth.prefill_inputs(w, S=512)
    pq, sq = _run_inner(q[0], "mxfp4", mul=lam, heads=w.Hq, ratio=w.Hq // w.Hkv)
    pk, sk = _run_inner(k[0], "mxfp4", mul=1.0 / lam, heads=w.Hkv, ratio=1)
    for h in range(w.Hq):
        rp, rs = F.quantize_rows(q[0, h], "mxfp4", mul=lam[h // 4][None, :])
        assert np.array_equal(pq[h], rp) and np.array_equal(untile_sf(sq[h], 512, 128, 32), rs)
    for h in range(w.Hkv):
        rp, rs = F.quantize_rows(k[0, h], "mxfp4", mul=(1.0 / lam[h])[None, :])
        assert np.array_equal(pk[h], rp) and np.array_equal(untile_sf(sk[h], 512, 128, 32), rs)


def test_full_size_long_prefill_tensors_bit_exact():
    """Every K and V element of the long causal NVFP4 workload (S = 16384)."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    w = synth.WORKLOADS[3]
    dev = torch.device("cuda:0")
    for h in (0, 5):
        k = synth.prefill_slice(w, "k", 0, h)
        v = synth.prefill_slice(w, "v", 0, h)
        pk, sk = fa4q.quantize(to_dev_bf16(k[None], dev), "nvfp4")
        pv, sv = fa4q.quantize(to_dev_bf16(v[None], dev), "nvfp4", axis=fa4q.FA4Q_AXIS_OUTER)
        rp, rs = F.quantize_rows(k, "nvfp4")
        assert np.array_equal(pk.cpu().numpy()[0], rp)
        assert np.array_equal(untile_sf(sk.cpu().numpy()[0], w.S, w.d, 16), rs)
        rp, rs = F.quantize_cols_transposed(v, "nvfp4")
        assert np.array_equal(pv.cpu().numpy()[0], rp)
        assert np.array_equal(untile_sf(sv.cpu().numpy()[0], w.d, w.S, 16), rs)


@pytest.mark.parametrize("fmt,d,S_q,S_k,Hq,Hkv,B,qmax,smooth,gs", [
    ("mxfp4", 128, 300, 300, 8, 2, 1, 0.0, True, (1.0, 1.0, 1.0)),
    ("nvfp4", 64, 129, 129, 4, 4, 2, 0.0, False, (0.5, 2.0, 0.25)),
    ("mxfp4", 128, 200, 333, 4, 1, 1, 7.25, False, (1.0, 1.0, 1.0)),
    ("nvfp4", 128, 4096, 4096, 32, 8, 1, 0.0, True, (1.0, 1.0, 1.0)),
])
def test_quantize_qkv_matches_separate_calls(fmt, d, S_q, S_k, Hq, Hkv, B, qmax, smooth, gs):
    """The one-launch Q/K/V quantisation writes exactly the bytes of the three separate calls
    (which the tests above pin bit-exactly to the oracle), padding bytes included."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(S_q + S_k + d)
    t = lambda shape: torch.from_numpy(synth.round_to_bf16(rng.normal(size=shape).astype(np.float32) * 2)
                                       ).to(dev).to(torch.bfloat16)
    q, k, v = t((B, Hq, S_q, d)), t((B, Hkv, S_k, d)), t((B, Hkv, S_k, d))
    mq = mk = None
    if smooth:
        lam = np.exp2(rng.integers(-3, 4, size=(Hkv, d))).astype(np.float32)
        mq = torch.from_numpy(lam).to(dev)
        mk = torch.from_numpy((1.0 / lam).astype(np.float32)).to(dev)
    g_q, g_k, g_v = gs
    sep = (*fa4q.quantize(q, fmt, fa4q.FA4Q_AXIS_INNER, qmax, g_q, mq, Hq, Hq // Hkv),
           *fa4q.quantize(k, fmt, fa4q.FA4Q_AXIS_INNER, qmax, g_k, mk, Hkv, 1),
           *fa4q.quantize(v, fmt, fa4q.FA4Q_AXIS_OUTER, qmax, g_v))
    fused = fa4q.quantize_qkv(q, k, v, fmt, qmax, g_q, g_k, g_v, mq, mk)
    torch.cuda.synchronize()
    for name, a, b in zip(("q", "q_sf", "k", "k_sf", "vt", "vt_sf"), sep, fused):
        assert a.shape == b.shape, (name, a.shape, b.shape)
        assert torch.equal(a, b), f"{name} differs"

"""One block-scaled FP4 tensor-core MMA (the prefill kernel's MMA path) against an FP64
product of the oracle-dequantised operands: pins operand swizzle, descriptors, scale-factor
TMEM layout and the per-format scale selection."""

import numpy as np
import pytest

from oracle import formats as F
from fa4q_testlib import tile_sf

pytestmark = pytest.mark.gpu


def _case(fmt, N, K, seed):
    rng = np.random.default_rng(seed)
    blk = F.block_size(fmt)
    ca = rng.integers(0, 16, size=(128, K), dtype=np.uint8)
    cb = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    if fmt == "nvfp4":
        sa = rng.integers(0x28, 0x48, size=(128, K // blk), dtype=np.uint8)
        sb = rng.integers(0x28, 0x48, size=(N, K // blk), dtype=np.uint8)
    else:
        sa = rng.integers(120, 134, size=(128, K // blk), dtype=np.uint8)
        sb = rng.integers(120, 134, size=(N, K // blk), dtype=np.uint8)
    return ca, cb, sa, sb


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("K", [64, 128])
@pytest.mark.parametrize("N", [16, 64, 128, 256])
def test_block_mma_matches_fp64(fmt, K, N):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    ca, cb, sa, sb = _case(fmt, N, K, seed=N * 1000 + K + (fmt == "mxfp4"))
    blk = F.block_size(fmt)
    A = F.dequantize_blocks(ca.reshape(128, K // blk, blk), sa, fmt).reshape(128, K)
    Bm = F.dequantize_blocks(cb.reshape(N, K // blk, blk), sb, fmt).reshape(N, K)
    ref = A @ Bm.T
    dev = torch.device("cuda:0")
    ta = torch.from_numpy(F.pack_nibbles(ca)).to(dev)
    tb = torch.from_numpy(F.pack_nibbles(cb)).to(dev)
    tsa = torch.from_numpy(tile_sf(sa, 128, K, blk)).to(dev)
    tsb = torch.from_numpy(tile_sf(sb, N, K, blk)).to(dev)
    got = fa4q.selftest_block_mma(ta, tsa, tb, tsb, N, K, fmt).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    bound = 1e-5 * (np.abs(A) @ np.abs(Bm).T) + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} of {bad.size} wrong; max err {np.abs(got - ref).max():.4g}"

"""Helpers for the GPU parity tests: layout conversions written from the C ABI's
documented layouts (not from the library), tolerance checks and input upload."""
import numpy as np


def untile_sf(buf, rows, cols, blk):
    """FA4Q_SF_TILED bytes of one [rows][cols] matrix -> row-major [rows][cols/blk]."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    nrt = -(-rows // 128)
    ng = -(-cols // 128) * (32 // blk)
    assert buf.size == nrt * ng * 512, (buf.size, nrt, ng)
    k = np.arange(cols // blk)
    r = np.arange(rows)
    off = ((r[:, None] // 128) * ng + k[None, :] // 4) * 512 + (r[:, None] % 32) * 16 \
        + ((r[:, None] % 128) // 32) * 4 + (k[None, :] % 4)
    return buf[off]


def tile_sf(sf_rm, rows, cols, blk):
    """Row-major [rows][cols/blk] -> FA4Q_SF_TILED bytes (padding zero)."""
    nrt = -(-rows // 128)
    ng = -(-cols // 128) * (32 // blk)
    out = np.zeros(nrt * ng * 512, dtype=np.uint8)
    k = np.arange(cols // blk)
    r = np.arange(rows)
    off = ((r[:, None] // 128) * ng + k[None, :] // 4) * 512 + (r[:, None] % 32) * 16 \
        + ((r[:, None] % 128) // 32) * 4 + (k[None, :] % 4)
    out[off] = sf_rm
    return out


def assert_close(got, ref, max_abs=2e-2, mean_rel=2e-3, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mr = err.sum() / max(np.abs(ref).sum(), 1e-30)
    assert err.max() <= max_abs and mr <= mean_rel, f"{what}: max_abs={err.max():.3e} mean_rel={mr:.3e}"
    return err.max(), mr


def to_dev_bf16(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(torch.bfloat16)

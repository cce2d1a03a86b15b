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
    """max |got - ref| <= max_abs and sum |got - ref| / sum |ref| <= mean_rel; prints the
    observed pair (visible with pytest -s or in the report of a failure)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mr = err.sum() / max(np.abs(ref).sum(), 1e-30)
    print(f"[parity] {what}: max_abs={err.max():.3e} mean_rel={mr:.3e} (bounds {max_abs:g} / {mean_rel:g})")
    assert err.max() <= max_abs and mr <= mean_rel, f"{what}: max_abs={err.max():.3e} mean_rel={mr:.3e}"
    return err.max(), mr


def bf16_ref(ref):
    """An FP64 oracle output rounded as the kernels round a bf16 output (to FP32, then to
    bfloat16 by round-to-nearest-even), for comparison with a bf16 result."""
    x = np.ascontiguousarray(np.asarray(ref, dtype=np.float64).astype(np.float32))
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32).astype(np.float64)


def to_dev_bf16(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(torch.bfloat16)

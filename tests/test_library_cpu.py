"""Host-side checks of the C ABI library: it loads without a GPU, exports every symbol the
header declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__.build()
    import microscaled_fp4_flashattention_b200 as fa4q
    return fa4q.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "fa4q.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa4q_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    import microscaled_fp4_flashattention_b200 as fa4q
    assert sorted(fa4q.EXPORTED) == names


def test_status_strings_and_version(L):
    assert L.fa4q_status_string(0) == b"ok"
    assert L.fa4q_status_string(4).startswith(b"a bounded")
    assert L.fa4q_version() == 100


def test_sf_tiled_bytes(L):
    assert L.fa4q_sf_tiled_bytes(128, 128, 0) == 2 * 512
    assert L.fa4q_sf_tiled_bytes(128, 128, 1) == 512
    assert L.fa4q_sf_tiled_bytes(129, 64, 0) == 2 * 2 * 512
    assert L.fa4q_sf_tiled_bytes(4096, 128, 0) == 32 * 2 * 512
    assert L.fa4q_sf_tiled_bytes(0, 128, 0) == 0


def test_argument_errors_without_gpu(L):
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: validation fails first
    # null input
    assert L.fa4q_quantize(None, 1, 16, 16, 16, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    # bad format / axis / misaligned stride
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 7, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 0, 5, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    assert L.fa4q_quantize(fake, 1, 16, 16, 12, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    # cols not a multiple of the block
    assert L.fa4q_quantize(fake, 1, 16, 24, 24, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 2
    # negative qmax, non-positive tensor scale
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 0, 0, -1.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 0, 0, 0.0, 0.0, None, 1, 1, 1, fake, fake, None) == 1
    # empty input is a no-op
    assert L.fa4q_quantize(fake, 0, 16, 16, 16, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 0
    F = ctypes.c_float
    # attention: unsupported head dim, GQA mismatch, causal with S_q != S_k
    args = [fake] * 6 + [F(1), F(1), F(1)]
    assert L.fa4q_attn_fwd(*args, 1, 4, 4, 128, 128, 96, 0, F(0), 0, F(0), fake, 1, None, None) == 2
    assert L.fa4q_attn_fwd(*args, 1, 6, 4, 128, 128, 128, 0, F(0), 0, F(0), fake, 1, None, None) == 1
    assert L.fa4q_attn_fwd(*args, 1, 4, 4, 128, 256, 128, 0, F(0), 1, F(0), fake, 1, None, None) == 1
    # conditional rescaling: threshold out of range; NVFP4 P with a kept reference
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 1, F(0), 0, F(0), 31, 0, fake, 1, None, None) == 1
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 1, F(0), 0, F(0), -1, 0, fake, 1, None, None) == 1
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 0, F(0), 0, F(0), 8, 0, fake, 1, None, None) == 2
    # inconsistent-normaliser flag must be 0 or 1
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 1, F(0), 0, F(0), 0, 2, fake, 1, None, None) == 1
    # rotated quantisation: head dims other than 64 / 128
    assert L.fa4q_quantize_rotated(fake, 1, 16, 96, 96, 0, F(0), F(1), None, 1, 1, 1, fake, fake, None) == 2
    assert L.fa4q_quantize_rotated(None, 1, 16, 128, 128, 0, F(0), F(1), None, 1, 1, 1, fake, fake, None) == 1
    # decode: group too large, workspace too small
    dargs = [fake] * 14
    assert L.fa4q_decode(*dargs, 1, 32, 2, 128, 4, 0, 0, 0, F(1), F(1), F(0), fake, fake, 1 << 30, 0, None) == 2
    assert L.fa4q_decode(*dargs, 1, 8, 2, 128, 4, 0, 0, 0, F(1), F(1), F(0), fake, fake, 16, 0, None) == 1
    # decode over a cache with no key slot at all (no pages, no BF16 set, no window), with the
    # automatic split count: refused as an argument error, with and without a workspace
    assert L.fa4q_decode(*dargs, 1, 8, 2, 128, 0, 0, 0, 0, F(1), F(1), F(0), fake, fake, 1 << 30, 0, None) == 1
    assert L.fa4q_decode_noalloc(*dargs, 1, 8, 2, 128, 0, 0, 0, 0, F(1), F(1), F(0), fake, 0, None) == 1
    # selftest: bad shapes
    assert L.fa4q_selftest_block_mma(fake, fake, fake, fake, 24, 64, 0, fake, None) == 2
    assert L.fa4q_selftest_block_mma(fake, fake, fake, fake, 128, 96, 0, fake, None) == 2


def test_binding_refuses_without_device(L):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(RuntimeError):
        fa4q._stream()


def test_decode_fp4q_plan_workspace_and_arguments(L):
    """The FP4 tensor-core decode's range rule and workspace size as fa4q.h states them (the
    split count is ceil(ceil(max_pages / 2) / T), T = tiles_per_split or 32, whatever the
    batch), and its argument checks (all return before any device call)."""
    for B, Hq, Hkv, P, tps in [(32, 32, 8, 512, 0), (2, 8, 2, 11, 0), (2, 8, 2, 16, 3), (1, 16, 1, 9, 0),
                               (1, 4, 1, 1, 0), (3, 8, 2, 32, 4), (1, 32, 8, 512, 0), (64, 32, 8, 512, 0)]:
        tiles = (P + 1) // 2
        T = tps if tps > 0 else 32
        splits = -(-tiles // T)
        part = B * Hq * splits * (128 + 2) * 4
        off_qt = -(-part // 1024) * 1024
        total = off_qt + B * Hkv * 2 * 128 * 64 + B * Hkv * 2 * 2 * 512
        assert L.fa4q_decode_fp4q_workspace_size(B, Hq, Hkv, 128, P, tps) == total
    assert L.fa4q_decode_fp4q_workspace_size(1, 4, 1, 128, 8, -1) == 0   # negative range length
    assert L.fa4q_decode_fp4q_workspace_size(1, 4, 1, 64, 8, 0) == 0     # d != 128
    assert L.fa4q_decode_fp4q_workspace_size(1, 4, 1, 128, 0, 0) == 0    # no pages
    P_, F = ctypes.c_void_p, ctypes.c_float
    fake = P_(0x1000)
    ptrs = [fake] * 7
    ws = L.fa4q_decode_fp4q_workspace_size(1, 8, 2, 128, 8, 0)

    def call(Hq=8, Hkv=2, d=128, fmt=0, q=fake, ws_bytes=ws, tps=0):
        return L.fa4q_decode_fp4q(q, *ptrs[1:], 16, 1, Hq, Hkv, d, 8, fmt, F(1), F(1), F(0), fake, fake,
                                  ws_bytes, tps, None)
    assert call(tps=-1) == 1                 # negative range length
    assert call(fmt=1) == 2                  # MXFP4 pages: the residual query is NVFP4
    assert call(fmt=5) == 1                  # unknown format
    assert call(q=None) == 1                 # null input
    assert call(Hq=34, Hkv=2) == 2           # G = 17 > 16 heads on the MMA's N side
    assert call(Hq=9, Hkv=2) == 1            # Hq not a multiple of Hkv
    assert call(d=64) == 2                   # head dimension other than 128
    assert call(ws_bytes=ws - 1) == 1        # workspace one byte short


def test_more_entry_points_reject_bad_arguments_without_gpu(L):
    """Hybrid prefill, fused Q/K/V quantisation, page quantisation, smoothing calibration and
    vertical-line selection: each error below is caught before any device call."""
    P_, F, D = ctypes.c_void_p, ctypes.c_float, ctypes.c_double
    fake = P_(0x1000)
    # hybrid prefill: bad format, window, head dim, missing vertical-line arrays, an NVFP4
    # V tensor scale that is not a bf16 value; an empty batch is a no-op
    def hyb(fmt=0, window=16, d=128, max_vl=0, vl=fake, B=1, g_v=1.0):
        return L.fa4q_attn_fwd_hybrid(*([fake] * 9), vl, vl, vl, vl, max_vl, vl, F(1), F(1), F(g_v), B, 4, 1, 128,
                                      d, window, fmt, F(0), F(0), fake, 1, None, None)
    assert hyb(fmt=3) == 1
    assert hyb(window=0) == 1
    assert hyb(d=64) == 2
    assert hyb(max_vl=8, vl=None) == 1
    assert hyb(g_v=1.1) == 2                 # 1.1 is not a bf16 value
    assert hyb(B=0, g_v=0.5) == 0
    assert hyb(B=0, fmt=1, g_v=1.1) == 0     # MXFP4 carries no tensor scale
    # fused Q/K/V quantisation: head dim, null input, GQA mismatch
    qkv = lambda q=fake, Hq=4, d=128: L.fa4q_quantize_qkv(q, fake, fake, 1, Hq, 2, 128, 128, d, 0, F(0), F(1),
                                                          F(1), F(1), None, None, *([fake] * 6), None)
    assert qkv(d=96) == 2
    assert qkv(q=None) == 1
    assert qkv(Hq=3) == 1
    # page quantisation: head dim, format, null input, empty length
    pages = lambda k=fake, L_=128, d=128, fmt=0: L.fa4q_quantize_kv_pages(
        k, fake, 1, 2, L_, d, fake, None, fake, 2, fmt, F(1), F(1), fake, fake, fake, fake, None)
    assert pages(d=64) == 2
    assert pages(fmt=4) == 1
    assert pages(k=None) == 1
    assert pages(L_=0) == 1
    # smoothing calibration: null input, GQA mismatch
    assert L.fa4q_smooth_calibrate(None, fake, 4, 2, 64, 128, fake, fake, None) == 1
    assert L.fa4q_smooth_calibrate(fake, fake, 5, 2, 64, 128, fake, fake, None) == 1
    # vertical-line selection: rho, head dim, too few selection slots, short workspace
    vws = L.fa4q_vlines_workspace_size(1, 4, 1, 64, 1024)
    assert vws > 0

    def vl(rho=0.05, d=128, max_select=64, ws_bytes=vws, ws=fake):
        return L.fa4q_select_vertical_lines(fake, fake, fake, fake, 1, 4, 1, 64, 1024, d, D(rho), F(0), fake, fake,
                                            fake, max_select, None, 0, None, None, ws, ws_bytes, None)
    assert vl(rho=0.0) == 1
    assert vl(rho=1.5) == 1
    assert vl(d=96) == 2
    assert vl(max_select=51) == 1           # ceil(0.05 * 1024) = 52 slots needed
    assert vl(ws_bytes=vws - 1) == 1
    assert vl(ws=P_(0x1008)) == 1           # the workspace must be 16-byte aligned (bulk copies)

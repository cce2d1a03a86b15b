"""Fused 4-bit microscaled FlashAttention for B200 - Python binding of libfa4q.so.

Argument marshalling only: every computation runs in the library's CUDA kernels.  PyTorch
supplies device memory and the current stream.  Importing works without a GPU (the library
loads and its symbols can be inspected); every compute call needs a CUDA device and raises
if the library or the device is missing - there is no CPU fallback.

The `fa4q_*` functions mirror the C ABI one to one (raw pointers and sizes).  The short
names (`quantize`, `attn_fwd`, ...) take torch tensors and allocate outputs.
"""
from __future__ import annotations

import ctypes
import math
import os

from ._build import LIB_PATH

FA4Q_NVFP4, FA4Q_MXFP4 = 0, 1
FA4Q_AXIS_INNER, FA4Q_AXIS_OUTER = 0, 1
FA4Q_SF_ROWMAJOR, FA4Q_SF_TILED = 0, 1
STATUS = {0: "FA4Q_OK", 1: "FA4Q_ERR_INVALID_ARG", 2: "FA4Q_ERR_UNSUPPORTED", 3: "FA4Q_ERR_CUDA",
          4: "FA4Q_ERR_TIMEOUT"}

EXPORTED = [
    "fa4q_status_string", "fa4q_version", "fa4q_sf_tiled_bytes", "fa4q_quantize",
    "fa4q_smooth_calibrate", "fa4q_attn_fwd", "fa4q_attn_fwd_ex", "fa4q_quantize_kv_pages",
    "fa4q_quantize_rotated", "fa4q_attn_fwd_hybrid",
    "fa4q_decode_fp4q", "fa4q_decode_fp4q_workspace_size",
    "fa4q_decode_workspace_size", "fa4q_decode", "fa4q_decode_noalloc", "fa4q_selftest_block_mma",
    "fa4q_device_status", "fa4q_selftest_wait_timeout", "fa4q_selftest_exp2",
    "fa4q_vlines_workspace_size", "fa4q_select_vertical_lines", "fa4q_quantize_qkv",
    "fa4q_selftest_bf16_mma",
]

_LIB = None


class Fa4qError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({lib().fa4q_status_string(code).decode()})")
        self.code = code


def lib() -> ctypes.CDLL:
    """The loaded libfa4q.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfa4q.so is missing at {LIB_PATH}; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, F, Z, U32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                ctypes.c_size_t, ctypes.c_uint32)
        L.fa4q_status_string.restype = ctypes.c_char_p
        L.fa4q_status_string.argtypes = [I]
        L.fa4q_version.restype = I
        L.fa4q_sf_tiled_bytes.restype = Z
        L.fa4q_sf_tiled_bytes.argtypes = [I64, I64, I]
        L.fa4q_quantize.restype = I
        L.fa4q_quantize.argtypes = [P, I64, I64, I64, I64, I, I, F, F, P, I64, I64, I, P, P, P]
        L.fa4q_attn_fwd_hybrid.restype = I
        L.fa4q_attn_fwd_hybrid.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, I, P, F, F, F, I, I, I, I, I,
                                           I, I, F, F, P, I, P, P]
        L.fa4q_decode_fp4q_workspace_size.restype = Z
        L.fa4q_decode_fp4q_workspace_size.argtypes = [I, I, I, I, I, I]
        L.fa4q_decode_fp4q.restype = I
        L.fa4q_decode_fp4q.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, F, F, P, P, Z, I, P]
        L.fa4q_quantize_rotated.restype = I
        L.fa4q_quantize_rotated.argtypes = [P, I64, I64, I64, I64, I, F, F, P, I64, I64, I, P, P, P]
        L.fa4q_smooth_calibrate.restype = I
        L.fa4q_smooth_calibrate.argtypes = [P, P, I, I, I, I, P, P, P]
        L.fa4q_attn_fwd.restype = I
        L.fa4q_attn_fwd.argtypes = [P, P, P, P, P, P, F, F, F, I, I, I, I, I, I, I, F, I, F, P, I, P, P]
        L.fa4q_attn_fwd_ex.restype = I
        L.fa4q_attn_fwd_ex.argtypes = [P, P, P, P, P, P, F, F, F, I, I, I, I, I, I, I, F, I, F, I, I, P, I, P, P]
        L.fa4q_quantize_kv_pages.restype = I
        L.fa4q_quantize_kv_pages.argtypes = [P, P, I, I, I, I, P, P, P, I, I, F, F, P, P, P, P, P]
        L.fa4q_decode_workspace_size.restype = Z
        L.fa4q_decode_workspace_size.argtypes = [I, I, I, I, I, I]
        L.fa4q_decode.restype = I
        L.fa4q_decode.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, F,
                                  F, P, P, Z, I, P]
        L.fa4q_decode_noalloc.restype = I
        L.fa4q_decode_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                          F, F, F, P, I, P]
        L.fa4q_selftest_block_mma.restype = I
        L.fa4q_selftest_block_mma.argtypes = [P, P, P, P, I, I, I, P, P]
        L.fa4q_selftest_bf16_mma.restype = I
        L.fa4q_selftest_bf16_mma.argtypes = [P, P, I, I, I, P, P]
        L.fa4q_device_status.restype = I
        L.fa4q_device_status.argtypes = [P, ctypes.POINTER(U32)]
        L.fa4q_selftest_wait_timeout.restype = I
        L.fa4q_selftest_wait_timeout.argtypes = [U32, P]
        L.fa4q_selftest_exp2.restype = I
        L.fa4q_selftest_exp2.argtypes = [P, P, I64, P]
        L.fa4q_quantize_qkv.restype = I
        L.fa4q_quantize_qkv.argtypes = [P, P, P, I, I, I, I, I, I, I, F, F, F, F, P, P, P, P, P, P, P, P, P]
        L.fa4q_vlines_workspace_size.restype = Z
        L.fa4q_vlines_workspace_size.argtypes = [I, I, I, I, I]
        L.fa4q_select_vertical_lines.restype = I
        L.fa4q_select_vertical_lines.argtypes = [P, P, P, P, I, I, I, I, I, I, ctypes.c_double, F, P, P, P, I, P, I, P, P,
                                                 P, Z, P]
        _LIB = L
    return _LIB


def _check(fn: str, code: int):
    if code != 0:
        raise Fa4qError(fn, code)


def _fmt(fmt) -> int:
    if isinstance(fmt, int):
        return fmt
    return {"nvfp4": FA4Q_NVFP4, "mxfp4": FA4Q_MXFP4}[fmt]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("fa4q compute calls need a CUDA device")
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def block_size(fmt) -> int:
    return 32 if _fmt(fmt) == FA4Q_MXFP4 else 16


def sf_tiled_bytes(rows: int, cols: int, fmt) -> int:
    return int(lib().fa4q_sf_tiled_bytes(rows, cols, _fmt(fmt)))


# ------------------------------------------------------------------------------------------
# tensor-level calls
# ------------------------------------------------------------------------------------------
def quantize(x, fmt, axis: int = FA4Q_AXIS_INNER, qmax: float = 0.0, tensor_scale: float = 1.0,
             smooth_mul=None, smooth_heads: int = 1, smooth_ratio: int = 1,
             sf_layout: int = FA4Q_SF_TILED, stream=None):
    """x: bf16 CUDA tensor [..., rows, cols] (leading dims = groups, contiguous).
    Returns (packed uint8, scales uint8) in the layouts of fa4q_quantize."""
    import torch
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
    rows, cols = x.shape[-2], x.shape[-1]
    groups = x.numel() // max(1, rows * cols)
    f = _fmt(fmt)
    blk = block_size(f)
    lead = tuple(x.shape[:-2])
    if axis == FA4Q_AXIS_INNER:
        packed = torch.empty(lead + (rows, cols // 2), dtype=torch.uint8, device=x.device)
        if sf_layout == FA4Q_SF_TILED:
            sf = torch.empty(lead + (sf_tiled_bytes(rows, cols, f),), dtype=torch.uint8, device=x.device)
        else:
            sf = torch.empty(lead + (rows, cols // blk), dtype=torch.uint8, device=x.device)
    else:
        rows_pad = (rows + 31) // 32 * 32
        packed = torch.empty(lead + (cols, rows_pad // 2), dtype=torch.uint8, device=x.device)
        if sf_layout == FA4Q_SF_TILED:
            sf = torch.empty(lead + (sf_tiled_bytes(cols, rows_pad, f),), dtype=torch.uint8, device=x.device)
        else:
            sf = torch.empty(lead + (cols, rows_pad // blk), dtype=torch.uint8, device=x.device)
    _check("fa4q_quantize", lib().fa4q_quantize(
        _ptr(x), groups, rows, cols, cols, f, axis, qmax, tensor_scale, _ptr(smooth_mul),
        smooth_heads, smooth_ratio, sf_layout, _ptr(packed), _ptr(sf), _stream(stream)))
    return packed, sf


def quantize_rotated(x, fmt, qmax: float = 0.0, tensor_scale: float = 1.0, smooth_mul=None,
                     smooth_heads: int = 1, smooth_ratio: int = 1, sf_layout: int = FA4Q_SF_TILED,
                     stream=None):
    """Hadamard-rotated rows quantised along cols (fa4q_quantize_rotated); x bf16 CUDA
    tensor [..., rows, cols], cols 64 or 128.  Returns (packed, scales) as quantize()."""
    import torch
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
    rows, cols = x.shape[-2], x.shape[-1]
    groups = x.numel() // max(1, rows * cols)
    f = _fmt(fmt)
    blk = block_size(f)
    lead = tuple(x.shape[:-2])
    packed = torch.empty(lead + (rows, cols // 2), dtype=torch.uint8, device=x.device)
    if sf_layout == FA4Q_SF_TILED:
        sf = torch.empty(lead + (sf_tiled_bytes(rows, cols, f),), dtype=torch.uint8, device=x.device)
    else:
        sf = torch.empty(lead + (rows, cols // blk), dtype=torch.uint8, device=x.device)
    _check("fa4q_quantize_rotated", lib().fa4q_quantize_rotated(
        _ptr(x), groups, rows, cols, cols, f, qmax, tensor_scale, _ptr(smooth_mul), smooth_heads,
        smooth_ratio, sf_layout, _ptr(packed), _ptr(sf), _stream(stream)))
    return packed, sf


def attn_fwd_hybrid(q, q_sf, k, k_sf, vt, vt_sf, q_bf16, k_bf16, v_bf16, vl_pos, vl_count, vl_k, vl_v,
                    vl_excl, *, B, Hq, Hkv, S, d, window, fmt, g_q=1.0, g_k=1.0, g_v=1.0, qmax_p=0.0,
                    sm_scale=0.0, out=None, out_fp32=False, lse=None, stream=None):
    """Hybrid-precision causal prefill (fa4q_attn_fwd_hybrid); vl_* may be None (no vertical
    lines).  Returns out [B, Hq, S, d]."""
    import torch
    if out is None:
        out = torch.empty((B, Hq, S, d), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    max_vl = 0 if vl_pos is None else int(vl_pos.shape[-1])
    _check("fa4q_attn_fwd_hybrid", lib().fa4q_attn_fwd_hybrid(
        _ptr(q), _ptr(q_sf), _ptr(k), _ptr(k_sf), _ptr(vt), _ptr(vt_sf), _ptr(q_bf16), _ptr(k_bf16),
        _ptr(v_bf16), _ptr(vl_pos), _ptr(vl_count), _ptr(vl_k), _ptr(vl_v), max_vl, _ptr(vl_excl), g_q, g_k,
        g_v, B, Hq, Hkv, S, d, window, _fmt(fmt), qmax_p, sm_scale, _ptr(out), int(out_fp32), _ptr(lse),
        _stream(stream)))
    return out


def decode_fp4q(q, k_pages, k_sf, vt_pages, vt_sf, block_table, fp4_len, n_phys_pages, *, fmt="nvfp4",
                g_k=1.0, g_v=1.0, sm_scale=0.0, tiles_per_split=0, out=None, workspace=None, stream=None):
    """FP4 tensor-core decode with a dual-residual query (fa4q_decode_fp4q); out [B, Hq, d].
    tiles_per_split: the scan restarts every that many 128-key tiles (0: the library's fixed
    default, 32); it is part of the result."""
    import torch
    B, Hq, d = q.shape
    Hkv = k_pages.shape[1]
    max_pages = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        need = int(lib().fa4q_decode_fp4q_workspace_size(B, Hq, Hkv, d, max_pages, tiles_per_split))
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check("fa4q_decode_fp4q", lib().fa4q_decode_fp4q(
        _ptr(q), _ptr(k_pages), _ptr(k_sf), _ptr(vt_pages), _ptr(vt_sf), _ptr(block_table), _ptr(fp4_len),
        n_phys_pages, B, Hq, Hkv, d, max_pages, _fmt(fmt), g_k, g_v, sm_scale, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), tiles_per_split, _stream(stream)))
    return out


def smooth_calibrate(q_cal, k_cal, stream=None):
    """q_cal bf16 [Hq, T, d], k_cal bf16 [Hkv, T, d] -> (mul_q, mul_k) float32 [Hkv, d]."""
    import torch
    Hq, T, d = q_cal.shape
    Hkv = k_cal.shape[0]
    mq = torch.empty((Hkv, d), dtype=torch.float32, device=q_cal.device)
    mk = torch.empty((Hkv, d), dtype=torch.float32, device=q_cal.device)
    _check("fa4q_smooth_calibrate", lib().fa4q_smooth_calibrate(
        _ptr(q_cal), _ptr(k_cal), Hq, Hkv, T, d, _ptr(mq), _ptr(mk), _stream(stream)))
    return mq, mk


def attn_fwd(q, q_sf, k, k_sf, vt, vt_sf, *, B, Hq, Hkv, S_q, S_k, d, fmt, causal,
             g_q=1.0, g_k=1.0, g_v=1.0, qmax_p=0.0, sm_scale=0.0, out=None, out_fp32=False,
             lse=None, rescale_tau=0, l_from_ptilde=False, stream=None):
    """Prefill attention on quantised operands; returns out [B, Hq, S_q, d].
    rescale_tau > 0 (conditional rescaling) or l_from_ptilde (the inconsistent normaliser)
    select the ablations of fa4q_attn_fwd_ex."""
    import torch
    if out is None:
        out = torch.empty((B, Hq, S_q, d), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    if rescale_tau or l_from_ptilde:
        _check("fa4q_attn_fwd_ex", lib().fa4q_attn_fwd_ex(
            _ptr(q), _ptr(q_sf), _ptr(k), _ptr(k_sf), _ptr(vt), _ptr(vt_sf), g_q, g_k, g_v, B, Hq, Hkv,
            S_q, S_k, d, _fmt(fmt), qmax_p, int(causal), sm_scale, int(rescale_tau), int(l_from_ptilde),
            _ptr(out), int(out_fp32), _ptr(lse), _stream(stream)))
        return out
    _check("fa4q_attn_fwd", lib().fa4q_attn_fwd(
        _ptr(q), _ptr(q_sf), _ptr(k), _ptr(k_sf), _ptr(vt), _ptr(vt_sf), g_q, g_k, g_v, B, Hq, Hkv,
        S_q, S_k, d, _fmt(fmt), qmax_p, int(causal), sm_scale, _ptr(out), int(out_fp32), _ptr(lse),
        _stream(stream)))
    return out


def quantize_qkv(q, k, v, fmt, qmax: float = 0.0, g_q=1.0, g_k=1.0, g_v=1.0, mul_q=None, mul_k=None,
                 out=None, stream=None):
    """Q, K (blocks along d, optional smoothing multipliers) and V (transposed) in one launch.
    q bf16 [B, Hq, S_q, d]; k, v bf16 [B, Hkv, S_k, d].  Returns (pq, sq, pk, sk, pv, sv) as
    quantize() gives them with the tiled scale layout; `out` may pass those six tensors."""
    import torch
    B, Hq, S_q, d = q.shape
    _, Hkv, S_k, _ = k.shape
    f = _fmt(fmt)
    if out is None:
        dev = q.device
        u8 = lambda *s: torch.empty(s, dtype=torch.uint8, device=dev)
        rp = (S_k + 31) // 32 * 32
        out = (u8(B, Hq, S_q, d // 2), u8(B, Hq, sf_tiled_bytes(S_q, d, f)),
               u8(B, Hkv, S_k, d // 2), u8(B, Hkv, sf_tiled_bytes(S_k, d, f)),
               u8(B, Hkv, d, rp // 2), u8(B, Hkv, sf_tiled_bytes(d, rp, f)))
    pq, sq, pk, sk, pv, sv = out
    _check("fa4q_quantize_qkv", lib().fa4q_quantize_qkv(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, S_q, S_k, d, f, qmax, g_q, g_k, g_v, _ptr(mul_q), _ptr(mul_k),
        _ptr(pq), _ptr(sq), _ptr(pk), _ptr(sk), _ptr(pv), _ptr(sv), _stream(stream)))
    return out


def quantize_kv_pages(k, v, fp4_len, excl_mask, block_table, n_phys_pages: int, fmt="nvfp4",
                      g_k=1.0, g_v=1.0, stream=None):
    """k, v bf16 [B, Hkv, L, d]; fp4_len int32 [B]; excl_mask uint64-as-int64 [B, Hkv, P] or None;
    block_table int32 [B, P].  Returns (k_pages, k_sf, vt_pages, vt_sf)."""
    import torch
    B, Hkv, L, d = k.shape
    max_pages = block_table.shape[1]
    f = _fmt(fmt)
    blk = block_size(f)
    dev = k.device
    kp = torch.zeros((n_phys_pages, Hkv, 64, d // 2), dtype=torch.uint8, device=dev)
    ks = torch.zeros((n_phys_pages, Hkv, 64, d // blk), dtype=torch.uint8, device=dev)
    vp = torch.zeros((n_phys_pages, Hkv, d, 32), dtype=torch.uint8, device=dev)
    vs = torch.zeros((n_phys_pages, Hkv, d, 64 // blk), dtype=torch.uint8, device=dev)
    _check("fa4q_quantize_kv_pages", lib().fa4q_quantize_kv_pages(
        _ptr(k), _ptr(v), B, Hkv, L, d, _ptr(fp4_len), _ptr(excl_mask), _ptr(block_table), max_pages,
        f, g_k, g_v, _ptr(kp), _ptr(ks), _ptr(vp), _ptr(vs), _stream(stream)))
    return kp, ks, vp, vs


def vlines_workspace_size(B, Hq, Hkv, n_obs, L) -> int:
    return int(lib().fa4q_vlines_workspace_size(B, Hq, Hkv, n_obs, L))


def select_vertical_lines(q_obs, k, v, n_prefix, *, rho=0.05, sm_scale=0.0, max_select=None,
                          max_pages=None, with_rows=True, workspace=None, stream=None):
    """Vertical-line tokens by accumulated column mass.

    q_obs bf16 [B, Hq, n_obs, d]; k, v bf16 [B, Hkv, L, d]; n_prefix int32 [B] (device).
    Returns a dict: mass [B, Hkv, L] fp32, positions [B, Hkv, max_select] int32 (ascending,
    valid up to counts), counts [B, Hkv] int32, excl (uint64 words as int64 [B, Hkv, max_pages]),
    hp_k / hp_v [B, Hkv, max_select, d] bf16 (when with_rows)."""
    import math
    import torch
    B, Hq, n_obs, d = q_obs.shape
    _, Hkv, L, _ = k.shape
    dev = k.device
    if max_select is None:
        max_select = max(1, int(math.ceil(rho * L - 1e-9)))
    if max_pages is None:
        max_pages = -(-L // 64)
    mass = torch.empty((B, Hkv, L), dtype=torch.float32, device=dev)
    positions = torch.empty((B, Hkv, max_select), dtype=torch.int32, device=dev)
    counts = torch.empty((B, Hkv), dtype=torch.int32, device=dev)
    excl = torch.empty((B, Hkv, max_pages), dtype=torch.int64, device=dev)
    hp_k = torch.zeros((B, Hkv, max_select, d), dtype=torch.bfloat16, device=dev) if with_rows else None
    hp_v = torch.zeros((B, Hkv, max_select, d), dtype=torch.bfloat16, device=dev) if with_rows else None
    ws_bytes = vlines_workspace_size(B, Hq, Hkv, n_obs, L)
    if workspace is None:
        workspace = torch.empty(max(16, ws_bytes), dtype=torch.uint8, device=dev)
    _check("fa4q_select_vertical_lines", lib().fa4q_select_vertical_lines(
        _ptr(q_obs), _ptr(k), _ptr(v) if with_rows else None, _ptr(n_prefix), B, Hq, Hkv, n_obs, L, d,
        rho, sm_scale, _ptr(mass), _ptr(positions), _ptr(counts), max_select, _ptr(excl), max_pages,
        _ptr(hp_k), _ptr(hp_v), _ptr(workspace), workspace.numel(), _stream(stream)))
    return {"mass": mass, "positions": positions, "counts": counts, "excl": excl, "hp_k": hp_k, "hp_v": hp_v}


def decode_workspace_size(B, Hq, Hkv, d, max_pages, num_splits=0) -> int:
    return int(lib().fa4q_decode_workspace_size(B, Hq, Hkv, d, max_pages, num_splits))


def decode(q, k_pages, k_sf, vt_pages, vt_sf, block_table, fp4_len, excl_mask, hp_k, hp_v, hp_count,
           win_k, win_v, win_len, *, fmt="nvfp4", g_k=1.0, g_v=1.0, sm_scale=0.0, num_splits=0,
           out=None, workspace=None, stream=None):
    """q bf16 [B, Hq, d] -> out bf16 [B, Hq, d] over the hybrid paged cache."""
    import torch
    B, Hq, d = q.shape
    Hkv = k_pages.shape[1] if k_pages is not None else hp_k.shape[1]
    max_pages = block_table.shape[1] if block_table is not None else 0
    max_hp = hp_k.shape[2] if hp_k is not None else 0
    W = win_k.shape[2] if win_k is not None else 0
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    ws_bytes = decode_workspace_size(B, Hq, Hkv, d, max_pages, num_splits)
    if workspace is None:
        workspace = torch.empty(max(16, ws_bytes), dtype=torch.uint8, device=q.device)
    _check("fa4q_decode", lib().fa4q_decode(
        _ptr(q), _ptr(k_pages), _ptr(k_sf), _ptr(vt_pages), _ptr(vt_sf), _ptr(block_table),
        _ptr(fp4_len), _ptr(excl_mask), _ptr(hp_k), _ptr(hp_v), _ptr(hp_count), _ptr(win_k),
        _ptr(win_v), _ptr(win_len), B, Hq, Hkv, d, max_pages, max_hp, W, _fmt(fmt), g_k, g_v, sm_scale,
        _ptr(out), _ptr(workspace), workspace.numel(), num_splits, _stream(stream)))
    return out


def decode_noalloc(q, k_pages, k_sf, vt_pages, vt_sf, block_table, fp4_len, excl_mask, hp_k, hp_v,
                   hp_count, win_k, win_v, win_len, *, fmt="nvfp4", g_k=1.0, g_v=1.0, sm_scale=0.0,
                   num_splits=0, out=None, stream=None):
    """decode() without a workspace: the split partials live in the library's static device
    array (for callers that cannot allocate device memory; see fa4q_decode_noalloc)."""
    import torch
    B, Hq, d = q.shape
    Hkv = k_pages.shape[1] if k_pages is not None else hp_k.shape[1]
    max_pages = block_table.shape[1] if block_table is not None else 0
    max_hp = hp_k.shape[2] if hp_k is not None else 0
    W = win_k.shape[2] if win_k is not None else 0
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _check("fa4q_decode_noalloc", lib().fa4q_decode_noalloc(
        _ptr(q), _ptr(k_pages), _ptr(k_sf), _ptr(vt_pages), _ptr(vt_sf), _ptr(block_table),
        _ptr(fp4_len), _ptr(excl_mask), _ptr(hp_k), _ptr(hp_v), _ptr(hp_count), _ptr(win_k),
        _ptr(win_v), _ptr(win_len), B, Hq, Hkv, d, max_pages, max_hp, W, _fmt(fmt), g_k, g_v, sm_scale,
        _ptr(out), num_splits, _stream(stream)))
    return out


def selftest_block_mma(a, a_sf, b, b_sf, N, K, fmt, stream=None):
    import torch
    d = torch.empty((128, N), dtype=torch.float32, device=a.device)
    _check("fa4q_selftest_block_mma", lib().fa4q_selftest_block_mma(
        _ptr(a), _ptr(a_sf), _ptr(b), _ptr(b_sf), N, K, _fmt(fmt), _ptr(d), _stream(stream)))
    return d


def selftest_bf16_mma(a, b, N, K, b_mn_major, stream=None):
    """One BF16 tensor-core product (fa4q_selftest_bf16_mma); returns FP32 [128, N]."""
    import torch
    out = torch.empty((128, N), dtype=torch.float32, device=a.device)
    _check("fa4q_selftest_bf16_mma", lib().fa4q_selftest_bf16_mma(_ptr(a), _ptr(b), N, K, int(b_mn_major),
                                                                  _ptr(out), _stream(stream)))
    torch.cuda.synchronize()
    return out


def device_status(stream=None):
    """(status code, detail bits) of the device status word; clears it."""
    detail = ctypes.c_uint32(0)
    code = lib().fa4q_device_status(_stream(stream), ctypes.byref(detail))
    return code, detail.value


def selftest_wait_timeout(wait_us: int, stream=None):
    _check("fa4q_selftest_wait_timeout", lib().fa4q_selftest_wait_timeout(wait_us, _stream(stream)))


def selftest_exp2(x, stream=None):
    """2^x through the prefill kernel's FMA-pipe exponential (x: CUDA float32, even length)."""
    import torch
    x = x.contiguous()
    y = torch.empty_like(x)
    _check("fa4q_selftest_exp2", lib().fa4q_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def default_sm_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)

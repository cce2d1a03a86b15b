"""Seeded synthetic inputs for the FP4 attention workloads.

This module only draws numbers: Gaussian tensors rounded to bfloat16, rotary
position embedding applied to them before rounding, planted outliers, the
paged-cache block table and the choice of full-precision decode tokens.  It
holds none of the attention or quantisation arithmetic; both the CUDA library's
callers and the CPU oracle take their inputs from here.

Every tensor slice is drawn from its own numpy PCG64 stream keyed by
(seed, stream, batch, head), so any (batch, head) slice of a large workload can
be regenerated on its own on the CPU without drawing the rest.

Streams (per workload seed = 20260000 + workload id):
    1 = Q, 2 = K, 3 = V, 4 = calibration draw, 5 = outlier / selection /
    block table, 6 = observation queries.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 20260000
STREAM_Q, STREAM_K, STREAM_V, STREAM_CAL, STREAM_SEL, STREAM_OBS = 1, 2, 3, 4, 5, 6


# ----------------------------------------------------------------------------
# workloads (the shapes of the five synthetic configurations)
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class PrefillWorkload:
    wid: int
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    d: int
    causal: bool
    fmt: str                  # "nvfp4" | "mxfp4"
    qmax: float = 0.0         # 0 = default rule (NVFP4: 6, MXFP4: OCP)
    qmax_p: float = 0.0       # scale bound for P (same convention)
    smooth: bool = False      # per-channel Q/K smoothing (calibrated)
    rope_base: float = 0.0    # 0 = no rotary embedding
    k_outlier_channels: int = 0
    k_outlier_scale: float = 1.0
    token_outlier_frac: float = 0.0
    token_outlier_scale: float = 1.0

    @property
    def flops(self) -> float:
        f = 4.0 * self.B * self.Hq * self.S * self.S * self.d
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class DecodeWorkload:
    wid: int
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int                    # keys per sequence, the current token included
    page: int = 64
    window: int = 128
    hp_frac: float = 0.05     # full-precision vertical-line share of the non-window prefix
    fmt: str = "nvfp4"

    @property
    def fp4_len(self) -> int:
        return self.L - self.window

    @property
    def n_pages(self) -> int:
        return -(-self.fp4_len // self.page)

    @property
    def n_hp(self) -> int:
        return int(math.ceil(self.hp_frac * self.fp4_len - 1e-9))


WORKLOADS = {
    1: PrefillWorkload(1, "tiny_noncausal_nvfp4_s128_d64", 1, 2, 2, 128, 64, False, "nvfp4"),
    2: PrefillWorkload(2, "causal_gqa_mxfp4_smooth_s4096", 1, 32, 8, 4096, 128, True, "mxfp4",
                       smooth=True, rope_base=1e4, k_outlier_channels=4, k_outlier_scale=20.0),
    3: PrefillWorkload(3, "causal_gqa_nvfp4_s16384", 1, 32, 8, 16384, 128, True, "nvfp4",
                       rope_base=1e6),
    4: DecodeWorkload(4, "decode_paged_nvfp4_b32_ctx32768", 32, 32, 8, 128, 32768),
    5: PrefillWorkload(5, "noncausal_mxfp4_uos_h40_s32768", 1, 40, 40, 32768, 128, False, "mxfp4",
                       qmax=7.25, qmax_p=7.25, token_outlier_frac=0.01, token_outlier_scale=8.0),
}


# ----------------------------------------------------------------------------
# primitive draws
# ----------------------------------------------------------------------------
def generator(wid: int, stream: int, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence([SEED_BASE + wid, stream, *[int(k) for k in key]])
    return np.random.Generator(np.random.PCG64(ss))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); finite inputs only."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-exact float32 values (the bfloat16 encoding)."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def normal(wid: int, stream: int, shape, *key: int) -> np.ndarray:
    return generator(wid, stream, *key).standard_normal(shape, dtype=np.float32)


def rope_rotate_half(x: np.ndarray, base: float, pos0: int = 0) -> np.ndarray:
    """Rotate-half rotary embedding over the last axis; positions along axis -2."""
    S, d = x.shape[-2], x.shape[-1]
    half = d // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(pos0, pos0 + S, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x64 = x.astype(np.float64)
    a, b = x64[..., :half], x64[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1).astype(np.float32)


# ----------------------------------------------------------------------------
# prefill inputs
# ----------------------------------------------------------------------------
def k_outlier_channels(w: PrefillWorkload, h_kv: int) -> np.ndarray:
    if w.k_outlier_channels == 0:
        return np.zeros(0, dtype=np.int64)
    g = generator(w.wid, STREAM_SEL, 1, h_kv)
    return np.sort(g.choice(w.d, size=w.k_outlier_channels, replace=False))


def token_outlier_positions(w: PrefillWorkload, S: int | None = None) -> np.ndarray:
    S = w.S if S is None else S
    if w.token_outlier_frac <= 0:
        return np.zeros(0, dtype=np.int64)
    n = int(round(w.token_outlier_frac * S))
    return np.sort(generator(w.wid, STREAM_SEL, 2).choice(S, size=n, replace=False))


def _slice(w: PrefillWorkload, stream: int, b: int, h: int, S: int, h_kv: int, tokens0: int = 0) -> np.ndarray:
    x = normal(w.wid, stream, (S, w.d), b, h)
    if w.rope_base:
        x = rope_rotate_half(x, w.rope_base, pos0=tokens0)
    if stream in (STREAM_K,) and w.k_outlier_channels:
        x[:, k_outlier_channels(w, h_kv)] *= np.float32(w.k_outlier_scale)
    if w.token_outlier_frac > 0:
        pos = token_outlier_positions(w, S)
        x[pos, :] *= np.float32(w.token_outlier_scale)
    return round_to_bf16(x)


def prefill_slice(w: PrefillWorkload, which: str, b: int, h: int, S: int | None = None) -> np.ndarray:
    """One [S, d] bf16-exact float32 slice of Q (h = q-head) or K/V (h = kv-head)."""
    S = w.S if S is None else S
    stream = {"q": STREAM_Q, "k": STREAM_K, "v": STREAM_V}[which]
    h_kv = h * w.Hkv // w.Hq if which == "q" else h
    return _slice(w, stream, b, h, S, h_kv)


def prefill_inputs(w: PrefillWorkload, S: int | None = None, heads: tuple[int, int] | None = None):
    """Full Q, K, V ([B, H, S, d] float32, bf16-exact) for a prefill workload.

    `S` overrides the sequence length (smaller parity cases of the same recipe);
    `heads` overrides (Hq, Hkv)."""
    S = w.S if S is None else S
    Hq, Hkv = heads if heads else (w.Hq, w.Hkv)
    ww = w if not heads else PrefillWorkload(**{**w.__dict__, "Hq": Hq, "Hkv": Hkv})
    q = np.stack([np.stack([prefill_slice(ww, "q", b, h, S) for h in range(Hq)]) for b in range(w.B)])
    k = np.stack([np.stack([prefill_slice(ww, "k", b, h, S) for h in range(Hkv)]) for b in range(w.B)])
    v = np.stack([np.stack([prefill_slice(ww, "v", b, h, S) for h in range(Hkv)]) for b in range(w.B)])
    return q, k, v


def calibration_inputs(w: PrefillWorkload, tokens: int = 512, heads: tuple[int, int] | None = None):
    """A separate calibration draw (stream 4) of Q and K with the same recipe: [Hq|Hkv, tokens, d]."""
    Hq, Hkv = heads if heads else (w.Hq, w.Hkv)
    qc, kc = [], []
    for h in range(Hq):
        x = normal(w.wid, STREAM_CAL, (tokens, w.d), 0, h)
        if w.rope_base:
            x = rope_rotate_half(x, w.rope_base)
        qc.append(round_to_bf16(x))
    for h in range(Hkv):
        x = normal(w.wid, STREAM_CAL, (tokens, w.d), 1, h)
        if w.rope_base:
            x = rope_rotate_half(x, w.rope_base)
        if w.k_outlier_channels:
            x[:, k_outlier_channels(w, h)] *= np.float32(w.k_outlier_scale)
        kc.append(round_to_bf16(x))
    return np.stack(qc), np.stack(kc)


# ----------------------------------------------------------------------------
# decode inputs
# ----------------------------------------------------------------------------
def decode_query(w: DecodeWorkload, b: int) -> np.ndarray:
    return round_to_bf16(normal(w.wid, STREAM_Q, (w.Hq, w.d), b))


def decode_kv_slice(w: DecodeWorkload, which: str, b: int, h: int, L: int | None = None) -> np.ndarray:
    L = w.L if L is None else L
    stream = STREAM_K if which == "k" else STREAM_V
    return round_to_bf16(normal(w.wid, stream, (L, w.d), b, h))


def decode_observation_queries(w: DecodeWorkload, b: int, n_obs: int = 64) -> np.ndarray:
    """[Hq, n_obs, d] bf16-valued observation queries (stream 6) from which the vertical-line
    tokens of sequence b are identified by accumulated column mass."""
    return round_to_bf16(normal(w.wid, STREAM_OBS, (w.Hq, n_obs, w.d), b))


def decode_hp_positions(w: DecodeWorkload, b: int, h: int, fp4_len: int | None = None, n_hp: int | None = None) -> np.ndarray:
    """Sorted positions of the full-precision vertical-line tokens, drawn without replacement
    from the non-window prefix [0, fp4_len)."""
    fp4_len = w.fp4_len if fp4_len is None else fp4_len
    n_hp = w.n_hp if n_hp is None else n_hp
    return np.sort(generator(w.wid, STREAM_SEL, 3, b, h).choice(fp4_len, size=n_hp, replace=False))


def decode_block_table(w: DecodeWorkload, n_pages: int | None = None) -> np.ndarray:
    """[B, n_pages] int32: logical page -> physical page in a shuffled pool of B*n_pages pages."""
    n_pages = w.n_pages if n_pages is None else n_pages
    perm = generator(w.wid, STREAM_SEL, 4).permutation(w.B * n_pages).astype(np.int32)
    return perm.reshape(w.B, n_pages)

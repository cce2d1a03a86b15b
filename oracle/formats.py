"""4-bit microscaling formats: element and scale codecs, block quantisation.

Test infrastructure (see the package header): never called by the CUDA path.

Sources
-------
* BitDecoding-FP4 (Algorithm-System Co-Design for Native FP4 KV Cache
  Decoding), section "The KV Cache Bottleneck in Long-Context LLM Serving":
  microscaling groups a tensor into fixed-size blocks that share one scale;
  elements are E2M1; MX blocks are 32 elements with an E8M0 scale; NVFP4 and
  MXFP4 differ in block size and scale format.  Section "Underflow-Aware
  Probability Scaling" names E4M3 scales (NVFP4).  NVFP4 blocks are 16
  elements with an unsigned E4M3 scale and an optional second-level FP32
  tensor scale g.
* MXAttention (Data-Free Optimal Scaling and Pre-Normalization Quantization for
  MXFP4 Attention), Abstract: power-of-two scaling, the OCP MXFP4 baseline and
  the universal optimal scaling bound Qmax = 7.25 (UOS).
* HiFA4, Abstract: Smooth-QK is a static per-channel rescaling of Q and K; it
  enters the quantiser as one FP32 multiply before the block maximum.

Readings where the pages are silent (each is listed in the design doc):
* E2M1 rounding is round-to-nearest-even on the grid {0,.5,1,1.5,2,3,4,6},
  saturating at 6; the sign bit is kept, so -0 encodes as 0x8.
* Packing: element 2i goes to the low nibble of byte i.
* UE4M3: OCP E4M3 without sign (bias 7, subnormals down to 2^-9, max 448),
  round-to-nearest-even, saturating at 448.
* UE8M0: byte b means 2^(b-127); the exponent is clamped to [-127, 127], so an
  all-zero block gets byte 0.
* NVFP4 scale: t = amax / (qmax*g) in FP32 (product first, one division),
  s = UE4M3(t); scaled element y = x / (float(s)*g) in FP32; a block whose
  scale encodes to zero has all its scaled elements taken as signed zeros.
* MXFP4 scale, OCP rule: e = floor(log2 amax) - 2.  UOS rule with bound qmax:
  the smallest e with amax <= qmax * 2^e.  y = x * 2^-e (exact).
"""
from __future__ import annotations

import numpy as np

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
NVFP4_BLOCK = 16
MXFP4_BLOCK = 32
UE4M3_MAX = 448.0


def block_size(fmt: str) -> int:
    return {"nvfp4": NVFP4_BLOCK, "mxfp4": MXFP4_BLOCK}[fmt]


# ----------------------------------------------------------------------------
# E2M1 element
# ----------------------------------------------------------------------------
def e2m1_encode(y) -> np.ndarray:
    """4-bit codes of already-scaled values y: sign bit 3, magnitude code 0..7.

    Round to nearest on the E2M1 grid, ties to the even code, saturating at 6
    (threshold form: each grid midpoint either belongs to the lower code, when
    the lower code is even, or to the upper one)."""
    y = np.asarray(y)
    a = np.abs(y)
    mag = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
           + (a > 2.5) + (a >= 3.5) + (a > 5.0)).astype(np.uint8)
    return (mag | (np.signbit(y).astype(np.uint8) << 3)).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    v = E2M1_VALUES[code & 7]
    return np.where(code & 8, -v, v)


# ----------------------------------------------------------------------------
# UE4M3 scale (NVFP4)
# ----------------------------------------------------------------------------
def ue4m3_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64) & 0x7F
    e = code >> 3
    m = code & 7
    sub = m * 2.0 ** -9
    nor = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    return np.where(e == 0, sub, nor)


def _rne(x: np.ndarray) -> np.ndarray:
    """Round half to even (numpy's rint does exactly this)."""
    return np.rint(x)


def ue4m3_encode(t) -> np.ndarray:
    """Unsigned E4M3 code of t >= 0: round to nearest even, saturate to 448 (0x7E)."""
    t = np.asarray(t, dtype=np.float64)
    out = np.zeros(t.shape, dtype=np.uint8)
    sat = t >= UE4M3_MAX
    sub = t < 2.0 ** -6
    # subnormal range: multiples of 2^-9; k = 8 lands exactly on the first normal (code 8)
    k = _rne(t * 2.0 ** 9)
    out = np.where(sub, k, out)
    nm = ~sub & ~sat
    mant, ex = np.frexp(np.where(nm, t, 1.0))       # t = mant * 2^ex, mant in [0.5, 1)
    E = ex - 1                                      # t = (2*mant) * 2^E, 2*mant in [1, 2)
    q = _rne((2.0 * mant - 1.0) * 8.0)
    carry = q == 8
    E = np.where(carry, E + 1, E)
    q = np.where(carry, 0, q)
    code_n = (E + 7) * 8 + q
    out = np.where(nm, code_n, out)
    out = np.where(sat, 0x7E, out)
    return np.minimum(out, 0x7E).astype(np.uint8)


# ----------------------------------------------------------------------------
# UE8M0 scale (MXFP4)
# ----------------------------------------------------------------------------
def ue8m0_decode(b) -> np.ndarray:
    return np.exp2(np.asarray(b, dtype=np.float64) - 127.0)


def mx_exponent(amax, qmax: float = 0.0) -> np.ndarray:
    """Shared power-of-two exponent e of MX blocks with block maxima amax (FP32 values).

    qmax == 0 -> OCP rule, e = floor(log2 amax) - 2.
    qmax  > 0 -> UOS rule, the smallest e with amax <= qmax * 2^e, decided by
                 exact comparison against ldexp(qmax, e).
    The result is clamped to [-127, 127]; amax == 0 gives -127."""
    amax = np.asarray(amax, dtype=np.float64)
    pos = amax > 0
    safe = np.where(pos, amax, 1.0)
    _, ex = np.frexp(safe)
    flog2 = ex - 1                                   # floor(log2 amax), exact
    if qmax == 0.0:
        e = flog2 - 2
    else:
        _, eq = np.frexp(qmax)
        e = flog2 - (eq - 1)                         # first guess, then settle by exact compares
        for _ in range(3):
            too_small = np.ldexp(qmax, e) < safe
            e = np.where(too_small, e + 1, e)
        for _ in range(3):
            can_lower = np.ldexp(qmax, e - 1) >= safe
            e = np.where(can_lower, e - 1, e)
    e = np.where(pos, e, -127)
    return np.clip(e, -127, 127).astype(np.int64)


# ----------------------------------------------------------------------------
# block quantisation
# ----------------------------------------------------------------------------
def quantize_blocks(x, fmt: str, qmax: float = 0.0, g: float = 1.0):
    """Quantise x[..., nblk, blk] (FP32 values), one scale per last-axis block.

    Returns (codes uint8 [..., nblk, blk], scale bytes uint8 [..., nblk]).
    NVFP4 follows the two-level rule with FP32 tensor scale g (qmax 0 -> 6);
    MXFP4 the OCP rule (qmax 0) or the UOS rule (qmax > 0)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    if fmt == "nvfp4":
        q = np.float32(6.0 if qmax == 0.0 else qmax)
        denom = np.float32(q * np.float32(g))                     # FP32 product first
        t = (amax / denom).astype(np.float32)                     # one FP32 division
        s = ue4m3_encode(t)
        sf = ue4m3_decode(s).astype(np.float32)
        div = (sf * np.float32(g)).astype(np.float32)[..., None]  # FP32 product
        with np.errstate(divide="ignore", invalid="ignore"):
            y = np.where(div > 0, x / np.where(div > 0, div, np.float32(1.0)), x * np.float32(0.0))
        return e2m1_encode(y.astype(np.float32)), s
    if fmt == "mxfp4":
        e = mx_exponent(amax, qmax)
        y = np.ldexp(x.astype(np.float64), -e[..., None])         # exact power-of-two scaling
        return e2m1_encode(y), (e + 127).astype(np.uint8)
    raise ValueError(fmt)


def dequantize_blocks(codes, sbytes, fmt: str, g: float = 1.0) -> np.ndarray:
    """FP64 values code * scale (* g for NVFP4)."""
    v = e2m1_decode(codes)
    if fmt == "nvfp4":
        return v * (ue4m3_decode(sbytes) * np.float64(np.float32(g)))[..., None]
    return v * ue8m0_decode(sbytes)[..., None]


def pack_nibbles(codes) -> np.ndarray:
    """[..., n] codes -> [..., n/2] bytes; element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


# ----------------------------------------------------------------------------
# tensor quantisation (the library's quantize call, canonical row-major layout)
# ----------------------------------------------------------------------------
def quantize_rows(x, fmt: str, qmax: float = 0.0, g: float = 1.0, mul=None):
    """Blocks along the last (contiguous) axis: x [..., cols] -> (packed [..., cols/2],
    scales [..., cols/blk]).  `mul` (broadcastable to x) is the Smooth-QK multiplier,
    applied as one FP32 multiply before the block maximum.  cols % blk == 0."""
    x = np.asarray(x, dtype=np.float32)
    if mul is not None:
        x = (x * np.asarray(mul, dtype=np.float32)).astype(np.float32)
    blk = block_size(fmt)
    cols = x.shape[-1]
    assert cols % blk == 0
    codes, s = quantize_blocks(x.reshape(x.shape[:-1] + (cols // blk, blk)), fmt, qmax, g)
    return pack_nibbles(codes.reshape(x.shape)), s


def quantize_cols_transposed(x, fmt: str, qmax: float = 0.0, g: float = 1.0):
    """Blocks along the token axis (-2) of x [..., S, d]; output transposed:
    (packed [..., d, S_pad/2], scales [..., d, S_pad/blk]) with S_pad = S rounded up
    to a multiple of 32 and zero tokens in the padding (zeros never raise a block maximum)."""
    x = np.asarray(x, dtype=np.float32)
    S = x.shape[-2]
    S_pad = -(-S // 32) * 32
    xt = np.swapaxes(x, -1, -2)
    if S_pad != S:
        pad = np.zeros(xt.shape[:-1] + (S_pad - S,), dtype=np.float32)
        xt = np.concatenate([xt, pad], axis=-1)
    return quantize_rows(np.ascontiguousarray(xt), fmt, qmax, g)


def dequantize_rows(packed, scales, fmt: str, g: float = 1.0) -> np.ndarray:
    codes = unpack_nibbles(packed)
    blk = block_size(fmt)
    cols = codes.shape[-1]
    v = dequantize_blocks(codes.reshape(codes.shape[:-1] + (cols // blk, blk)), scales, fmt, g)
    return v.reshape(codes.shape)

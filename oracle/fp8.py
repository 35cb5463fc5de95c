"""E4M3 encoding and per-block FP8 quantisation, written from the definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source for the quantised path: "Speed Up Image Generation with FLUX 3 Image
Klein on NVIDIA Blackwell GPUs", section "Quantized and sparse attention"
(FP8 query/key and FP8 value attention, ``qk_dtype: fp8``, ``v_dtype: fp8``).
The page fixes neither the FP8 format details nor the scale granularity; the
workload definitions fix e4m3 with one scale per (head, 128-token block).

E4M3 (OCP 8-bit floating point, "E4M3" encoding): 1 sign bit, 4 exponent bits
with bias 7, 3 mantissa bits.  Normal values (-1)^s 2^(E-7) (1 + M/8) for
E = 1..15 except E = 15, M = 7 which is NaN; subnormals (-1)^s 2^-6 (M/8) for
E = 0.  No infinities.  Largest finite value 448, smallest normal 2^-6,
smallest subnormal 2^-9.

Quantiser arithmetic (a reading; the page is silent), all in IEEE binary32:
  amax  = max |x| over the block,
  scale = RN(amax / 448),  inv = RN(448 / amax)   (scale = inv = 1 if amax == 0),
  code  = e4m3_satfinite_RNE(RN(x * inv)).
Dequantised value = decode(code) * scale.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_MIN_SUBNORMAL = 2.0 ** -9
BLOCK = 128


def e4m3_decode(codes) -> np.ndarray:
    """float64 value of every e4m3 code (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    val = np.where(E == 0, np.ldexp(M / 8.0, -6), np.ldexp(1.0 + M / 8.0, E - 7))
    val = np.where((E == 15) & (M == 7), np.nan, val)
    return sign * val


def e4m3_encode(x) -> np.ndarray:
    """Round to nearest, ties to even, saturating to +-448 (no NaN inputs).

    Works on the exact value of ``x`` (any float array): the step sizes are
    powers of two, so the scaled mantissa is exact in float64 and ``np.rint``
    (round half to even) gives the RNE decision.
    """
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, ex = np.frexp(a)                       # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                # unbiased exponent, clamped at the subnormal range
    q = np.rint(np.ldexp(a, 3 - e))           # a / 2^(e-3): 8..15.x (normal) or 0..8 (subnormal)
    # q in [8, 16] for normals (16 = carry into the next binade), [0, 8] in the subnormal range.
    carry = q >= 16
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 8, q)
    sub = q < 8                               # only possible when e == -6
    code = np.where(sub, q, ((e + 7) << 3) | (q.astype(np.int64) - 8)).astype(np.int64)
    code = np.where(a == 0, 0, code)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def block_scales(amax: np.ndarray):
    """(scale, inv) in float32 from a float32 block maximum (binary32 RN division;
    float64 division rounded once to float32 is correctly rounded)."""
    amax = np.asarray(amax, dtype=np.float32).astype(np.float64)
    zero = amax == 0
    safe = np.where(zero, 1.0, amax)
    scale = np.where(zero, 1.0, (safe / E4M3_MAX)).astype(np.float32)
    inv = np.where(zero, 1.0, (E4M3_MAX / safe)).astype(np.float32)
    return scale, inv


def quantize_blocks(x, block: int = BLOCK):
    """Per-(b, h, token-block) e4m3 quantisation of float32 ``x [B, H, S, d]``.

    Returns (codes uint8 [B, H, S, d], scale float32 [B, H, ceil(S/block)]).
    """
    x = np.asarray(x, dtype=np.float32)
    B, H, S, d = x.shape
    nblk = -(-S // block)
    pad = nblk * block - S
    xp = np.pad(x, ((0, 0), (0, 0), (0, pad), (0, 0))).reshape(B, H, nblk, block, d)
    amax = np.abs(xp).max(axis=(3, 4))
    scale, inv = block_scales(amax)
    y = (xp.astype(np.float64) * inv.astype(np.float64)[..., None, None]).astype(np.float32)
    codes = e4m3_encode(y).reshape(B, H, nblk * block, d)[:, :, :S]
    return codes, scale


def dequantize_blocks(codes, scale, block: int = BLOCK) -> np.ndarray:
    """float64 ``decode(code) * scale`` of ``codes [B, H, S, d]``."""
    codes = np.asarray(codes)
    S = codes.shape[2]
    s = np.repeat(np.asarray(scale, dtype=np.float64), block, axis=2)[:, :, :S, None]
    return e4m3_decode(codes) * s


def rounding_ambiguous(y, rel: float = 2.0 ** -20) -> np.ndarray:
    """True where ``y`` (the value about to be encoded) lies within a relative
    ``rel`` of an e4m3 rounding midpoint, so that a last-bit difference in
    the arithmetic before the encoder may legitimately flip the code."""
    y = np.abs(np.asarray(y, dtype=np.float64))
    a = np.minimum(y, E4M3_MAX)
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, -6)
    t = np.ldexp(a, 3 - e)
    frac = t - np.floor(t)
    tol = np.maximum(np.ldexp(rel * a, 3 - e), 2.0 ** -40)
    return (np.abs(frac - 0.5) <= tol) & (y < E4M3_MAX)

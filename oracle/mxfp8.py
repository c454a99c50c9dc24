"""Bit-exact MXFP8 block quantiser and exact dequantiser (oracle; test
infrastructure only).

What the pages fix: FLAMIA ("FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel
Olarak Güvenli Eğitim İçin Flash Mikro-Ölçeklemeli Dikkat Mekanizması",
section "FLAMIA Mimarisi ve Temel Tasarım İlkeleri") runs attention on MXFP8
operands with scales that must never let a future token influence the past,
and quantises inside fused kernels; FlashAttention-3 ("FlashAttention,
pelatihan multi-GPU, dan kuantisasi bobot", section 1) scales small blocks
independently to contain outliers.  The block geometry is the workload's:
one shared scale per 32 contiguous head-dim elements of one token and one
head, so no scale ever covers two tokens (hence never a document or causal
boundary).

What the pages leave open, and the reading taken here:
  * element format E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; exponent field 0 encodes subnormals m * 2^-9; code 0x7F / 0xFF is
    NaN; largest finite magnitude 448);
  * scale format E8M0: code c stands for 2^(c - 127);
  * scale rule: X is the smallest integer with amax <= 448 * 2^X, so no
    element of the block is clipped; the code is X + 127 clamped to
    [0, 254]; a block of zeros gets code 127 (scale 1);
  * element rule: x * 2^-(code - 127), rounded to the nearest E4M3 value with
    ties to the even code, magnitudes past 448 saturating to 448, the sign
    kept (a negative value that rounds to zero becomes 0x80);
  * inputs are finite.
"""
from __future__ import annotations

import numpy as np

__all__ = ["E4M3_MAX", "e4m3_decode_table", "e4m3_encode", "e8m0_scale_codes",
           "quantize_mxfp8_ref", "dequantize_mxfp8_ref", "BLOCK"]

BLOCK = 32
E4M3_MAX = 448.0


def e4m3_decode_table() -> np.ndarray:
    """Value of every E4M3 code 0..255 (NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * m * 2.0 ** -9
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_POS = e4m3_decode_table()[:0x7F]          # codes 0..126, increasing values


def e4m3_encode(y) -> np.ndarray:
    """Round fp64 values to E4M3 codes: nearest, ties to the even code,
    saturating at 448, sign kept."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    hi = np.searchsorted(_POS, a, side="left")          # _POS[hi-1] < a <= _POS[hi]
    hi = np.clip(hi, 0, len(_POS) - 1)
    lo = np.clip(hi - 1, 0, len(_POS) - 1)
    d_hi = np.abs(_POS[hi] - a)
    d_lo = np.abs(a - _POS[lo])
    take_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(take_lo, lo, hi)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    neg = np.signbit(y)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def e8m0_scale_codes(amax) -> np.ndarray:
    """E8M0 code of each block: X = min integer with amax <= 448 * 2^X,
    code = clamp(X + 127, 0, 254); amax == 0 gives 127."""
    amax = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(amax)                        # amax = f * 2^e, f in [0.5, 1)
    x = e.astype(np.int64) - 9                   # 448 * 2^(e-9) = 0.875 * 2^e
    x = np.where(amax > E4M3_MAX * np.ldexp(1.0, x), x + 1, x)
    x = np.where(amax == 0.0, 0, x)
    return np.clip(x + 127, 0, 254).astype(np.uint8)


def quantize_mxfp8_ref(x):
    """Quantise ``x`` (finite values, last dimension a multiple of 32) to
    E4M3 element codes with one E8M0 scale code per 32 contiguous elements
    of the last dimension.

    Returns (codes uint8, same shape as x; scales uint8, shape [..., n/32]).
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    assert n % BLOCK == 0, "last dimension must be a multiple of 32"
    blocks = x.reshape(x.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    sc = e8m0_scale_codes(amax)
    step = np.ldexp(1.0, -(sc.astype(np.int64) - 127))[..., None]
    codes = e4m3_encode(blocks * step)
    return codes.reshape(x.shape), sc


def dequantize_mxfp8_ref(codes, scales):
    """Exact value of every element: E4M3 value * 2^(scale code - 127), fp64."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    n = codes.shape[-1]
    vals = e4m3_decode_table()[codes.astype(np.int64)]
    blocks = vals.reshape(codes.shape[:-1] + (n // BLOCK, BLOCK))
    mult = np.ldexp(1.0, scales.astype(np.int64) - 127)[..., None]
    return (blocks * mult).reshape(codes.shape)

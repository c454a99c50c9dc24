"""NVFP4 block quantiser and exact dequantiser (oracle; test infrastructure
only).

What the pages fix: FLAMIA ("FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel
Olarak Güvenli Eğitim İçin Flash Mikro-Ölçeklemeli Dikkat Mekanizması",
section "FLAMIA Mimarisi ve Temel Tasarım İlkeleri") offers a mixed
NVFP4/FP8 path besides MXFP8, with scales that must never carry information
from future tokens to past ones and with document-local scaling.

What the pages leave open, and the reading taken here:
  * element format E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit;
    magnitudes 0, 0.5 (exponent field 0), 1, 1.5, 2, 3, 4, 6; no infinity or
    NaN; code = sign << 3 | magnitude index;
  * one scale per 16 contiguous head-dim elements of one token and one head,
    an unsigned E4M3 value (the E4M3 decode table's positive finite codes);
    no per-tensor scale: one computed over the whole tensor would make every
    token's quantisation depend on future tokens;
  * scale rule: S = the smallest E4M3 value with amax <= 6 S (no element
    clipped while amax <= 6 * 448); S = 448 beyond that (elements then
    saturate at 6); a block of zeros gets S = 1;
  * element rule: the fp32 quotient fp32(x / S) (an IEEE division, rounded
    to nearest), rounded to the nearest E2M1 value, ties to the even code
    (mantissa bit 0), magnitudes past 6 saturating to 6, the sign kept (a
    negative value that rounds to zero keeps its sign bit);
  * dequantised value: E2M1 value times S, exact in bf16 (a 2-bit times a
    4-bit significand).
  * the mixed path (``ref_attention_nvfp4_mxfp8``): Q and K in NVFP4 for the
    score product, V in MXFP8 (exactly dequantised, as the MXFP8 path).
"""
from __future__ import annotations

import numpy as np

from .attention import ref_attention
from .mxfp8 import dequantize_mxfp8_ref, e4m3_decode_table, quantize_mxfp8_ref

__all__ = ["NV_BLOCK", "E2M1_MAX", "e2m1_decode_table", "e2m1_encode", "nvfp4_scale_codes",
           "quantize_nvfp4_ref", "dequantize_nvfp4_ref", "ref_attention_nvfp4_mxfp8"]

NV_BLOCK = 16
E2M1_MAX = 6.0
_E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E4M3 = e4m3_decode_table()
_E4M3_POS_CODES = np.arange(1, 0x7F)               # positive finite E4M3 codes 1..126
_E4M3_POS = _E4M3[_E4M3_POS_CODES]                  # increasing


def e2m1_decode_table() -> np.ndarray:
    """Value of every E2M1 code 0..15."""
    return np.concatenate([_E2M1_POS, -_E2M1_POS])


def e2m1_encode(y) -> np.ndarray:
    """Round values to E2M1 codes: nearest, ties to the even code,
    saturating at 6, sign kept."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    hi = np.clip(np.searchsorted(_E2M1_POS, a, side="left"), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    d_hi = np.abs(_E2M1_POS[hi] - a)
    d_lo = np.abs(a - _E2M1_POS[lo])
    take_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(take_lo, lo, hi)
    code = np.where(a >= E2M1_MAX, 7, code)
    return (code | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def nvfp4_scale_codes(amax) -> np.ndarray:
    """E4M3 scale code per block from the block's largest magnitude."""
    amax = np.asarray(amax, dtype=np.float64)
    need = amax / E2M1_MAX
    idx = np.searchsorted(_E4M3_POS, need, side="left")   # first value >= need
    idx = np.clip(idx, 0, len(_E4M3_POS) - 1)             # past 448: 448
    code = _E4M3_POS_CODES[idx]
    code = np.where(amax == 0.0, 0x38, code)              # E4M3 0x38 = 1.0
    return code.astype(np.uint8)


def quantize_nvfp4_ref(x):
    """x: [..., C] with C % 16 == 0.  Returns (codes uint8 [..., C] (E2M1,
    one per byte), scales uint8 [..., C / 16] (E4M3))."""
    x = np.asarray(x, dtype=np.float64)
    if x.shape[-1] % NV_BLOCK:
        raise ValueError("last dimension must be a multiple of 16")
    blocks = x.reshape(x.shape[:-1] + (x.shape[-1] // NV_BLOCK, NV_BLOCK))
    scodes = nvfp4_scale_codes(np.abs(blocks).max(axis=-1))
    s = _E4M3[scodes].astype(np.float32)
    q = (blocks.astype(np.float32) / s[..., None]).astype(np.float32)   # IEEE fp32 division
    codes = e2m1_encode(q).reshape(x.shape)
    return codes, scodes


def dequantize_nvfp4_ref(codes, scales) -> np.ndarray:
    codes = np.asarray(codes)
    vals = e2m1_decode_table()[codes]
    blocks = vals.reshape(vals.shape[:-1] + (vals.shape[-1] // NV_BLOCK, NV_BLOCK))
    return (blocks * _E4M3[np.asarray(scales)][..., None]).reshape(vals.shape)


def ref_attention_nvfp4_mxfp8(q, k, v, cu_seqlens, causal: bool, scale: float):
    """Attention of the mixed path: Q, K quantised to NVFP4 and V to MXFP8,
    all exactly dequantised, then the fp64 attention.  (out, lse)."""
    qd = dequantize_nvfp4_ref(*quantize_nvfp4_ref(q))
    kd = dequantize_nvfp4_ref(*quantize_nvfp4_ref(k))
    vd = dequantize_mxfp8_ref(*quantize_mxfp8_ref(np.asarray(v, dtype=np.float64)))
    return ref_attention(qd, kd, vd, cu_seqlens, causal, scale)

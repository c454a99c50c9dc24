"""Incoherent processing of Q and K before MXFP8 quantisation (oracle; test
infrastructure only).

What the pages fix: "FlashAttention, pelatihan multi-GPU, dan kuantisasi
bobot", section 1 (FlashAttention-3's FP8 support): so that outlier
activations do not cost FP8 precision, Q and K are multiplied by a random
orthogonal matrix before they are quantised, which spreads extreme values
over the head dimension.  Because the matrix is orthogonal the scores are
unchanged in exact arithmetic: (Q M)(K M)^T = Q M M^T K^T = Q K^T.

What the pages leave open, and the reading taken here:
  * the construction: M = diag(s) H_d, with H_d the Sylvester Hadamard
    matrix (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]; entries +-1,
    H_d H_d^T = d I) and s a vector of d random signs drawn by the caller
    from its seeded generator and passed in; one draw per call, the same M
    for every token and head, applied to Q and K, never to V;
  * normalisation: M is used unnormalised, so M M^T = d I and the scores
    come out multiplied by d; the softmax scale is divided by d instead
    (exact: d is a power of two).  That keeps the rotation free of a
    rounded 1/sqrt(d) factor;
  * precision: the rotated rows are computed in fp32 by the fast
    Walsh-Hadamard butterfly in a fixed order (span h = 1, 2, 4, ..., d/2;
    each pair (a, b) at distance h becomes (a + b, a - b), round to nearest),
    the sign flips first (exact).  A kernel that quantises the rotated rows
    takes its E4M3 rounding decisions on these same fp32 values, so its codes
    can be compared bit for bit with the oracle quantiser's.
"""
from __future__ import annotations

import numpy as np

from .attention import ref_attention
from .mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref

__all__ = ["hadamard", "incoherent_matrix", "rotate_fp64", "rotate_fp32",
           "incoherent_operands", "ref_attention_incoherent_mxfp8"]


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order d (a power of two), fp64 +-1."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def incoherent_matrix(signs) -> np.ndarray:
    """M = diag(signs) H_d (unnormalised: M M^T = d I)."""
    s = np.asarray(signs, dtype=np.float64)
    return s[:, None] * hadamard(s.shape[0])


def rotate_fp64(x, signs) -> np.ndarray:
    """x M along the last axis, by the matrix product in fp64 (the plain
    definition)."""
    return np.asarray(x, dtype=np.float64) @ incoherent_matrix(signs)


def rotate_fp32(x, signs) -> np.ndarray:
    """x M along the last axis in fp32, by the butterfly in the fixed order
    stated in the module docstring (the values a quantising kernel rounds)."""
    s = np.asarray(signs, dtype=np.float32)
    y = np.asarray(x, dtype=np.float32) * s          # sign flips: exact
    d = y.shape[-1]
    h = 1
    while h < d:
        blocks = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a = blocks[..., 0, :]
        b = blocks[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(y.shape)   # fp32 adds, RNE
        h *= 2
    return y


def incoherent_operands(q, k, v, scale: float, signs):
    """The operands the attention sees under incoherent processing: Q and K
    rotated (fp32, as above), the three quantised and exactly dequantised by
    the oracle quantiser, and the softmax scale divided by d.  Returns
    (qd, kd, vd, scale / d)."""
    d = np.asarray(q).shape[-1]
    qd = dequantize_mxfp8_ref(*quantize_mxfp8_ref(rotate_fp32(q, signs)))
    kd = dequantize_mxfp8_ref(*quantize_mxfp8_ref(rotate_fp32(k, signs)))
    vd = dequantize_mxfp8_ref(*quantize_mxfp8_ref(np.asarray(v, dtype=np.float64)))
    return qd, kd, vd, scale / d


def ref_attention_incoherent_mxfp8(q, k, v, cu_seqlens, causal: bool, scale: float, signs):
    """Attention on MXFP8 operands with incoherent processing: the fp64
    attention of ``incoherent_operands``.  Returns (out, lse) like
    ``ref_attention``."""
    qd, kd, vd, s = incoherent_operands(q, k, v, scale, signs)
    return ref_attention(qd, kd, vd, cu_seqlens, causal, s)

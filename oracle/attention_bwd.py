"""fp64 reference gradients of exact attention (oracle; test infrastructure
only).

The pages measure the attention forward and backward together (FLAMIA,
"FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin
Flash Mikro-Ölçeklemeli Dikkat Mekanizması", section "Performans
Sonuçları"; "FlashAttention và IO" notes that a forward-only measurement
says little about training) but print no backward formulas.  The gradients
are therefore the plain derivatives of the forward definition the forward
oracle writes out (``oracle.attention``): per document and head, with
S = scale Q K^T (masked), P = row-softmax(S), O = P V and an upstream
gradient dO of the output,

    dV = P^T dO
    dP = dO V^T
    D_i = sum_j P_ij dP_ij  (= dO_i . O_i)
    dS = P * (dP - D)          (elementwise, D broadcast along each row)
    dQ = scale dS K
    dK = scale dS^T Q

computed on the full masked matrices in fp64.  Masked entries have P = 0
and so contribute nothing; a row that sees no key has P = 0 and all its
gradients are 0.

Layouts as the forward oracle: q, k, v, dout and the results are [T, H, d].

MXFP8 (``ref_attention_bwd_mxfp8``).  FLAMIA (section "FLAMIA Mimarisi ve
Temel Tasarım İlkeleri") asks for the forward and backward passes to agree
numerically, for quantised operands reused across orientations, and for
scales that carry no information from future tokens.  Reading taken: the
backward differentiates exactly what the MXFP8 forward computed, so it runs
on the same quantised operands: Q, K, V quantised per (token, head, 32
head-dim elements) and exactly dequantised, as in the forward oracle; the
upstream gradient dO quantised the same way; gradients with respect to the
dequantised operands, passed straight through the quantiser.  Every scale
covers one token of one head, so none crosses a document or causal
boundary, and the dequantised values serve every orientation of every
product unchanged.
"""
from __future__ import annotations

import numpy as np

from .attention import doc_bounds, ref_probabilities
from .mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref

__all__ = ["ref_attention_bwd", "ref_attention_bwd_mxfp8"]


def ref_attention_bwd(q, k, v, dout, cu_seqlens, causal: bool, scale: float):
    """(dq, dk, dv), each fp64 [T, H, d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    H = q.shape[1]
    for a, b in doc_bounds(cu_seqlens):
        if b <= a:
            continue
        for h in range(H):
            qh, kh, vh, doh = q[a:b, h], k[a:b, h], v[a:b, h], dout[a:b, h]
            p = ref_probabilities(qh, kh, scale, causal)          # [L, L]
            o = p @ vh
            dv[a:b, h] = p.T @ doh
            dp = doh @ vh.T
            dd = np.sum(doh * o, axis=1, keepdims=True)
            ds = p * (dp - dd)
            dq[a:b, h] = scale * (ds @ kh)
            dk[a:b, h] = scale * (ds.T @ qh)
    return dq, dk, dv


def ref_attention_bwd_mxfp8(q, k, v, dout, cu_seqlens, causal: bool, scale: float):
    """(dq, dk, dv) of the MXFP8 path, fp64 [T, H, d]: the gradients above
    on the exactly dequantised MXFP8 operands (q, k, v and dout quantised
    per token, head and 32 head-dim elements)."""
    def deq(x):
        return dequantize_mxfp8_ref(*quantize_mxfp8_ref(np.asarray(x, dtype=np.float64)))

    return ref_attention_bwd(deq(q), deq(k), deq(v), deq(dout), cu_seqlens, causal, scale)

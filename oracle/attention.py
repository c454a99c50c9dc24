"""fp64 reference attention (oracle; test infrastructure only).

What is computed, per "FlashAttention và IO" (aihero.vn):
  * section "Ma trận trung gian là một khoản chi phí": dense attention forms
    the full n x n score matrix of one head, applies softmax and multiplies
    by V.  ``ref_attention`` does exactly that, one (document, head) at a
    time, on fp64 copies of the inputs.
  * section "Softmax qua nhiều khối cần thống kê chạy": the running maximum m,
    normaliser l and weighted sum u, with the old part multiplied by
    exp(m - m_new) when a block raises the maximum, and the result u / l.
    ``online_replay`` replays that recurrence literally, block by block, for
    one query row; it is used only to pin the worked example.

Readings where the pages are silent (each one is listed in the design notes):
  * the score is ``scale * q . k`` with the caller's ``scale`` (the pages write
    softmax(QK^T)V without a factor; the workloads pass 1/sqrt(d));
  * causal means key j is visible to query i iff j <= i, both counted from the
    start of their document; keys of other documents are never visible;
  * the per-row log-sum-exp is the natural log of the row's normaliser in
    scaled-score units: lse_i = max_j s_ij + ln sum_j exp(s_ij - max_j s_ij);
  * a row that sees no key (impossible for causal self-attention, kept for
    completeness) has output 0 and lse = -inf.

Layouts: q, k, v are [T, H, d] (token-major, heads, head dim); the output is
[T, H, d] and lse is [H, T].  ``cu_seqlens`` holds num_docs + 1 increasing
offsets starting at 0 and ending at T.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "doc_bounds",
    "visible_count",
    "score_matrix",
    "ref_probabilities",
    "ref_attention",
    "ref_attention_rows",
    "online_replay",
]


def doc_bounds(cu_seqlens) -> list[tuple[int, int]]:
    """Half-open token ranges [a, b) of the packed documents."""
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    return [(cu[i], cu[i + 1]) for i in range(len(cu) - 1)]


def _visible(L: int, causal: bool) -> np.ndarray:
    """Boolean L x L visibility inside one document (row = query, col = key)."""
    if causal:
        return np.tril(np.ones((L, L), dtype=bool))
    return np.ones((L, L), dtype=bool)


def visible_count(cu_seqlens, causal: bool) -> np.ndarray:
    """Number of keys each token's query sees, an int64 vector of length T."""
    bounds = doc_bounds(cu_seqlens)
    T = bounds[-1][1] if bounds else 0
    cnt = np.zeros(T, dtype=np.int64)
    for a, b in bounds:
        L = b - a
        cnt[a:b] = np.arange(1, L + 1) if causal else L
    return cnt


def score_matrix(q, k, scale: float, causal: bool) -> np.ndarray:
    """Masked scaled scores of one document and head: s_ij = scale * q_i . k_j,
    or -inf where key j is not visible to query i.  q: [L, d], k: [L, d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    s = np.float64(scale) * (q @ k.T)
    s[~_visible(q.shape[0], causal)] = -np.inf
    return s


def _softmax_rows(s: np.ndarray):
    """Row softmax of a masked score block; returns (P, lse).  Fully masked
    rows give P = 0 and lse = -inf."""
    m = s.max(axis=1)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(s - m_safe[:, None])
    e[~finite, :] = 0.0
    l = e.sum(axis=1)
    p = np.zeros_like(e)
    p[finite] = e[finite] / l[finite, None]
    lse = np.full(s.shape[0], -np.inf)
    lse[finite] = m[finite] + np.log(l[finite])
    return p, lse


def ref_probabilities(q, k, scale: float, causal: bool) -> np.ndarray:
    """The full probability matrix P = row-softmax(S) of one document and head."""
    p, _ = _softmax_rows(score_matrix(q, k, scale, causal))
    return p


def ref_attention(q, k, v, cu_seqlens, causal: bool, scale: float,
                  row_chunk: int = 2048):
    """Exact attention of every (document, head) by its definition.

    For each document and head the masked score matrix S is formed, turned
    into P by a row softmax, and O = P V.  For memory the rows of S are taken
    ``row_chunk`` at a time; each chunk holds whole rows, so the result is the
    same as forming S at once.  Inputs are converted to fp64 exactly.

    Returns (out [T, H, d] fp64, lse [H, T] fp64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, H, d = q.shape
    out = np.zeros((T, H, v.shape[2]), dtype=np.float64)
    lse = np.full((H, T), -np.inf, dtype=np.float64)
    for a, b in doc_bounds(cu_seqlens):
        L = b - a
        if L == 0:
            continue
        for h in range(H):
            kd = k[a:b, h, :]
            vd = v[a:b, h, :]
            for r0 in range(0, L, row_chunk):
                r1 = min(L, r0 + row_chunk)
                s = np.float64(scale) * (q[a + r0:a + r1, h, :] @ kd.T)
                if causal:
                    rows = np.arange(r0, r1)[:, None]
                    cols = np.arange(L)[None, :]
                    s[cols > rows] = -np.inf
                p, lse_rows = _softmax_rows(s)
                out[a + r0:a + r1, h, :] = p @ vd
                lse[h, a + r0:a + r1] = lse_rows
    return out, lse


def ref_attention_rows(q, k, v, cu_seqlens, causal: bool, scale: float,
                       tokens, heads):
    """Exact attention for selected (token, head) rows only, each computed on
    its own from the definition (scores against the visible keys of its
    document, softmax, weighted sum of values).  Used for sampled checks at
    sizes where the full oracle would take too long.

    Returns (out [n, d] fp64, lse [n] fp64) for the n requested rows.
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    tokens = np.asarray(tokens, dtype=np.int64).reshape(-1)
    heads = np.asarray(heads, dtype=np.int64).reshape(-1)
    n = tokens.shape[0]
    dv = v.shape[2]
    out = np.zeros((n, dv), dtype=np.float64)
    lse = np.full(n, -np.inf, dtype=np.float64)
    for r in range(n):
        t, h = int(tokens[r]), int(heads[r])
        doc = int(np.searchsorted(cu, t, side="right")) - 1
        a, b = int(cu[doc]), int(cu[doc + 1])
        hi = t + 1 if causal else b
        kk = np.asarray(k[a:hi, h, :], dtype=np.float64)
        vv = np.asarray(v[a:hi, h, :], dtype=np.float64)
        qq = np.asarray(q[t, h, :], dtype=np.float64)
        s = np.float64(scale) * (kk @ qq)
        if s.size == 0:
            continue
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        out[r] = (e / l) @ vv
        lse[r] = m + np.log(l)
    return out, lse


def online_replay(scores, values, blocks):
    """Replay the running-statistics recurrence for ONE query row.

    ``scores``: the row's scores s_j (already scaled), ``values``: the value
    rows v_j (shape [n] or [n, dv]), ``blocks``: a sequence of index lists,
    processed in the given order.  Starting from m = -inf, l = 0, u = 0, each
    block with maximum m_b does
        m_new = max(m, m_b)
        l     = l * exp(m - m_new) + sum_j exp(s_j - m_new)
        u     = u * exp(m - m_new) + sum_j exp(s_j - m_new) * v_j
        m     = m_new
    and the result is u / l ("FlashAttention và IO", section "Softmax qua
    nhiều khối cần thống kê chạy").

    Returns (result, trace) where trace lists (m, l, u) after every block.
    """
    s = np.asarray(scores, dtype=np.float64)
    vals = np.asarray(values, dtype=np.float64)
    m = -np.inf
    l = 0.0
    u = np.zeros(vals.shape[1:], dtype=np.float64)
    trace = []
    for blk in blocks:
        idx = np.asarray(list(blk), dtype=np.int64)
        sb = s[idx]
        m_new = max(m, float(sb.max()))
        shrink = np.exp(m - m_new) if np.isfinite(m) else 0.0
        w = np.exp(sb - m_new)
        l = l * shrink + float(w.sum())
        u = u * shrink + np.tensordot(w, vals[idx], axes=(0, 0))
        m = m_new
        trace.append((m, l, np.array(u, copy=True)))
    return u / l, trace

"""Pins of the fp64 attention oracle against things other than itself:
the pages' worked example, a library routine on special cases, 50-digit
brute force, closed forms and invariants.  CPU only."""
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.attention import (online_replay, ref_attention, ref_attention_rows,
                              ref_probabilities, score_matrix, visible_count,
                              doc_bounds)
from exact_tiled_attention_39_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _num(s: str) -> float:
    if s == "ln2":
        return math.log(2.0)
    return float(Fraction(s))


def _rand_pack(rng, lengths, H, d, scale_q=1.0):
    T = sum(lengths)
    q = rng.standard_normal((T, H, d)) * scale_q
    k = rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return q, k, v, cu


# ----------------------------------------------------------------- worked example
def test_worked_example_forward_trace():
    g = _golden()
    s = [_num(x) for x in g["scores"]]
    v = [_num(x) for x in g["values"]]
    res, trace = online_replay(s, v, [[0], [1]])
    assert abs(res - _num(g["result"])) <= 1e-15
    for got, want in zip(trace, g["trace_forward"]):
        m, l, u = got
        assert abs(m - _num(want["m"])) <= 1e-15
        assert abs(l - _num(want["l"])) <= 1e-15
        assert abs(float(u) - _num(want["u"])) <= 1e-15


def test_worked_example_reverse_order():
    g = _golden()
    s = [_num(x) for x in g["scores"]]
    v = [_num(x) for x in g["values"]]
    res, _ = online_replay(s, v, [[1], [0]])
    assert abs(res - _num(g["trace_reverse_result"])) <= 1e-15
    res1, _ = online_replay(s, v, [[0, 1]])
    assert abs(res1 - 7.0 / 3.0) <= 1e-15


def test_worked_example_weights_and_definition():
    """The same case through the full-matrix oracle: a 2-token document,
    q_1 = e_0, k_0 = 0, k_1 = e_0 and scale ln 2 give scores [0, ln 2] for
    row 1; V rows 1 and 3 give 7/3 and lse = ln 3."""
    g = _golden()
    d = 4
    q = np.zeros((2, 1, d)); q[1, 0, 0] = 1.0
    k = np.zeros((2, 1, d)); k[1, 0, 0] = 1.0
    v = np.zeros((2, 1, d)); v[0, 0, :] = 1.0; v[1, 0, :] = 3.0
    for causal in (False, True):
        out, lse = ref_attention(q, k, v, [0, 2], causal, math.log(2.0))
        np.testing.assert_allclose(out[1, 0], 7.0 / 3.0, rtol=0, atol=1e-15)
        assert abs(lse[0, 1] - math.log(3.0)) <= 1e-15
        p = ref_probabilities(q[:, 0], k[:, 0], math.log(2.0), causal)
        np.testing.assert_allclose(p[1], [_num(w) for w in g["weights"]], atol=1e-15)
    out, lse = ref_attention(q, k, v, [0, 2], True, math.log(2.0))
    np.testing.assert_allclose(out[0, 0], 1.0, atol=0)       # row 0 sees key 0 only
    assert lse[0, 0] == 0.0


# ----------------------------------------------------------------- invariants
def test_row_stochastic_and_masked_zero():
    rng = np.random.default_rng(5)
    for causal in (False, True):
        q = rng.standard_normal((37, 8)) * 3
        k = rng.standard_normal((37, 8)) * 3
        p = ref_probabilities(q, k, 0.3, causal)
        assert (p >= 0).all()
        assert np.abs(p.sum(axis=1) - 1.0).max() <= 1e-12
        if causal:
            assert (p[np.triu_indices(37, 1)] == 0.0).all()


def test_score_matrix_orientation():
    """s_ij = scale * q_i . k_j (row = query): a transposed product or a
    swapped mask fails this asymmetric case."""
    q = np.array([[1.0, 0.0], [0.0, 2.0], [1.0, 1.0]])
    k = np.array([[0.0, 1.0], [3.0, 0.0], [1.0, -1.0]])
    s = score_matrix(q, k, 0.5, causal=True)
    want = np.array([[0.0, -np.inf, -np.inf],
                     [1.0, 0.0, -np.inf],
                     [0.5, 1.5, 0.0]])
    np.testing.assert_array_equal(s, want)


def test_visible_count_by_hand():
    cu = [0, 3, 3, 5]
    np.testing.assert_array_equal(visible_count(cu, True), [1, 2, 3, 1, 2])
    np.testing.assert_array_equal(visible_count(cu, False), [3, 3, 3, 2, 2])
    assert doc_bounds(cu) == [(0, 3), (3, 3), (3, 5)]


# ----------------------------------------------------------------- library special case
def _sdpa_reference(q, k, v, cu, causal, scale):
    T, H, d = q.shape
    mask = torch.zeros((T, T), dtype=torch.bool)
    for a, b in doc_bounds(cu):
        blk = torch.ones((b - a, b - a), dtype=torch.bool)
        if causal:
            blk = torch.tril(blk)
        mask[a:b, a:b] = blk
    qt = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None]
    kt = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    vt = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=mask, scale=scale)
    return o[0].numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_tiny_workload(causal):
    inp = workloads.make_inputs("tiny")
    q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
    cu = inp["cu_seqlens"].numpy()
    out, _ = ref_attention(q, k, v, cu, causal, inp["scale"])
    want = _sdpa_reference(q, k, v, cu, causal, inp["scale"])
    assert np.abs(out - want).max() <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_small_packs(causal):
    rng = np.random.default_rng(11)
    for lengths in ([1, 7, 130, 3], [64, 0, 200], [257]):
        q, k, v, cu = _rand_pack(rng, lengths, 3, 16, scale_q=2.0)
        out, lse = ref_attention(q, k, v, cu, causal, 0.25, row_chunk=50)
        want = _sdpa_reference(q, k, v, cu, causal, 0.25)
        assert np.abs(out - want).max() <= 1e-12
        rows_t = np.arange(cu[-1]).repeat(3)
        rows_h = np.tile(np.arange(3), cu[-1])
        o2, l2 = ref_attention_rows(q, k, v, cu, causal, 0.25, rows_t, rows_h)
        assert np.abs(o2 - want[rows_t, rows_h]).max() <= 1e-12
        assert np.abs(l2 - lse[rows_h, rows_t]).max() <= 1e-12


# ----------------------------------------------------------------- brute force
def test_brute_force_50_digits():
    """Direct exp-sum at 50 significant digits, no max subtraction."""
    getcontext().prec = 50
    rng = np.random.default_rng(3)
    lengths = [5, 3]
    q, k, v, cu = _rand_pack(rng, lengths, 2, 3, scale_q=1.5)
    scale = 0.7
    for causal in (False, True):
        out, lse = ref_attention(q, k, v, cu, causal, scale)
        for a, b in doc_bounds(cu):
            for h in range(2):
                for i in range(a, b):
                    hi = i + 1 if causal else b
                    num = [Decimal(0)] * 3
                    den = Decimal(0)
                    for j in range(a, hi):
                        s = Decimal(scale) * sum(Decimal(float(q[i, h, c])) * Decimal(float(k[j, h, c]))
                                                 for c in range(3))
                        e = s.exp()
                        den += e
                        for c in range(3):
                            num[c] += e * Decimal(float(v[j, h, c]))
                    for c in range(3):
                        assert abs(float(num[c] / den) - out[i, h, c]) <= 1e-13
                    assert abs(float(den.ln()) - lse[h, i]) <= 1e-13


# ----------------------------------------------------------------- closed forms
def test_zero_queries_give_mean_and_log_count():
    rng = np.random.default_rng(1)
    lengths = [4, 1, 9]
    q, k, v, cu = _rand_pack(rng, lengths, 2, 5)
    q[:] = 0.0
    for causal in (False, True):
        out, lse = ref_attention(q, k, v, cu, causal, 0.9)
        cnt = visible_count(cu, causal)
        for a, b in doc_bounds(cu):
            for i in range(a, b):
                hi = i + 1 if causal else b
                np.testing.assert_allclose(out[i], v[a:hi].mean(axis=0), atol=1e-14)
        np.testing.assert_allclose(lse, np.log(cnt)[None, :].repeat(2, 0), atol=1e-14)


def test_constant_values_and_first_token():
    rng = np.random.default_rng(2)
    lengths = [6, 2, 11]
    q, k, v, cu = _rand_pack(rng, lengths, 2, 4, scale_q=3.0)
    vc = np.full_like(v, -1.25)
    out, _ = ref_attention(q, k, vc, cu, True, 0.5)
    np.testing.assert_allclose(out, -1.25, atol=1e-14)
    out, lse = ref_attention(q, k, v, cu, True, 0.5)
    for a, b in doc_bounds(cu):
        np.testing.assert_array_equal(out[a], v[a])
        for h in range(2):
            assert abs(lse[h, a] - 0.5 * float(q[a, h] @ k[a, h])) <= 1e-14


def test_key_shift_invariance():
    rng = np.random.default_rng(4)
    lengths = [13, 7]
    q, k, v, cu = _rand_pack(rng, lengths, 2, 6)
    w = rng.standard_normal(6)
    scale = 0.4
    for causal in (False, True):
        o1, l1 = ref_attention(q, k, v, cu, causal, scale)
        o2, l2 = ref_attention(q, k + w, v, cu, causal, scale)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        shift = scale * np.einsum("thd,d->ht", q, w)
        np.testing.assert_allclose(l2 - l1, shift, atol=1e-12)


def test_packing_order_invariance_exact():
    rng = np.random.default_rng(6)
    lengths = [5, 17, 1, 30]
    q, k, v, cu = _rand_pack(rng, lengths, 2, 8)
    out, lse = ref_attention(q, k, v, cu, True, 0.3)
    perm = [2, 0, 3, 1]
    bounds = doc_bounds(cu)
    idx = np.concatenate([np.arange(*bounds[p]) for p in perm])
    cu2 = np.concatenate([[0], np.cumsum([lengths[p] for p in perm])])
    out2, lse2 = ref_attention(q[idx], k[idx], v[idx], cu2, True, 0.3)
    np.testing.assert_array_equal(out2, out[idx])
    np.testing.assert_array_equal(lse2, lse[:, idx])


def test_row_chunking_does_not_change_result():
    rng = np.random.default_rng(8)
    q, k, v, cu = _rand_pack(rng, [300, 45], 2, 8)
    o1, l1 = ref_attention(q, k, v, cu, True, 0.3, row_chunk=7)
    o2, l2 = ref_attention(q, k, v, cu, True, 0.3, row_chunk=4096)
    np.testing.assert_allclose(o1, o2, atol=1e-15)
    np.testing.assert_allclose(l1, l2, atol=1e-15)


def test_online_replay_any_partition_and_order():
    """The running statistics reach the direct softmax-weighted sum for any
    partition of the keys into blocks and any block order (the recurrence's
    exactness claim), including blocks whose maximum is below the running
    one, a block holding the row maximum last, and scores far apart
    (exp(-100) weights); the final l is the direct sum of exp(s - max)."""
    rng = np.random.default_rng(23)
    for trial in range(40):
        n = int(rng.integers(1, 40))
        s = rng.normal(0.0, 3.0, n)
        if trial % 4 == 0:
            s[int(rng.integers(0, n))] += 100.0        # one dominant key
        v = rng.normal(size=(n, 5))
        perm = rng.permutation(n)
        cuts = np.sort(rng.choice(np.arange(1, n), size=min(n - 1, int(rng.integers(0, 6))),
                                  replace=False)) if n > 1 else []
        blocks = [list(b) for b in np.split(perm, cuts)]
        got, trace = online_replay(s, v, blocks)
        w = np.exp(s - s.max())
        want = (w[:, None] * v).sum(0) / w.sum()
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
        m_final, l_final, _ = trace[-1]
        assert m_final == s.max()
        np.testing.assert_allclose(l_final, w.sum(), rtol=1e-13)

"""Pins of the fp64 attention gradients (oracle/attention_bwd.py), checked
against things other than the oracle itself: autograd of a library routine
(torch's scaled-dot-product attention in fp64 with an explicit mask),
central finite differences of the forward oracle, exact identities, and the
gradient of the pages' worked example worked out by hand.  CPU only."""
import math

import numpy as np
import pytest
import torch

from oracle.attention import ref_attention
from oracle.attention_bwd import ref_attention_bwd

RAGGED = [1, 5, 0, 17, 33]


def _pack(lengths, H, d, seed):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    q, k, v, do = (rng.standard_normal((T, H, d)) for _ in range(4))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return q, k, v, do, cu


def _sdpa_grads(q, k, v, do, cu, causal, scale):
    """Autograd of torch SDPA (fp64) with a block-diagonal boolean mask."""
    T, H, d = q.shape
    mask = torch.zeros((T, T), dtype=torch.bool)
    for a, b in zip(cu[:-1], cu[1:]):
        blk = torch.ones((b - a, b - a), dtype=torch.bool)
        mask[a:b, a:b] = torch.tril(blk) if causal else blk
    tq, tk, tv = (torch.tensor(x.transpose(1, 0, 2), requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    o.backward(torch.tensor(do.transpose(1, 0, 2)))
    return tuple(t.grad.numpy().transpose(1, 0, 2) for t in (tq, tk, tv))


@pytest.mark.parametrize("causal", [False, True])
def test_matches_autograd_of_library_attention(causal):
    q, k, v, do, cu = _pack(RAGGED, 2, 8, seed=4)
    got = ref_attention_bwd(q, k, v, do, cu, causal, 0.3)
    want = _sdpa_grads(q, k, v, do, cu, causal, 0.3)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)


def test_central_finite_differences():
    """d/dx of L = sum(dO * O) for every input element of a tiny pack."""
    q, k, v, do, cu = _pack([4, 3], 1, 3, seed=9)
    scale = 0.7
    dq, dk, dv = ref_attention_bwd(q, k, v, do, cu, True, scale)

    def loss(q_, k_, v_):
        o, _ = ref_attention(q_, k_, v_, cu, True, scale)
        return float(np.sum(do * o))

    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            fp = loss(q, k, v)
            x[idx] = old - h
            fm = loss(q, k, v)
            x[idx] = old
            assert abs((fp - fm) / (2 * h) - g[idx]) <= 1e-7


def test_exact_identities():
    """Per document and head: the key gradients sum to zero (adding one vector
    to every key shifts each row's scores by a constant, which softmax
    ignores); the value gradients sum to the output gradients (each row of P
    sums to one); one-token documents pass dO straight to dV and have no
    query or key gradient."""
    q, k, v, do, cu = _pack([1, 9, 1, 40], 3, 5, seed=2)
    dq, dk, dv = ref_attention_bwd(q, k, v, do, cu, True, 0.41)
    for a, b in zip(cu[:-1], cu[1:]):
        np.testing.assert_allclose(dk[a:b].sum(axis=0), 0.0, atol=1e-12)
        np.testing.assert_allclose(dv[a:b].sum(axis=0), do[a:b].sum(axis=0), atol=1e-12)
        if b - a == 1:          # zero up to fp64 rounding of dO . v computed two ways
            np.testing.assert_allclose(dq[a:b], 0.0, atol=1e-12)
            np.testing.assert_allclose(dk[a:b], 0.0, atol=1e-12)
            np.testing.assert_allclose(dv[a:b], do[a:b], rtol=0, atol=1e-15)


def test_gradient_of_the_worked_example():
    """The worked example ("FlashAttention và IO", section "Softmax qua nhiều
    khối cần thống kê chạy": scores [0, ln 2], values [1, 3], result 7/3)
    with an upstream gradient of 1 on that row, by hand: weights (1/3, 2/3);
    dV = (1/3, 2/3); dP = (1, 3); D = 7/3; dS = P (dP - D) = (-4/9, 4/9);
    with q = e0, k0 = 0, k1 = e0 and scale ln 2: dq = ln2 (4/9) e0,
    dk0 = -ln2 (4/9) e0, dk1 = ln2 (4/9) e0."""
    d = 2
    q = np.zeros((2, 1, d)); q[1, 0, 0] = 1.0
    k = np.zeros((2, 1, d)); k[1, 0, 0] = 1.0
    v = np.zeros((2, 1, d)); v[0] = 1.0; v[1] = 3.0
    do = np.zeros((2, 1, d)); do[1, 0, 0] = 1.0          # only row 1, only column 0
    dq, dk, dv = ref_attention_bwd(q, k, v, do, [0, 2], True, math.log(2.0))
    c = math.log(2.0) * 4.0 / 9.0
    np.testing.assert_allclose(dv[:, 0, 0], [1.0 / 3.0, 2.0 / 3.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(dv[:, 0, 1], [0.0, 0.0], atol=0)
    np.testing.assert_allclose(dq[1, 0], [c, 0.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(dq[0, 0], [0.0, 0.0], atol=0)
    np.testing.assert_allclose(dk[0, 0], [-c, 0.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(dk[1, 0], [c, 0.0], rtol=0, atol=1e-15)


def test_mistakes_are_caught():
    """A dropped D term, a transposed dS or a missing scale each break the
    autograd comparison: the pins above can fail."""
    q, k, v, do, cu = _pack([6, 11], 1, 4, seed=5)
    want = _sdpa_grads(q, k, v, do, cu, True, 0.5)
    from oracle.attention import ref_probabilities
    p = ref_probabilities(q[6:, 0], k[6:, 0], 0.5, True)
    dp = do[6:, 0] @ v[6:, 0].T
    wrong_ds = p * dp                                   # D dropped
    wrong_dq = 0.5 * (wrong_ds @ k[6:, 0])
    assert np.abs(wrong_dq - want[0][6:, 0]).max() > 1e-3
    o = p @ v[6:, 0]
    ds = p * (dp - np.sum(do[6:, 0] * o, axis=1, keepdims=True))
    assert np.abs(0.5 * (ds.T @ k[6:, 0]) - want[0][6:, 0]).max() > 1e-3   # transposed
    assert np.abs(ds @ k[6:, 0] - want[0][6:, 0]).max() > 1e-3            # no scale


def test_mxfp8_gradients_are_those_of_the_mxfp8_forward():
    """Forward/backward consistency: the MXFP8 gradients are the derivatives
    of the MXFP8 forward oracle's loss sum(deq(dO) * O(deq(Q), deq(K),
    deq(V))) with respect to the dequantised operands (central finite
    differences on those values), and they differ from the bf16 gradients
    by the quantisation alone (checked against autograd of torch's fp64
    attention on the dequantised inputs)."""
    from oracle.mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref
    from oracle.attention_bwd import ref_attention_bwd_mxfp8

    def deq(x):
        return dequantize_mxfp8_ref(*quantize_mxfp8_ref(x))

    q, k, v, do, cu = _pack([5, 3], 1, 32, seed=21)
    scale = 0.3
    dq, dk, dv = ref_attention_bwd_mxfp8(q, k, v, do, cu, True, scale)
    qd, kd, vd, dod = deq(q), deq(k), deq(v), deq(do)
    assert not np.array_equal(qd, q)        # the quantiser does change the values
    want = _sdpa_grads(qd, kd, vd, dod, cu, True, scale)
    for g, w in zip((dq, dk, dv), want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)

    def loss(q_, k_, v_):
        o, _ = ref_attention(q_, k_, v_, cu, True, scale)
        return float(np.sum(dod * o))

    h = 1e-6
    rng = np.random.default_rng(3)
    for x, g in ((qd, dq), (kd, dk), (vd, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            old = x[idx]
            x[idx] = old + h
            fp = loss(qd, kd, vd)
            x[idx] = old - h
            fm = loss(qd, kd, vd)
            x[idx] = old
            assert abs((fp - fm) / (2 * h) - g[idx]) <= 1e-7

"""Pins of the incoherent-processing oracle (oracle/incoherent.py) against
textbook values, closed forms, exact integer arithmetic, an fp32 rounding
bound and the property the pages give it (outliers cost less precision).
CPU only."""
import numpy as np
import pytest
import torch

from oracle.attention import ref_attention, score_matrix
from oracle.incoherent import (hadamard, incoherent_matrix, ref_attention_incoherent_mxfp8,
                               rotate_fp32, rotate_fp64)
from oracle.mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref


def _signs(d, seed):
    return np.where(np.random.default_rng(seed).random(d) < 0.5, -1.0, 1.0)


def test_hadamard_textbook_values():
    assert np.array_equal(hadamard(1), [[1.0]])
    assert np.array_equal(hadamard(2), [[1, 1], [1, -1]])
    assert np.array_equal(hadamard(4), [[1, 1, 1, 1], [1, -1, 1, -1],
                                        [1, 1, -1, -1], [1, -1, -1, 1]])
    with pytest.raises(ValueError):
        hadamard(96)


@pytest.mark.parametrize("d", [1, 2, 8, 32, 64, 128])
def test_hadamard_rows_are_orthogonal(d):
    h = hadamard(d)
    assert set(np.unique(h)) <= {-1.0, 1.0}
    assert np.array_equal(h @ h.T, d * np.eye(d))
    m = incoherent_matrix(_signs(d, d))
    assert np.array_equal(m @ m.T, d * np.eye(d))


@pytest.mark.parametrize("d", [64, 128])
def test_butterfly_is_the_matrix_product_exactly_on_integers(d):
    """Small integers: every partial sum is exact in fp32, so the butterfly
    and the fp64 matrix product must agree bit for bit."""
    rng = np.random.default_rng(5)
    x = rng.integers(-100, 101, size=(7, 3, d)).astype(np.float32)
    s = _signs(d, 6)
    assert np.array_equal(rotate_fp32(x, s).astype(np.float64), rotate_fp64(x, s))


@pytest.mark.parametrize("d", [64, 128])
def test_butterfly_within_its_fp32_rounding_bound(d):
    """Each of the log2(d) stages rounds once a partial sum bounded by
    sum |x|: |fp32 - exact| <= log2(d) * 2^-24 * sum |x| per element."""
    g = torch.Generator().manual_seed(8)
    x = torch.randn((64, 2, d), generator=g).to(torch.bfloat16).float().numpy()
    s = _signs(d, 9)
    err = np.abs(rotate_fp32(x, s).astype(np.float64) - rotate_fp64(x, s))
    bound = np.log2(d) * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum(-1, keepdims=True)
    assert (err <= bound).all()
    assert err.max() > 0          # not trivially exact: the bound is doing work


def test_transform_twice_is_d_times_identity():
    """H H = d I (H symmetric): two unsigned transforms give d x, exactly on
    integers."""
    d = 128
    x = np.random.default_rng(10).integers(-50, 51, size=(4, d)).astype(np.float32)
    ones = np.ones(d)
    assert np.array_equal(rotate_fp32(rotate_fp32(x, ones), ones), d * x)


def test_scores_and_attention_unchanged_without_quantisation():
    """(Q M)(K M)^T / d = Q K^T: with the scale divided by d the attention
    of the rotated inputs is the plain attention (fp64)."""
    g = torch.Generator().manual_seed(11)
    L, H, d = 96, 2, 64
    q, k, v = (torch.randn((L, H, d), generator=g).double().numpy() for _ in range(3))
    s = _signs(d, 12)
    qr, kr = rotate_fp64(q, s), rotate_fp64(k, s)
    for h in range(H):
        a = score_matrix(q[:, h], k[:, h], 0.125, True)
        b = score_matrix(qr[:, h], kr[:, h], 0.125 / d, True)
        fin = np.isfinite(a)
        assert np.array_equal(fin, np.isfinite(b))
        assert np.allclose(a[fin], b[fin], rtol=1e-12, atol=1e-12)
    o1, l1 = ref_attention(q, k, v, [0, L], True, 0.125)
    o2, l2 = ref_attention(qr, kr, v, [0, L], True, 0.125 / d)
    assert np.allclose(o1, o2, rtol=1e-11, atol=1e-12)
    assert np.allclose(l1, l2, rtol=1e-11, atol=1e-12)


def test_outlier_channels_cost_less_precision_after_rotation():
    """The purpose the pages give: with the long-context outlier recipe
    (channels 5 and 70 of Q and K x20 before the bf16 cast), MXFP8 attention
    is far closer to the exact bf16-input attention when Q and K are rotated
    first (measured about 4x on this sample; required 2x)."""
    g = torch.Generator().manual_seed(3)
    L, H, d = 512, 2, 128
    q, k, v = (torch.randn((L, H, d), generator=g) for _ in range(3))
    for x in (q, k):
        x[:, :, 5] *= 20
        x[:, :, 70] *= 20
    q, k, v = (t.to(torch.bfloat16).double().numpy() for t in (q, k, v))
    scale = 1.0 / np.sqrt(d)
    exact, _ = ref_attention(q, k, v, [0, L], True, scale)

    def deq(x):
        return dequantize_mxfp8_ref(*quantize_mxfp8_ref(x))

    plain, _ = ref_attention(deq(q), deq(k), deq(v), [0, L], True, scale)
    rotated, _ = ref_attention_incoherent_mxfp8(q, k, v, [0, L], True, scale, _signs(d, 0))
    e_plain = np.abs(plain - exact).mean()
    e_rot = np.abs(rotated - exact).mean()
    assert e_rot < 0.5 * e_plain, (e_rot, e_plain)

"""Pins of the NVFP4 quantiser oracle (oracle/nvfp4.py): hand-computed E2M1
values, codes and E4M3 scale codes from the format definitions, an
exhaustive nearest-value search, no clipping and tightness of the scale,
the round-trip error bound, per-token independence, exactness on
representable inputs.  CPU only."""
import numpy as np
import pytest
import torch

from oracle.attention import ref_attention
from oracle.mxfp8 import dequantize_mxfp8_ref, e4m3_decode_table, quantize_mxfp8_ref
from oracle.nvfp4 import (dequantize_nvfp4_ref, e2m1_decode_table, e2m1_encode,
                          nvfp4_scale_codes, quantize_nvfp4_ref, ref_attention_nvfp4_mxfp8)

E4M3 = e4m3_decode_table()


def test_e2m1_table_by_hand():
    t = e2m1_decode_table()
    assert list(t[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(t[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert np.signbit(t[8])


@pytest.mark.parametrize("x,code", [
    (0.0, 0), (0.2, 0), (0.25, 0), (0.26, 1), (0.75, 2), (1.25, 2), (1.26, 3),
    (1.75, 4), (2.5, 4), (2.6, 5), (3.5, 6), (5.0, 6), (5.1, 7), (6.0, 7), (100.0, 7),
    (-0.1, 8), (-0.75, 10), (-5.0, 14), (-7.0, 15)])
def test_e2m1_encode_by_hand(x, code):
    """Ties go to the even code: 0.25 -> 0, 0.75 -> 1.0 (code 2), 1.25 -> 1.0,
    1.75 -> 2.0 (code 4), 2.5 -> 2.0, 3.5 -> 4.0 (code 6), 5 -> 4.0."""
    assert int(e2m1_encode(x)) == code


def test_e2m1_encode_matches_brute_force():
    t = e2m1_decode_table()

    def brute(x):
        a = abs(x)
        if a >= 6.0:
            c = 7
        else:
            best = min(abs(t[i] - a) for i in range(8))
            c = min((i for i in range(8) if abs(t[i] - a) == best), key=lambda i: (i & 1, i))
        return c | (8 if np.signbit(x) else 0)

    vals = list(t[:8])
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    xs = np.concatenate([np.random.default_rng(1).uniform(0, 8, 300), mids, vals, [0.0]])
    xs = np.concatenate([xs, -xs])
    np.testing.assert_array_equal(e2m1_encode(xs), [brute(float(x)) for x in xs])


@pytest.mark.parametrize("amax,value", [
    (6.0, 1.0), (7.0, 1.25), (0.0, 1.0), (6 * 448.0, 448.0), (1e6, 448.0),
    (1e-6, 2.0 ** -9), (3.0, 0.5), (6.75, 1.125)])
def test_scale_codes_by_hand(amax, value):
    """7 / 6 = 1.1667 lies between the E4M3 values 1.125 and 1.25, so 1.25;
    6.75 / 6 = 1.125 exactly; tiny blocks get the smallest positive E4M3
    value 2^-9; past 6 * 448 the scale stays 448."""
    assert E4M3[int(nvfp4_scale_codes(amax))] == value


def test_no_clipping_and_tight_scales():
    rng = np.random.default_rng(4)
    x = rng.normal(0.0, 1.0, (300, 64)) * np.exp(rng.uniform(-6, 6, (300, 1)))
    codes, scales = quantize_nvfp4_ref(x)
    s = E4M3[scales]
    amax = np.abs(x.reshape(300, 4, 16)).max(-1)
    assert (amax <= 6.0 * s).all()                       # nothing clipped
    pos = np.sort(E4M3[1:0x7F])
    prev = np.array([pos[max(np.searchsorted(pos, v) - 1, 0)] for v in s.ravel()]).reshape(s.shape)
    tight = s > pos[0]
    assert (amax[tight] > 6.0 * prev[tight]).all()       # the next smaller scale would clip


def test_roundtrip_error_bound():
    """|deq - x| <= S * ulp/2 of the E2M1 binade of |x| / S (0.5 below 2,
    1 below 4, 2 above), up to the fp32 division's rounding."""
    g = torch.Generator().manual_seed(6)
    x = torch.randn((200, 128), generator=g).to(torch.bfloat16).double().numpy()
    codes, scales = quantize_nvfp4_ref(x)
    deq = dequantize_nvfp4_ref(codes, scales)
    s = np.repeat(E4M3[scales], 16, axis=-1)
    r = np.abs(x) / s
    half_ulp = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
    assert (np.abs(deq - x) <= half_ulp * s * (1 + 1e-6)).all()


def test_scales_are_per_token():
    rng = np.random.default_rng(8)
    x = rng.normal(size=(10, 3, 64))
    c1, s1 = quantize_nvfp4_ref(x)
    y = x.copy()
    y[7] *= 1000.0
    c2, s2 = quantize_nvfp4_ref(y)
    keep = [i for i in range(10) if i != 7]
    assert np.array_equal(c1[keep], c2[keep]) and np.array_equal(s1[keep], s2[keep])


def test_representable_inputs_are_lossless():
    """Values that are E2M1 grid points times a per-block E4M3 scale whose
    block reaches 6 come back exactly, and the mixed-path attention on them
    is the plain attention (V representable in MXFP8 as well)."""
    rng = np.random.default_rng(9)
    grid = e2m1_decode_table()
    L, H, d = 40, 2, 64

    def representable():
        c = rng.integers(0, 16, (L, H, d))
        c[..., ::16] = 7                                     # each block's max is 6 * S
        s = E4M3[rng.integers(0x30, 0x40, (L, H, d // 16))]   # scales 0.5 .. 1.875
        return grid[c] * np.repeat(s, 16, axis=-1)

    q, k = representable(), representable()
    v = rng.integers(-8, 9, (L, H, d)).astype(np.float64) / 4.0   # exact in MXFP8 too
    for x in (q, k):
        assert np.array_equal(dequantize_nvfp4_ref(*quantize_nvfp4_ref(x)), x)
    assert np.array_equal(dequantize_mxfp8_ref(*quantize_mxfp8_ref(v)), v)
    cu = [0, 17, L]
    o1, l1 = ref_attention_nvfp4_mxfp8(q, k, v, cu, True, 0.2)
    o2, l2 = ref_attention(q, k, v, cu, True, 0.2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)

"""Pins of the bit-exact MXFP8 quantiser oracle: hand-computed codes from
the E4M3 / E8M0 format definitions, rounding bounds, and the per-token
independence of scales.  CPU only."""
import numpy as np
import pytest

from oracle.mxfp8 import (e4m3_decode_table, e4m3_encode, e8m0_scale_codes,
                          quantize_mxfp8_ref, dequantize_mxfp8_ref)


def test_decode_table_by_hand():
    t = e4m3_decode_table()
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and np.signbit(t[0x80])
    assert t[0x01] == 2.0 ** -9            # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9        # largest subnormal
    assert t[0x08] == 2.0 ** -6            # smallest normal
    assert t[0x38] == 1.0
    assert t[0x39] == 1.125
    assert t[0x7E] == 448.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert t[0xB8] == -1.0
    pos = t[:0x7F]
    assert (np.diff(pos) > 0).all()        # positive codes are monotone


@pytest.mark.parametrize("x,code", [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE),
    (449.0, 0x7E), (464.0, 0x7E), (1e9, 0x7E), (-1e9, 0xFE),
    (0.0, 0x00), (-0.0, 0x80),
    (1.0625, 0x38),        # tie between 1.0 (0x38) and 1.125 (0x39): even
    (1.1875, 0x3A),        # tie between 1.125 and 1.25: even code 0x3A
    (1.0626, 0x39),
    (2.0 ** -10, 0x00),    # half the smallest subnormal: tie to even (zero)
    (3 * 2.0 ** -10, 0x02),  # tie between 0x01 and 0x02: even
    (-(2.0 ** -11), 0x80),   # rounds to zero, keeps the sign
    (2.0 ** -6, 0x08),
    (240.0, 0x77),         # 1.875 * 2^7
    (0.3, 0x2A),           # between 0.28125 (0x29) and 0.3125 (0x2A): nearer 0x2A
])
def test_encode_by_hand(x, code):
    assert int(e4m3_encode(np.array([x]))[0]) == code


@pytest.mark.parametrize("amax,code", [
    (0.0, 127), (448.0, 127), (448.0000001, 128), (1.0, 119),
    (1.75, 119), (1.7500001, 120), (2.0 ** 200, 254), (2.0 ** -200, 0),
    (224.0, 126), (224.5, 127), (896.0, 128),
])
def test_scale_codes_by_hand(amax, code):
    assert int(e8m0_scale_codes(np.array([amax]))[0]) == code


def test_roundtrip_bounds_and_no_clipping():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 3, 128)).astype(np.float32)
    x[:, :, 5] *= 20
    x[:, :, 70] *= 20
    x[3, 1, 40:50] = 0.0
    x[7, 2, 64:96] = 0.0                     # a whole zero block
    x = x.astype(np.float64)
    codes, sc = quantize_mxfp8_ref(x)
    assert codes.shape == x.shape and sc.shape == (64, 3, 4)
    deq = dequantize_mxfp8_ref(codes, sc)
    X = sc.astype(np.int64) - 127
    step = np.repeat(np.ldexp(1.0, X), 32, axis=-1)
    amax = np.repeat(np.abs(x).reshape(64, 3, 4, 32).max(-1), 32, axis=-1)
    assert (amax <= 448.0 * step).all()                  # nothing clipped
    normal = np.abs(x) >= 2.0 ** -6 * step
    err = np.abs(x - deq)
    assert (err[normal] <= 2.0 ** -4 * np.abs(x[normal])).all()
    assert (err[~normal] <= 2.0 ** -10 * step[~normal]).all()
    assert sc[7, 2, 2] == 127 and (codes[7, 2, 64:96] == 0).all()
    # the block maximum keeps at least half of the E4M3 range (tight scale)
    nz = amax > 0
    assert (amax[nz] > 224.0 * step[nz]).all()


def test_scale_is_tight():
    """X is the smallest exponent that avoids clipping: halving the scale
    would push amax past 448."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 2, 64)) * np.exp(rng.uniform(-20, 20, (50, 2, 1)))
    _, sc = quantize_mxfp8_ref(x)
    amax = np.abs(x).reshape(50, 2, 2, 32).max(-1)
    X = sc.astype(np.int64) - 127
    assert (amax <= 448.0 * np.ldexp(1.0, X)).all()
    assert (amax > 448.0 * np.ldexp(1.0, X - 1)).all()


def test_scales_are_per_token():
    """Perturbing one token changes no other token's bytes: a scale never
    spans two tokens, so none spans a document or causal boundary."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 2, 128))
    c0, s0 = quantize_mxfp8_ref(x)
    y = x.copy()
    y[17] *= 1000.0
    c1, s1 = quantize_mxfp8_ref(y)
    keep = np.ones(40, dtype=bool); keep[17] = False
    np.testing.assert_array_equal(c0[keep], c1[keep])
    np.testing.assert_array_equal(s0[keep], s1[keep])
    assert not np.array_equal(s0[17], s1[17])


def test_encode_matches_brute_force_search():
    """Every finite magnitude's code by exhaustive search over the 256-code
    table, written independently of the encoder: the nearest finite value,
    an exact tie going to the code whose last bit is 0, magnitudes past 448
    to 448; the sign bit set for negative inputs.  Random magnitudes over
    the whole range, every midpoint between neighbours (the ties), the
    neighbours themselves and values past saturation."""
    from oracle.mxfp8 import e4m3_decode_table, e4m3_encode

    table = e4m3_decode_table()
    finite = [(c, table[c]) for c in range(128) if np.isfinite(table[c])]

    def brute(x):
        a = abs(x)
        if a >= 448.0:
            code = max(c for c, v in finite if v == 448.0)
        else:
            best = min(abs(v - a) for _, v in finite)
            cands = [c for c, v in finite if abs(v - a) == best]
            code = min(cands, key=lambda c: (c & 1, c))
        return code | (0x80 if np.signbit(x) else 0)

    vals = sorted(v for _, v in finite)
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    rng = np.random.default_rng(17)
    rand = np.exp(rng.uniform(np.log(1e-4), np.log(600.0), 400))
    xs = np.concatenate([rand, mids, vals, [448.0, 460.0, 1e4, 0.0]])
    xs = np.concatenate([xs, -xs])
    got = e4m3_encode(xs)
    want = np.array([brute(float(x)) for x in xs], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)

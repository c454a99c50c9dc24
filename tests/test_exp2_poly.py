"""Pins of the FMA-pipe 2^x used for part of the softmax weights: the
coefficients the kernel is built with (read from its source) are checked
against the exact function, and the bit-level construction (floor by a
rounded-down add of 1.5 * 2^23, exponent-field add) is emulated in fp32 with
numpy.  CPU only."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_tiled_attention_39_b200", "csrc", "attn_fwd_sm100.cuh")


def _coeffs():
    src = open(SRC).read()
    vals = {}
    for name in ("kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(name + r"\s*=\s*([-0-9.e+]+)f;", src)
        vals[name] = np.float32(float(m.group(1)))
    return vals["kExp2C1"], vals["kExp2C2"], vals["kExp2C3"]


def _poly(f):
    c1, c2, c3 = _coeffs()
    f = f.astype(np.float32)
    q = np.float32(c3) * f + np.float32(c2)
    q = q * f + np.float32(c1)
    return q * f + np.float32(1.0)


def _exp2_emulated(x):
    """The kernel's construction in fp32: clamp at -127, j = floor(x) from a
    round-down add of 1.5 * 2^23, f = x - j, result bits = bits(p(f)) + j << 23."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    j = np.floor(x.astype(np.float64))                  # what the rounded-down add yields
    t = (np.float32(12582912.0) + j.astype(np.float32)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    q = _poly(f)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_polynomial_relative_error():
    f = np.linspace(0.0, 1.0, 200001)
    rel = np.abs(_poly(f).astype(np.float64) / np.exp2(f) - 1.0)
    assert rel.max() < 1.0e-4


def test_polynomial_is_one_at_zero():
    assert _poly(np.zeros(1))[0] == np.float32(1.0)


def test_construction_matches_exp2():
    x = np.concatenate([np.linspace(-120.0, 8.0, 100001), [-3.5, -1.0, 0.0, 0.25, 7.999]])
    y = _exp2_emulated(x).astype(np.float64)
    rel = np.abs(y / np.exp2(np.asarray(x, dtype=np.float32).astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4
    assert _exp2_emulated(np.array([0.0]))[0] == 1.0
    assert _exp2_emulated(np.array([3.0]))[0] == 8.0


def test_masked_scores_give_exact_zero():
    y = _exp2_emulated(np.array([-np.inf, -1e30, -127.0, -500.0], dtype=np.float32))
    assert (y == 0.0).all() and not np.signbit(y).any()

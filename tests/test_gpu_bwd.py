"""Parity of the backward (dQ, dK, dV) through the C ABI against the fp64
oracle (oracle/attention_bwd.py), element by element.

The forward runs first (our kernel) to give out and lse, as a training step
would; the oracle recomputes everything in fp64 from the same bf16 inputs.
Gradients are not normalised like the forward's output, so the bounds are
taken relative to each gradient tensor's largest magnitude: the forward's
per-element budgets (2e-2 max, 2e-3 mean for an output of unit scale)
applied to that scale."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import workloads
from oracle.attention_bwd import ref_attention_bwd, ref_attention_bwd_mxfp8

BWD_REL_MAX = 2e-2
BWD_REL_MEAN = 2e-3

pytestmark = pytest.mark.gpu


def _inputs(lengths, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    q, k, v, do = (torch.randn((T, H, d), generator=g).to(torch.bfloat16) for _ in range(4))
    return q, k, v, do


def _run(q, k, v, do, cu, causal, scale, max_seqlen, num_seqs=None, dtype=A.ATTN_BF16):
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    T, H, d = q.shape
    out = torch.empty_like(qd)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    cud = cu.to(dev) if cu is not None else None
    A.attn_fwd(qd, kd, vd, cud, out, lse, causal, scale, max_seqlen=max_seqlen,
               num_seqs=num_seqs, dtype=dtype)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    ws = A.attn_bwd(qd, kd, vd, out, dod, lse, cud, dq, dk, dv, causal, scale,
                    max_seqlen=max_seqlen, num_seqs=num_seqs, dtype=dtype)
    assert A.attn_get_device_error(ws) == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check(got, ref, name):
    g = got.double().numpy()
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    e = np.abs(g - ref)
    scale = max(float(np.abs(ref).max()), 1e-6)
    assert e.max() <= BWD_REL_MAX * scale, (name, float(e.max()), scale)
    assert e.mean() <= BWD_REL_MEAN * scale, (name, float(e.mean()), scale)
    return float(e.max()) / scale, float(e.mean()) / scale


def _compare(lengths, H, d, causal, seed, dense=False):
    q, k, v, do = _inputs(lengths, H, d, seed)
    scale = 1.0 / math.sqrt(d)
    cu = workloads.cu_from_lengths(lengths)
    if dense:
        got = _run(q, k, v, do, None, causal, scale, lengths[0], num_seqs=len(lengths))
    else:
        got = _run(q, k, v, do, cu, causal, scale, max(lengths))
    ref = ref_attention_bwd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                            do.double().numpy(), cu.numpy(), causal, scale)
    return [_check(gt, rf, n) for gt, rf, n in zip(got, ref, ("dq", "dk", "dv"))]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_bwd_packed_ragged(d, causal):
    """Ragged packed documents: a one-token document, an empty one, tails of
    1, 2, 44 and 64 rows past a tile edge, an exact tile, several query and
    key tiles."""
    _compare([1, 130, 0, 300, 129, 64, 256, 44], 2, d, causal, seed=11)


def test_bwd_dense_batch():
    """Dense mode (no cu_seqlens): B = 2 documents of 384 tokens, 3 heads."""
    _compare([384, 384], 3, 128, True, seed=12, dense=True)


def test_bwd_long_document():
    """One 2048-token document: 16 key tiles, up to 16 query tiles each."""
    _compare([2048], 2, 128, True, seed=13)


def test_bwd_bad_seqlens_leaves_outputs():
    """cu_seqlens whose last entry is not T: the device records
    ATTN_ERR_BAD_SEQLENS and dq, dk, dv keep their contents."""
    dev = torch.device("cuda:0")
    T, H, d = 256, 2, 64
    q, k, v, do = (t.to(dev) for t in _inputs([T], H, d, seed=14))
    out = torch.zeros_like(q)
    lse = torch.zeros((H, T), dtype=torch.float32, device=dev)
    cu = torch.tensor([0, 100, 200], dtype=torch.int32, device=dev)   # 200 != T
    dq, dk, dv = (torch.full_like(q, 7.0) for _ in range(3))
    ws = A.attn_bwd(q, k, v, out, do, lse, cu, dq, dk, dv, True, 0.125, max_seqlen=128)
    assert A.attn_get_device_error(ws) == 5
    for t in (dq, dk, dv):
        assert bool((t == 7.0).all())


# ---------------------------------------------------------------- MXFP8
def _outlier_inputs(lengths, H, d, seed):
    """Q, K with two outlier channels x20 (the long-context recipe), V and dO
    plain, all rounded to bf16."""
    g = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    x = [torch.randn((T, H, d), generator=g) for _ in range(4)]
    for t in x[:2]:
        t[:, :, 5] *= 20
        t[:, :, 70 % d] *= 20
    return [t.to(torch.bfloat16) for t in x]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_bwd_mxfp8_packed_ragged(d, causal):
    """The MXFP8 backward (out and lse from the MXFP8 forward) against the
    fp64 gradient oracle of the MXFP8 path (gradients on the exactly
    dequantised Q, K, V, dO), every element, ragged pack with outliers."""
    lengths = [1, 130, 0, 300, 129, 64, 256, 44]
    q, k, v, do = _outlier_inputs(lengths, 2, d, seed=51 + d)
    scale = 1.0 / math.sqrt(d)
    cu = workloads.cu_from_lengths(lengths)
    got = _run(q, k, v, do, cu, causal, scale, max(lengths), dtype=A.ATTN_MXFP8)
    ref = ref_attention_bwd_mxfp8(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                  do.double().numpy(), cu.numpy(), causal, scale)
    for gt, rf, n in zip(got, ref, ("dq", "dk", "dv")):
        _check(gt, rf, n)


def test_bwd_mxfp8_long_document():
    """One 2048-token document with outlier channels, d 128, MXFP8."""
    q, k, v, do = _outlier_inputs([2048], 2, 128, seed=53)
    cu = workloads.cu_from_lengths([2048])
    scale = 1.0 / math.sqrt(128)
    got = _run(q, k, v, do, cu, True, scale, 2048, dtype=A.ATTN_MXFP8)
    ref = ref_attention_bwd_mxfp8(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                  do.double().numpy(), cu.numpy(), True, scale)
    for gt, rf, n in zip(got, ref, ("dq", "dk", "dv")):
        _check(gt, rf, n)


def test_bwd_mxfp8_no_leak_across_documents():
    """Scales cover one token of one head, so the quantised operands of a
    document do not depend on any other document: changing every other
    document's Q, K, V and dO (by large values, which would move any scale
    shared with them) leaves this document's dK and dV bit-identical and its
    dQ equal up to the order of the fp32 accumulator's additions."""
    lengths = [200, 450, 90]
    q, k, v, do = _outlier_inputs(lengths, 2, 128, seed=55)
    cu = workloads.cu_from_lengths(lengths)
    got = _run(q, k, v, do, cu, True, 0.088, 450, dtype=A.ATTN_MXFP8)
    g = torch.Generator().manual_seed(56)
    x2 = [t.clone() for t in (q, k, v, do)]
    for t in x2:
        t[:200] = (torch.randn(t[:200].shape, generator=g) * 50).bfloat16()
        t[650:] = (torch.randn(t[650:].shape, generator=g) * 50).bfloat16()
    got2 = _run(*x2, cu, True, 0.088, 450, dtype=A.ATTN_MXFP8)
    doc = slice(200, 650)
    assert torch.equal(got2[1][doc], got[1][doc]) and torch.equal(got2[2][doc], got[2][doc])
    dq_a, dq_b = got[0][doc].float(), got2[0][doc].float()
    assert float((dq_a - dq_b).abs().max()) <= 2 ** -7 * float(dq_a.abs().max())

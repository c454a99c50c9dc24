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
from oracle.attention_bwd import ref_attention_bwd

BWD_REL_MAX = 2e-2
BWD_REL_MEAN = 2e-3

pytestmark = pytest.mark.gpu


def _inputs(lengths, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    q, k, v, do = (torch.randn((T, H, d), generator=g).to(torch.bfloat16) for _ in range(4))
    return q, k, v, do


def _run(q, k, v, do, cu, causal, scale, max_seqlen, num_seqs=None):
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    T, H, d = q.shape
    out = torch.empty_like(qd)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    cud = cu.to(dev) if cu is not None else None
    A.attn_fwd(qd, kd, vd, cud, out, lse, causal, scale, max_seqlen=max_seqlen,
               num_seqs=num_seqs)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    ws = A.attn_bwd(qd, kd, vd, out, dod, lse, cud, dq, dk, dv, causal, scale,
                    max_seqlen=max_seqlen, num_seqs=num_seqs)
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

"""The allocation-free entry point ``attn_fwd_noalloc``.

Some callers cannot allocate device memory (a plugin handed only its input
and output buffers, code under a memory budget fixed up front, a
latency-critical path that cannot take cudaMalloc's implicit
synchronisation).  ``attn_fwd_noalloc`` serves them with the library's fixed
device scratch instead of a caller workspace.  This test calls it through
the C ABI twice in a row, on two different packs (so the second call runs on
scratch the first one left behind), and checks each result against the
workspace entry point ``attn_fwd`` within the tolerances the other GPU tests
use.  It sits in its own file, collected last, and passes alone or after the
other tests.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    A.lib()


def _pack(lengths, H, d, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    T = sum(lengths)
    dev = torch.device("cuda:0")
    q, k, v = (torch.randn([T, H, d], generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
    return q, k, v, workloads.cu_from_lengths(lengths).to(dev)


def test_no_alloc_matches_workspace_entry_point_twice():
    dev = torch.device("cuda:0")
    cases = [([300, 129, 1, 640, 77], 3, 128, True, 11),
             ([1000, 24, 0, 513], 2, 64, False, 12)]
    for lengths, H, d, causal, seed in cases:
        q, k, v, cu = _pack(lengths, H, d, seed)
        T = q.shape[0]
        scale = 1.0 / d ** 0.5
        ref_out = torch.empty_like(q)
        ref_lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        ws = A.attn_fwd(q, k, v, cu, ref_out, ref_lse, causal, scale, max_seqlen=max(lengths))
        assert A.attn_get_device_error(ws) == 0
        out = torch.full_like(q, float("nan"))
        lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=dev)
        A.attn_fwd_noalloc(q, k, v, cu, out, lse, causal, scale, max_seqlen=max(lengths))
        torch.cuda.synchronize()
        e = (out.float() - ref_out.float()).abs()
        assert float(e.max()) <= MAX_ABS and float(e.mean()) <= MEAN_ABS
        assert float((lse - ref_lse).abs().max()) <= LSE_ABS
        assert torch.isfinite(out.float()).all()


def _edge_pack(n_short, long_len):
    """n_short one-token documents then one of long_len tokens (1 head, d 64)."""
    return [1] * n_short + [long_len]


def test_no_alloc_size_limit_edges():
    """The fixed scratch holds the work lists of problems with
    total_tokens / 128 + num_seqs <= 32751 (integer division).  A problem
    exactly at that edge runs and matches attn_fwd; one past it is rejected
    on the host with ATTN_ERR_WORKSPACE before anything is launched."""
    dev = torch.device("cuda:0")
    # at the edge: 32494 + 1 documents, 32768 tokens -> 256 + 32495 = 32751
    lengths = _edge_pack(32494, 274)
    assert sum(lengths) // 128 + len(lengths) == 32751
    q, k, v, cu = _pack(lengths, 1, 64, seed=13)
    T = q.shape[0]
    ref_out = torch.empty_like(q)
    ref_lse = torch.empty((1, T), dtype=torch.float32, device=dev)
    ws = A.attn_fwd(q, k, v, cu, ref_out, ref_lse, True, 0.125, max_seqlen=274)
    assert A.attn_get_device_error(ws) == 0
    out = torch.full_like(q, float("nan"))
    lse = torch.full((1, T), float("nan"), dtype=torch.float32, device=dev)
    A.attn_fwd_noalloc(q, k, v, cu, out, lse, True, 0.125, max_seqlen=274)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))
    # one past the edge: 32495 + 1 documents, 32768 tokens -> 32752
    lengths = _edge_pack(32495, 273)
    assert sum(lengths) // 128 + len(lengths) == 32752
    q, k, v, cu = _pack(lengths, 1, 64, seed=14)
    lse = torch.empty((1, q.shape[0]), dtype=torch.float32, device=dev)
    with pytest.raises(A.AttnError) as ei:
        A.attn_fwd_noalloc(q, k, v, cu, torch.empty_like(q), lse, True, 0.125, max_seqlen=273)
    assert ei.value.code == 4


def test_no_alloc_rejects_problems_beyond_its_scratch():
    x = torch.empty((8, 1, 64), dtype=torch.bfloat16, device="cuda:0")
    lse = torch.empty((1, 8), dtype=torch.float32, device="cuda:0")
    # 32752 documents need a work list longer than the fixed scratch holds;
    # the check happens on the host, before anything is launched.
    cu = torch.zeros(32753, dtype=torch.int32, device="cuda:0")
    with pytest.raises(A.AttnError) as ei:
        A.attn_fwd_noalloc(x, x, x, cu, x, lse, True, 0.125, max_seqlen=8)
    assert ei.value.code == 4


@pytest.mark.parametrize("bad", ["lse_shape", "lse_dtype", "out_dtype", "q_noncontig", "cu_dtype"])
def test_no_alloc_binding_rejects_bad_tensors(bad):
    """The binding checks every tensor before the call: a wrong shape, type
    or layout would otherwise let the kernel write out of bounds."""
    dev = torch.device("cuda:0")
    q, k, v, cu = _pack([100, 28], 2, 64, seed=15)
    out = torch.empty_like(q)
    lse = torch.empty((2, 128), dtype=torch.float32, device=dev)
    if bad == "lse_shape":
        lse = torch.empty((2, 127), dtype=torch.float32, device=dev)
    elif bad == "lse_dtype":
        lse = torch.empty((2, 128), dtype=torch.float16, device=dev)
    elif bad == "out_dtype":
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    elif bad == "q_noncontig":
        q = torch.empty((2, 128, 64), dtype=torch.bfloat16, device=dev).transpose(0, 1)
    else:
        cu = cu.to(torch.int64)
    with pytest.raises(ValueError):
        A.attn_fwd_noalloc(q, k, v, cu, out, lse, True, 0.125, max_seqlen=100)

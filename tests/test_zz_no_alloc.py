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


def test_no_alloc_rejects_problems_beyond_its_scratch():
    x = torch.empty((8, 1, 64), dtype=torch.bfloat16, device="cuda:0")
    lse = torch.empty((1, 8), dtype=torch.float32, device="cuda:0")
    # 32752 documents need a work list longer than the fixed scratch holds;
    # the check happens on the host, before anything is launched.
    cu = torch.zeros(32753, dtype=torch.int32, device="cuda:0")
    with pytest.raises(A.AttnError) as ei:
        A.attn_fwd_noalloc(x, x, x, cu, x, lse, True, 0.125, max_seqlen=8)
    assert ei.value.code == 4

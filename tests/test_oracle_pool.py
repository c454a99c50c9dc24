"""The pooled oracle (tests/oracle_pool.py) returns what one ref_attention
call over the whole pack returns: the problems are independent, so splitting
them across processes changes nothing but the BLAS summation order inside a
product (single-threaded in the workers), i.e. the last bits.  CPU only."""
import numpy as np
import torch

from exact_tiled_attention_39_b200 import workloads
from oracle.attention import ref_attention
from oracle_pool import full_reference


def test_pool_equals_single_call():
    lengths = [5, 0, 130, 64, 257]
    g = torch.Generator().manual_seed(3)
    T, H, d = sum(lengths), 3, 16
    q, k, v = (torch.randn((T, H, d), generator=g).double().numpy() for _ in range(3))
    cu = workloads.cu_from_lengths(lengths).numpy()
    for causal in (True, False):
        ro, rl = ref_attention(q, k, v, cu, causal, 0.25)
        po, pl = full_reference(q, k, v, lengths, causal, 0.25, workers=3, row_chunk=64)
        assert np.abs(po - ro).max() <= 1e-12 and np.abs(pl - rl).max() <= 1e-12
        po, pl = full_reference(q, k, v, lengths, causal, 0.25, heads=[2, 0], workers=2)
        assert np.abs(po - ro[:, [2, 0]]).max() <= 1e-12
        assert np.abs(pl - rl[[2, 0]]).max() <= 1e-12

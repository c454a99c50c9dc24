"""The incoherent-processing pre-pass on the GPU against the oracle: the
rotated rows' E4M3 codes and E8M0 scales must equal, bit for bit, those of
the oracle quantiser applied to the oracle's fp32 butterfly
(oracle/incoherent.py), on the long-context outlier recipe and on plain
normal rows, head dims 64 and 128, with a ragged number of rows."""
import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from oracle.incoherent import rotate_fp32
from oracle.mxfp8 import quantize_mxfp8_ref

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("outliers", [False, True])
def test_rotated_codes_bit_identical(d, outliers):
    g = torch.Generator().manual_seed(31 + d)
    T, H = 1000, 3                                   # 3000 rows: not a multiple of 128
    x = torch.randn((T, H, d), generator=g)
    if outliers:
        x[:, :, 5] *= 20
        x[:, :, 70 % d] *= 20
    x = x.to(torch.bfloat16)
    signs = torch.where(torch.rand(d, generator=g) < 0.5, -1.0, 1.0).float()
    dev = torch.device("cuda:0")
    codes = torch.zeros((T, H, d), dtype=torch.uint8, device=dev)
    scales = torch.zeros((T, H, d // 32), dtype=torch.uint8, device=dev)
    A.attn_quantize_mxfp8_rotated(x.to(dev), signs.to(dev), codes, scales)
    torch.cuda.synchronize()
    ref_codes, ref_scales = quantize_mxfp8_ref(rotate_fp32(x.float().numpy(), signs.numpy()))
    assert np.array_equal(scales.cpu().numpy(), ref_scales)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)

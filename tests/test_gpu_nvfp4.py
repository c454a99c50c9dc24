"""GPU parity of the mixed NVFP4 / FP8 path (FLAMIA page, section "FLAMIA
Mimarisi ve Temel Tasarım İlkeleri"): the NVFP4 pre-pass, every E2M1 code
and every E4M3 scale byte equal to the oracle quantiser's (oracle/nvfp4.py)
on hand-built blocks (zeros, ties, saturation, tiny and huge magnitudes,
signed zeros), on random rows with outlier channels and on the full
workload's Q and K; and the attention (dtype ATTN_NVFP4: block-scaled E2M1
score product, P V on MXFP8 V) against the oracle run on the exactly
dequantised operands, element by element on ragged packs and on every
element of the full workload, with the no-leak property of its scales."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads
from oracle.mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref
from oracle.nvfp4 import dequantize_nvfp4_ref, quantize_nvfp4_ref, ref_attention_nvfp4_mxfp8
from helpers import BF16_MEAN_ABS, LSE_ABS, MXFP8_MAX_ABS, run_gpu
from oracle_pool import full_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    A.lib()


def _gpu_quant(x):
    """x: CPU bf16 [..., C].  Returns (codes one per byte, scales) as numpy."""
    dev = torch.device("cuda:0")
    xd = x.to(dev).contiguous()
    C = x.shape[-1]
    packed = torch.zeros(x.shape[:-1] + (C // 2,), dtype=torch.uint8, device=dev)
    scales = torch.zeros(x.shape[:-1] + (C // 16,), dtype=torch.uint8, device=dev)
    A.attn_quantize_nvfp4(xd, packed, scales)
    torch.cuda.synchronize()
    p = packed.cpu().numpy()
    codes = np.stack([p & 15, p >> 4], axis=-1).reshape(x.shape)
    return codes, scales.cpu().numpy()


def _check(x):
    codes, scales = _gpu_quant(x)
    ref_codes, ref_scales = quantize_nvfp4_ref(x.double().numpy())
    assert np.array_equal(scales, ref_scales)
    assert np.array_equal(codes, ref_codes)


def test_hand_blocks():
    rows = []
    rows.append([0.0] * 16)                                          # zero block: S = 1
    rows.append([-0.0] + [0.0] * 15)
    rows.append([6.0, -6.0, 3.0, 0.25, 0.75, 5.0, -5.0, 2.5] + [0.0] * 8)   # ties at S = 1
    rows.append([1e-6] + [0.0] * 15)                                 # below the smallest scale
    rows.append([3e4, -1e3, 1.0] + [0.0] * 13)                       # past 6 * 448: saturation
    rows.append([448 * 6.0, 1.0] + [0.0] * 14)
    rows.append([7.0, -0.01, 0.02] + [0.5] * 13)                     # sign of rounded zeros
    rows.append([float(v) for v in np.linspace(-3, 3, 16)])
    x = torch.tensor(rows, dtype=torch.float32).to(torch.bfloat16)[:, None, :]
    _check(x)


@pytest.mark.parametrize("d", [64, 128])
def test_random_rows_with_outliers(d):
    g = torch.Generator().manual_seed(61 + d)
    x = torch.randn((1000, 3, d), generator=g)
    x[:, :, 5] *= 20
    x[:, :, 70 % d] *= 20
    x[7] *= 1e-4
    x[8] *= 300.0
    _check(x.to(torch.bfloat16))


def test_full_workload_q_k():
    inp = workloads.make_inputs("mxfp8_packed")
    for name in ("q", "k"):
        _check(inp[name])


# ---------------------------------------------------------------- attention
def _outlier_pack(lengths, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    x = [torch.randn((T, H, d), generator=g) for _ in range(3)]
    for t in x[:2]:
        t[:, :, 5] *= 20
        t[:, :, 70 % d] *= 20
    return [t.to(torch.bfloat16) for t in x]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_nvfp4_attention_ragged(d, causal):
    lengths = [1, 127, 300, 0, 129, 513, 64]
    q, k, v = _outlier_pack(lengths, 2, d, seed=71 + d)
    cu = workloads.cu_from_lengths(lengths)
    scale = 1.0 / math.sqrt(d)
    out, lse, ws = run_gpu(q, k, v, cu, causal, scale, dtype=A.ATTN_NVFP4)
    assert A.attn_get_device_error(ws) == 0
    ro, rl = ref_attention_nvfp4_mxfp8(q.double().numpy(), k.double().numpy(),
                                       v.double().numpy(), cu.numpy(), causal, scale)
    e = np.abs(out.double().numpy() - ro)
    assert e.max() <= MXFP8_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


def test_nvfp4_full_workload_every_element():
    inp = workloads.make_inputs("nvfp4_packed")
    out, lse, ws = run_gpu(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], True, inp["scale"],
                           dtype=A.ATTN_NVFP4, max_seqlen=max(inp["lengths"]))
    assert A.attn_get_device_error(ws) == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    qd = dequantize_nvfp4_ref(*quantize_nvfp4_ref(inp["q"].double().numpy()))
    kd = dequantize_nvfp4_ref(*quantize_nvfp4_ref(inp["k"].double().numpy()))
    vd = dequantize_mxfp8_ref(*quantize_mxfp8_ref(inp["v"].double().numpy()))
    ro, rl = full_reference(qd, kd, vd, inp["lengths"], True, inp["scale"])
    e = np.abs(out.double().numpy() - ro)
    assert e.max() <= MXFP8_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


def test_nvfp4_no_causal_leakage():
    """Scales cover 16 elements of one token: changing later tokens of a
    document, or other documents, leaves earlier rows bit-identical (the
    pre-pass included)."""
    lengths = [200, 450, 90]
    q, k, v = _outlier_pack(lengths, 2, 128, seed=75)
    cu = workloads.cu_from_lengths(lengths)
    out, lse, _ = run_gpu(q, k, v, cu, True, 0.088, dtype=A.ATTN_NVFP4)
    i = 200 + 260
    g = torch.Generator().manual_seed(76)
    x2 = [t.clone() for t in (q, k, v)]
    for t in x2:
        t[i + 1:650] = (torch.randn(t[i + 1:650].shape, generator=g) * 50).bfloat16()
        t[:200] = (torch.randn(t[:200].shape, generator=g) * 50).bfloat16()
    out2, lse2, _ = run_gpu(*x2, cu, True, 0.088, dtype=A.ATTN_NVFP4)
    assert torch.equal(out2[200:i + 1], out[200:i + 1])
    assert torch.equal(lse2[:, 200:i + 1], lse[:, 200:i + 1])

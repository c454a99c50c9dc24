"""Incoherent processing on the GPU against the oracle: the rotating
pre-pass's E4M3 codes and E8M0 scales must equal, bit for bit, those of the
oracle quantiser applied to the oracle's fp32 butterfly
(oracle/incoherent.py), on the long-context outlier recipe and on plain
normal rows, head dims 64 and 128, with a ragged number of rows; the MXFP8
forward with incoherent processing (attn_fwd_incoherent) element by element
against the oracle on ragged packs and the full outlier workload; and the
error it saves on outlier channels against plain MXFP8."""
import functools
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads
from oracle.incoherent import (incoherent_operands, ref_attention_incoherent_mxfp8,
                               rotate_fp32)
from oracle.mxfp8 import quantize_mxfp8_ref
from helpers import BF16_MEAN_ABS, LSE_ABS, MXFP8_MAX_ABS, run_gpu
from oracle_pool import full_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    A.lib()


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


# ---------------------------------------------------------------- attention
def _signs(d, seed):
    return workloads.draw_signs(seed, d)


def _run_incoherent(q, k, v, cu, causal, scale, signs, max_seqlen):
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    T, H, d = q.shape
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=dev)
    ws = A.attn_fwd_incoherent(qd, kd, vd, cu.to(dev), out, lse, causal, scale, signs.to(dev),
                               max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    assert A.attn_get_device_error(ws) == 0
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_incoherent_attention_ragged(d, causal):
    """attn_fwd_incoherent on a ragged pack with outlier channels, element by
    element against the oracle of incoherent processing (rotation in fp32,
    MXFP8 quantisation, fp64 attention with the scale divided by d)."""
    lengths = [1, 127, 300, 0, 129, 513, 64]
    g = torch.Generator().manual_seed(41 + d)
    T, H = sum(lengths), 2
    x = [torch.randn((T, H, d), generator=g) for _ in range(3)]
    for t in x[:2]:
        t[:, :, 5] *= 20
        t[:, :, 70 % d] *= 20
    q, k, v = (t.to(torch.bfloat16) for t in x)
    cu = workloads.cu_from_lengths(lengths)
    scale = 1.0 / math.sqrt(d)
    signs = _signs(d, 7 + d)
    out, lse = _run_incoherent(q, k, v, cu, causal, scale, signs, max(lengths))
    ro, rl = ref_attention_incoherent_mxfp8(q.double().numpy(), k.double().numpy(),
                                            v.double().numpy(), cu.numpy(), causal, scale,
                                            signs.numpy())
    e = np.abs(out.double().numpy() - ro)
    assert e.max() <= MXFP8_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


@functools.lru_cache(maxsize=1)
def _full_case():
    """The incoherent workload on the GPU (incoherent and plain MXFP8) and
    the oracle's outputs for it: incoherent, and exact on the bf16 inputs."""
    inp = workloads.make_inputs("mxfp8_incoherent")
    cu = inp["cu_seqlens"]
    ms = max(inp["lengths"])
    got_rot = _run_incoherent(inp["q"], inp["k"], inp["v"], cu, True, inp["scale"],
                              inp["signs"], ms)
    got_plain = run_gpu(inp["q"], inp["k"], inp["v"], cu, True, inp["scale"],
                        dtype=A.ATTN_MXFP8, max_seqlen=ms)[:2]
    q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
    qd, kd, vd, s = incoherent_operands(q, k, v, inp["scale"], inp["signs"].numpy())
    ref_rot = full_reference(qd, kd, vd, inp["lengths"], True, s)
    exact = full_reference(q, k, v, inp["lengths"], True, inp["scale"])
    return got_rot, got_plain, ref_rot, exact


def test_incoherent_full_workload_every_element():
    """The full incoherent workload (config-5 inputs, outlier channels)
    against the oracle of incoherent processing, every element."""
    (out, lse), _, (ro, rl), _ = _full_case()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    e = np.abs(out.double().numpy() - ro)
    assert e.max() <= MXFP8_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


def test_incoherent_cuts_outlier_error():
    """What incoherent processing is for: on the outlier workload the GPU's
    MXFP8 output with rotated Q and K is much closer to the exact attention
    on the bf16 inputs than plain MXFP8 (the oracle pin asks for 2x)."""
    (out_r, _), (out_p, _), _, (ex, _) = _full_case()
    e_rot = float(np.abs(out_r.double().numpy() - ex).mean())
    e_plain = float(np.abs(out_p.double().numpy() - ex).mean())
    assert e_rot < 0.5 * e_plain, (e_rot, e_plain)

"""GPU parity of the MXFP8 path: the fused quantisation pre-pass against the
bit-exact CPU quantiser (every byte), and MXFP8 attention against the fp64
oracle run on the dequantised inputs (FLAMIA page, section "FLAMIA Mimarisi
ve Temel Tasarım İlkeleri": quantisation fused into the kernels, scales that
never carry information from future tokens)."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads
from oracle.attention import ref_attention
from oracle.mxfp8 import quantize_mxfp8_ref, dequantize_mxfp8_ref
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
    dev = torch.device("cuda:0")
    xd = x.to(dev).contiguous()
    codes = torch.empty(x.shape, dtype=torch.uint8, device=dev)
    scales = torch.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=torch.uint8, device=dev)
    A.attn_quantize_mxfp8(xd, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _deq(x_bf16):
    c, s = quantize_mxfp8_ref(x_bf16.double().numpy())
    return dequantize_mxfp8_ref(c, s)


def test_quantiser_bytes_hand_cases():
    vals = [0.0, -0.0, 1.0, -1.0, 448.0, 1.0625, 1.1875, 3 * 2.0 ** -10, 2.0 ** -10, 240.0,
            1e-30, -1e-30, 65504.0, 3.0e38, -2.5e-38, 0.3]
    x = torch.zeros(8, 64)
    for i, v in enumerate(vals):
        x[i // 2, (i % 2) * 32 + 3] = v
        x[i // 2, (i % 2) * 32 + 7] = v / 3
    x[5, 0:32] = 0.0                      # a whole zero block
    x[6, 32:64] = torch.linspace(-5, 5, 32)
    xb = x.to(torch.bfloat16)
    gc, gs = _gpu_quant(xb)
    rc, rs = quantize_mxfp8_ref(xb.double().numpy())
    np.testing.assert_array_equal(gs, rs)
    np.testing.assert_array_equal(gc, rc)


def test_quantiser_bytes_full_workload():
    inp = workloads.make_inputs("mxfp8_packed")
    for name in ("q", "k", "v"):
        gc, gs = _gpu_quant(inp[name])
        rc, rs = quantize_mxfp8_ref(inp[name].double().numpy())
        np.testing.assert_array_equal(gs, rs)
        np.testing.assert_array_equal(gc, rc)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_mxfp8_ragged_pack_vs_oracle(causal, d):
    """d = 128 runs the block-scaled kernel; d = 64 the bf16 kernel on the
    exactly dequantised values.  Outlier channels in two different 32-element
    scale blocks."""
    lengths = [1, 127, 129, 300, 0, 513, 64, 256]
    g = torch.Generator("cpu").manual_seed(31 + d)
    T, H = sum(lengths), 2
    q = torch.randn([T, H, d], generator=g)
    k = torch.randn([T, H, d], generator=g)
    v = torch.randn([T, H, d], generator=g)
    for t in (q, k):
        t[:, :, 5] *= 20
        t[:, :, 70 if d == 128 else 40] *= 20
    q, k, v = (t.bfloat16() for t in (q, k, v))
    cu = workloads.cu_from_lengths(lengths)
    scale = 1.0 / math.sqrt(d)
    out, lse, ws = run_gpu(q, k, v, cu, causal, scale, dtype=A.ATTN_MXFP8)
    assert A.attn_get_device_error(ws) == 0
    ro, rl = ref_attention(_deq(q), _deq(k), _deq(v), cu.numpy(), causal, scale)
    assert np.abs(out.double().numpy() - ro).max() <= MXFP8_MAX_ABS
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


def test_mxfp8_no_causal_leakage():
    """The pre-pass is included: perturbing later tokens of a document, or
    other documents, leaves earlier rows bit-identical."""
    lengths = [200, 450, 90]
    g = torch.Generator("cpu").manual_seed(6)
    q, k, v = (torch.randn([740, 2, 128], generator=g).bfloat16() for _ in range(3))
    cu = workloads.cu_from_lengths(lengths)
    out, lse, _ = run_gpu(q, k, v, cu, True, 0.088, dtype=A.ATTN_MXFP8)
    i = 200 + 260
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    for t in (q2, k2, v2):
        t[i + 1:650] = (torch.randn(t[i + 1:650].shape, generator=g) * 50).bfloat16()
        t[:200] = (torch.randn(t[:200].shape, generator=g) * 50).bfloat16()
    out2, lse2, _ = run_gpu(q2, k2, v2, cu, True, 0.088, dtype=A.ATTN_MXFP8)
    assert torch.equal(out2[200:i + 1], out[200:i + 1])
    assert torch.equal(lse2[:, 200:i + 1], lse[:, 200:i + 1])


def test_mxfp8_full_workload_every_element():
    """The full MXFP8 workload (outlier channels, packed documents) against
    the fp64 oracle on the exactly dequantised inputs, every element of out
    and lse."""
    inp = workloads.make_inputs("mxfp8_packed")
    cu = inp["cu_seqlens"]
    out, lse, ws = run_gpu(inp["q"], inp["k"], inp["v"], cu, True, inp["scale"],
                           dtype=A.ATTN_MXFP8, max_seqlen=max(inp["lengths"]))
    assert A.attn_get_device_error(ws) == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    ro, rl = full_reference(_deq(inp["q"]), _deq(inp["k"]), _deq(inp["v"]), inp["lengths"],
                            True, inp["scale"])
    e = np.abs(out.double().numpy() - ro)
    assert e.max() <= MXFP8_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


def test_mxfp8_repeat_runs_bit_identical():
    """Repeated runs of the whole MXFP8 path (quantisation pre-pass and the
    block-scaled kernel) agree bit for bit: each row is computed by one CTA in
    a fixed order."""
    inp = workloads.make_inputs("mxfp8_packed")
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    cu = inp["cu_seqlens"].to(dev)
    T, H, d = q.shape
    ms = max(inp["lengths"])
    ws = A.make_workspace(A.Shape(T, len(inp["lengths"]), H, d, ms), A.ATTN_MXFP8, dev)
    first = None
    for _ in range(3):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=dev)
        A.attn_fwd(q, k, v, cu, out, lse, True, inp["scale"], dtype=A.ATTN_MXFP8,
                   workspace=ws, max_seqlen=ms)
        torch.cuda.synchronize()
        assert A.attn_get_device_error(ws) == 0
        if first is None:
            first = (out.clone(), lse.clone())
        else:
            assert torch.equal(out.view(torch.int16), first[0].view(torch.int16))
            assert torch.equal(lse.view(torch.int32), first[1].view(torch.int32))

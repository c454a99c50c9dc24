"""Edge cases of the block-scaled forward forms (MXFP8, NVFP4 / FP8 mixed,
incoherent MXFP8) at head dim 128, where the kernel uses 112-key tiles while
the query tiles stay 128 rows: document lengths on and around multiples of
112 and 128 (so the causal diagonal falls on either side of a key-tile edge,
and a key tile reaches past the document's end), a dense batch (no
cu_seqlens), and repeated runs.  Every element is compared with the fp64
oracle run on the exactly dequantised operands ("FlashAttention và IO",
section "Bài tập kiểm tính đúng trước khi đo tốc độ": check every output
against a plain reference before timing; FLAMIA page, section "FLAMIA
Mimarisi ve Temel Tasarım İlkeleri": block-scaled products whose scales stay
inside one token)."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads
from oracle.attention import ref_attention
from oracle.incoherent import incoherent_operands
from oracle.mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref
from oracle.nvfp4 import dequantize_nvfp4_ref, quantize_nvfp4_ref
from helpers import BF16_MEAN_ABS, LSE_ABS, MXFP8_MAX_ABS, run_gpu

pytestmark = pytest.mark.gpu

# on, just below and just past multiples of 112 and 128 keys
EDGE_LENGTHS = [111, 112, 113, 127, 128, 129, 224, 225, 255, 256, 257, 336, 337, 448, 449]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    A.lib()


def _inputs(lengths, H, seed, outliers=True):
    g = torch.Generator("cpu").manual_seed(seed)
    T = sum(lengths)
    x = [torch.randn([T, H, 128], generator=g) for _ in range(3)]
    if outliers:
        for t in x[:2]:
            t[:, :, 5] *= 20
            t[:, :, 70] *= 20
    return [t.bfloat16() for t in x]


def _mx(x):
    return dequantize_mxfp8_ref(*quantize_mxfp8_ref(x.double().numpy()))


def _nv(x):
    return dequantize_nvfp4_ref(*quantize_nvfp4_ref(x.double().numpy()))


def _check(out, lse, ro, rl):
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    e = np.abs(out.double().numpy() - ro)
    assert e.max() <= MXFP8_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse.double().numpy() - rl).max() <= LSE_ABS


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("form", ["mxfp8", "nvfp4"])
def test_key_tile_edges(form, causal):
    q, k, v = _inputs(EDGE_LENGTHS, 2, seed=401)
    cu = workloads.cu_from_lengths(EDGE_LENGTHS)
    scale = 1.0 / math.sqrt(128)
    dtype = A.ATTN_MXFP8 if form == "mxfp8" else A.ATTN_NVFP4
    out, lse, ws = run_gpu(q, k, v, cu, causal, scale, dtype=dtype)
    assert A.attn_get_device_error(ws) == 0
    qk = _mx if form == "mxfp8" else _nv
    ro, rl = ref_attention(qk(q), qk(k), _mx(v), cu.numpy(), causal, scale)
    _check(out, lse, ro, rl)


@pytest.mark.parametrize("causal", [True, False])
def test_incoherent_key_tile_edges(causal):
    q, k, v = _inputs(EDGE_LENGTHS, 2, seed=402)
    cu = workloads.cu_from_lengths(EDGE_LENGTHS)
    scale = 1.0 / math.sqrt(128)
    signs = workloads.draw_signs(403, 128)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((2, q.shape[0]), float("nan"), dtype=torch.float32, device=dev)
    ws = A.attn_fwd_incoherent(qd, kd, vd, cu.to(dev), out, lse, causal, scale, signs.to(dev),
                               max_seqlen=max(EDGE_LENGTHS))
    torch.cuda.synchronize()
    assert A.attn_get_device_error(ws) == 0
    qr, kr, vr, s = incoherent_operands(q.double().numpy(), k.double().numpy(),
                                        v.double().numpy(), scale, signs.numpy())
    ro, rl = ref_attention(qr, kr, vr, cu.numpy(), causal, s)
    _check(out.cpu(), lse.cpu(), ro, rl)


@pytest.mark.parametrize("form", ["mxfp8", "nvfp4"])
def test_dense_batch_without_cu_seqlens(form):
    """B = 3 documents of 337 tokens given as one dense batch (no cu_seqlens)
    equal the same documents given through cu_seqlens, bit for bit, and match
    the oracle."""
    B, N = 3, 337
    q, k, v = _inputs([B * N], 2, seed=404)
    dtype = A.ATTN_MXFP8 if form == "mxfp8" else A.ATTN_NVFP4
    scale = 1.0 / math.sqrt(128)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    out = torch.empty_like(qd)
    lse = torch.empty((2, B * N), dtype=torch.float32, device=dev)
    ws = A.attn_fwd(qd, kd, vd, None, out, lse, True, scale, dtype=dtype, max_seqlen=N,
                    num_seqs=B)
    torch.cuda.synchronize()
    assert A.attn_get_device_error(ws) == 0
    cu = workloads.cu_from_lengths([N] * B)
    out2, lse2, ws2 = run_gpu(q, k, v, cu, True, scale, dtype=dtype)
    assert A.attn_get_device_error(ws2) == 0
    assert torch.equal(out.cpu().view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse.cpu(), lse2)
    qk = _mx if form == "mxfp8" else _nv
    ro, rl = ref_attention(qk(q), qk(k), _mx(v), cu.numpy(), True, scale)
    _check(out2, lse2, ro, rl)


@pytest.mark.parametrize("form", ["nvfp4", "incoherent"])
def test_repeat_runs_bit_identical(form):
    """Each row is computed by one CTA in a fixed order: repeated calls on
    the same inputs give the same bits (the pre-pass included)."""
    lengths = [700, 129, 1000, 1]
    q, k, v = _inputs(lengths, 4, seed=405)
    cu = workloads.cu_from_lengths(lengths)
    scale = 1.0 / math.sqrt(128)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    cud = cu.to(dev)
    signs = workloads.draw_signs(406, 128).to(dev)
    outs = []
    for _ in range(3):
        out = torch.empty_like(qd)
        lse = torch.empty((4, q.shape[0]), dtype=torch.float32, device=dev)
        if form == "incoherent":
            ws = A.attn_fwd_incoherent(qd, kd, vd, cud, out, lse, True, scale, signs,
                                       max_seqlen=max(lengths))
        else:
            ws = A.attn_fwd(qd, kd, vd, cud, out, lse, True, scale, dtype=A.ATTN_NVFP4,
                            max_seqlen=max(lengths))
        torch.cuda.synchronize()
        assert A.attn_get_device_error(ws) == 0
        outs.append((out.cpu().view(torch.int16), lse.cpu()))
    for o, l_ in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l_, outs[0][1])

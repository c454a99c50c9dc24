"""GPU parity of the bf16 attention path (through the C ABI) against the fp64
oracle: element by element on small and ragged cases and on every element of
the full-size workloads (sampled rows as a fast path), and bit-exact on
everything the masking and the document offsets decide."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads
from oracle.attention import ref_attention, ref_attention_rows, visible_count
from oracle.schedule import schedule_ref
from helpers import (BF16_MAX_ABS, BF16_MEAN_ABS, LSE_ABS, errors, run_gpu)
from oracle_pool import full_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    A.lib()


def _pack(lengths, H, d, seed, q_scale=1.0):
    g = torch.Generator("cpu").manual_seed(seed)
    T = sum(lengths)
    q = (torch.randn([T, H, d], generator=g) * q_scale).to(torch.bfloat16)
    k = torch.randn([T, H, d], generator=g).to(torch.bfloat16)
    v = torch.randn([T, H, d], generator=g).to(torch.bfloat16)
    return q, k, v, workloads.cu_from_lengths(lengths)


def _oracle(q, k, v, cu, causal, scale):
    return ref_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                         cu.numpy(), causal, scale)


def _check(out, lse, ref_out, ref_lse, cu):
    # rows of empty documents do not exist; every token belongs to a document
    mx, mean, le = errors(out, lse, ref_out, ref_lse)
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS and le <= LSE_ABS, (mx, mean, le)
    return mx, mean, le


# ---------------------------------------------------------------- worked case
def test_worked_example_on_gpu():
    """Scores [0, ln 2] and values [1, 3] must give 7/3 and lse = ln 3
    ("FlashAttention và IO", section "Softmax qua nhiều khối cần thống kê chạy")."""
    d = 64
    q = torch.zeros([2, 1, d]); q[1, 0, 0] = 1.0
    k = torch.zeros([2, 1, d]); k[1, 0, 0] = 1.0
    v = torch.zeros([2, 1, d]); v[0] = 1.0; v[1] = 3.0
    scale = float(torch.tensor(math.log(2.0), dtype=torch.float32))
    for causal in (False, True):
        out, lse, _ = run_gpu(q.bfloat16(), k.bfloat16(), v.bfloat16(),
                              torch.tensor([0, 2], dtype=torch.int32), causal, scale)
        assert torch.all(out[1, 0].float() == 2.328125)        # bf16(7/3)
        assert abs(float(lse[0, 1]) - math.log(3.0)) <= 1e-3
    out, lse, _ = run_gpu(q.bfloat16(), k.bfloat16(), v.bfloat16(),
                          torch.tensor([0, 2], dtype=torch.int32), True, scale)
    assert torch.all(out[0, 0].float() == 1.0) and abs(float(lse[0, 0])) <= 1e-6


# ---------------------------------------------------------------- small exact cases
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload(causal):
    inp = workloads.make_inputs("tiny")
    out, lse, _ = run_gpu(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], causal, inp["scale"])
    ro, rl = _oracle(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], causal, inp["scale"])
    _check(out, lse, ro, rl, inp["cu_seqlens"])


RAGGED = [1, 127, 128, 129, 0, 255, 256, 257, 300, 513, 2, 64, 384]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_pack(d, causal):
    q, k, v, cu = _pack(RAGGED, 3, d, seed=10 + d + causal)
    scale = 1.0 / math.sqrt(d)
    out, lse, _ = run_gpu(q, k, v, cu, causal, scale)
    ro, rl = _oracle(q, k, v, cu, causal, scale)
    _check(out, lse, ro, rl, cu)


def test_dense_mode_matches_packed():
    """cu_seqlens = NULL (B equal documents) gives the same bits as the
    explicit offsets of the same documents."""
    q, k, v, _ = _pack([384] * 3, 2, 128, seed=3)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    outs = []
    for cu in (None, workloads.cu_from_lengths([384] * 3).to(dev)):
        out = torch.empty_like(qd)
        lse = torch.empty((2, 1152), dtype=torch.float32, device=dev)
        A.attn_fwd(qd, kd, vd, cu, out, lse, True, 0.1, max_seqlen=384, num_seqs=3)
        outs.append((out.cpu(), lse.cpu()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("d", [64, 128])
def test_forced_rescales(d):
    """Scores that grow along the keys (q_i close to a fixed direction u,
    k_j = ramp_j * u) make every row's running maximum rise by more than the
    lazy threshold many times; the result stays exact, and repeated runs are
    bit-identical (O is rescaled between products, never while one runs)."""
    lengths = [700, 1030]
    T, H = sum(lengths), 2
    g = torch.Generator("cpu").manual_seed(21)
    q = (1.0 + 0.1 * torch.randn([T, H, d], generator=g)).bfloat16()
    ramp = torch.linspace(0.2, 6.0, T)[:, None, None]
    k = (ramp * torch.ones([T, H, d])).bfloat16()
    v = torch.randn([T, H, d], generator=g).bfloat16()
    cu = workloads.cu_from_lengths(lengths)
    sc = 0.09 * math.sqrt(128 / d)
    for causal in (False, True):
        out, lse, _ = run_gpu(q, k, v, cu, causal, sc)
        ro, rl = _oracle(q, k, v, cu, causal, sc)
        _check(out, lse, ro, rl, cu)
        out2, lse2, _ = run_gpu(q, k, v, cu, causal, sc)
        assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
        assert torch.equal(lse2.view(torch.int32), lse.view(torch.int32))


# ---------------------------------------------------------------- bit-exact masking
@pytest.mark.parametrize("causal", [False, True])
def test_masking_counts_bit_exact(causal):
    """With Q = 0 every visible key has weight exactly 1, so exp(lse) is the
    number of keys each row sees; rounded it must equal the oracle's count
    for every row and head."""
    q, k, v, cu = _pack(RAGGED, 2, 128, seed=4)
    q = torch.zeros_like(q)
    _, lse, _ = run_gpu(q, k, v, cu, causal, 0.088)
    cnt = visible_count(cu.numpy(), causal)
    got = np.rint(np.exp(lse.double().numpy()))
    np.testing.assert_array_equal(got, np.broadcast_to(cnt, got.shape))


def test_packing_order_bit_identical():
    """Tiles are counted from each document's start, so permuting documents in
    the pack permutes the output rows bit for bit."""
    lengths = [300, 129, 1, 640, 77]
    q, k, v, cu = _pack(lengths, 2, 128, seed=5)
    out, lse, _ = run_gpu(q, k, v, cu, True, 0.088)
    perm = [3, 0, 4, 2, 1]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    idx = torch.from_numpy(np.concatenate([np.arange(starts[p], starts[p + 1]) for p in perm]))
    cu2 = workloads.cu_from_lengths([lengths[p] for p in perm])
    out2, lse2, _ = run_gpu(q[idx], k[idx], v[idx], cu2, True, 0.088)
    assert torch.equal(out2, out[idx]) and torch.equal(lse2, lse[:, idx])


def test_no_causal_leakage():
    """Changing tokens after position i of a document, or any token of another
    document, leaves rows <= i of that document bit-identical."""
    lengths = [200, 450, 90]
    q, k, v, cu = _pack(lengths, 2, 128, seed=6)
    out, lse, _ = run_gpu(q, k, v, cu, True, 0.088)
    i = 200 + 260            # inside document 1
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    g = torch.Generator("cpu").manual_seed(99)
    for t in (q2, k2, v2):
        t[i + 1:650] = (torch.randn(t[i + 1:650].shape, generator=g) * 3).bfloat16()
        t[:200] = (torch.randn(t[:200].shape, generator=g) * 3).bfloat16()
        t[650:] = (torch.randn(t[650:].shape, generator=g) * 3).bfloat16()
    out2, lse2, _ = run_gpu(q2, k2, v2, cu, True, 0.088)
    assert torch.equal(out2[200:i + 1], out[200:i + 1])
    assert torch.equal(lse2[:, 200:i + 1], lse[:, 200:i + 1])


# ---------------------------------------------------------------- offsets and schedule
def test_schedule_matches_oracle():
    for causal in (False, True):
        lengths = [1, 700, 0, 256, 257, 4000, 31]
        q, k, v, cu = _pack(lengths, 1, 64, seed=7)
        _, _, ws = run_gpu(q, k, v, cu, causal, 0.125)
        hdr = ws[:8].cpu().view(torch.int32)
        n = int(hdr[1])
        got = ws[256:256 + 16 * n].cpu().view(torch.int32).reshape(n, 4).numpy()
        np.testing.assert_array_equal(got, schedule_ref(cu.numpy(), causal, 2))   # bf16: pairs of query tiles
        assert A.attn_get_device_error(ws) == 0


@pytest.mark.parametrize("bad", ["first", "last", "decreasing", "too_long"])
def test_bad_seqlens_reported_output_untouched(bad):
    lengths = [100, 200, 300]
    q, k, v, cu = _pack(lengths, 2, 64, seed=8)
    cu = cu.clone()
    max_seqlen = 300
    if bad == "first":
        cu[0] = 1
    elif bad == "last":
        cu[-1] = 599
    elif bad == "decreasing":
        cu[1] = 350
    else:
        max_seqlen = 250
    out, lse, ws = run_gpu(q, k, v, cu, True, 0.125, max_seqlen=max_seqlen)
    assert torch.isnan(out.float()).all() and torch.isnan(lse).all()   # untouched
    assert A.attn_get_device_error(ws) == 5
    assert A.attn_get_device_error(ws) == 0                            # cleared


def test_empty_documents_only_and_zero_tokens():
    dev = torch.device("cuda:0")
    x = torch.empty((0, 2, 64), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((2, 0), dtype=torch.float32, device=dev)
    A.attn_fwd(x, x, x, torch.zeros(3, dtype=torch.int32, device=dev), x, lse, True, 0.1,
               max_seqlen=0)
    torch.cuda.synchronize()


# ---------------------------------------------------------------- full sizes
def _sample_rows(lengths, H, n, seed):
    rng = np.random.default_rng(seed)
    starts = np.concatenate([[0], np.cumsum(lengths)])
    T = int(starts[-1])
    toks = set(rng.integers(0, T, n).tolist())
    for a, b in zip(starts[:-1], starts[1:]):          # document edges and tile edges
        for off in (0, 1, 127, 128, 255, 256):
            if a + off < b:
                toks.add(int(a + off))
        if b > a:
            toks.add(int(b - 1))
    toks = np.array(sorted(toks))
    heads = rng.integers(0, H, len(toks))
    return toks, heads


@pytest.mark.parametrize("name", ["dense_causal", "packed_causal", "long_outlier"])
def test_full_workload_every_element(name):
    """The full-size workloads in the launch configuration bench.py times,
    compared with the fp64 oracle on every element of out and lse (every
    (document, head) problem, computed in a spawned process pool)."""
    inp = workloads.make_inputs(name)
    cu = inp["cu_seqlens"]
    out, lse, ws = run_gpu(inp["q"], inp["k"], inp["v"], cu, True, inp["scale"],
                           max_seqlen=max(inp["lengths"]))
    assert A.attn_get_device_error(ws) == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    ro, rl = full_reference(inp["q"].double().numpy(), inp["k"].double().numpy(),
                            inp["v"].double().numpy(), inp["lengths"], True, inp["scale"])
    mx, mean, le = errors(out, lse, ro, rl)
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS and le <= LSE_ABS, (mx, mean, le)


@pytest.mark.parametrize("name", ["dense_causal", "packed_causal"])
def test_full_workload_sampled_rows(name):
    """Fast path of the check above: sampled rows (every document's edges and
    tile edges plus random rows), each computed on its own by the oracle."""
    inp = workloads.make_inputs(name)
    w = inp["workload"]
    cu = inp["cu_seqlens"]
    out, lse, ws = run_gpu(inp["q"], inp["k"], inp["v"], cu, True, inp["scale"],
                           max_seqlen=max(inp["lengths"]))
    assert A.attn_get_device_error(ws) == 0
    toks, heads = _sample_rows(inp["lengths"], w.heads, 384, seed=1)
    ro, rl = ref_attention_rows(inp["q"].double().numpy(), inp["k"].double().numpy(),
                                inp["v"].double().numpy(), cu.numpy(), True, inp["scale"],
                                toks, heads)
    e = np.abs(out[toks, heads].double().numpy() - ro)
    assert e.max() <= BF16_MAX_ABS and e.mean() <= BF16_MEAN_ABS, (e.max(), e.mean())
    assert np.abs(lse[heads, toks].double().numpy() - rl).max() <= LSE_ABS


@pytest.mark.parametrize("name", ["packed_causal", "long_outlier"])
def test_repeat_runs_bit_identical(name):
    """Each output row is computed by one CTA in a fixed order (no atomics, no
    split reductions), so repeated runs agree bit for bit whatever order the
    units are claimed in.  A difference exposes a synchronisation fault, e.g.
    O read or rescaled while a P V product is still in flight."""
    inp = workloads.make_inputs(name)
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    cu = inp["cu_seqlens"].to(dev)
    T, H, d = q.shape
    ws = A.make_workspace(A.Shape(T, len(inp["lengths"]), H, d, max(inp["lengths"])),
                          A.ATTN_BF16, dev)
    first = None
    for _ in range(3):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=dev)
        A.attn_fwd(q, k, v, cu, out, lse, True, inp["scale"], workspace=ws,
                   max_seqlen=max(inp["lengths"]))
        torch.cuda.synchronize()
        assert A.attn_get_device_error(ws) == 0
        if first is None:
            first = (out.clone(), lse.clone())
        else:
            assert torch.equal(out.view(torch.int16), first[0].view(torch.int16))
            assert torch.equal(lse.view(torch.int32), first[1].view(torch.int32))


def test_many_documents_unsorted_schedule():
    """18000 one-token documents and three longer ones: more work-list
    entries than the schedule builder sorts in shared memory (16384), so the
    list stays in document order; every row is still right (a one-token
    document's output is its own value row and its lse its own score)."""
    lengths = [1] * 18000 + [300, 129, 700]
    q, k, v, cu = _pack(lengths, 1, 64, seed=21)
    out, lse, ws = run_gpu(q, k, v, cu, True, 0.125, max_seqlen=700)
    assert A.attn_get_device_error(ws) == 0
    hdr = ws[:8].cpu().view(torch.int32)
    assert int(hdr[1]) == 18000 + 2 + 1 + 3        # pairs of query tiles
    # one-token documents: exact
    assert torch.equal(out[:18000], v[:18000])
    s = (q[:18000, 0].double() * k[:18000, 0].double()).sum(-1) * 0.125
    assert np.abs(lse[0, :18000].double().numpy() - s.numpy()).max() <= 1e-4
    # the long documents against the oracle
    sub = slice(18000, None)
    ro, rl = _oracle(q[sub], k[sub], v[sub], workloads.cu_from_lengths([300, 129, 700]), True, 0.125)
    _check(out[sub], lse[:, sub], ro, rl, None)

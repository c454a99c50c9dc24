"""The seeded input generators: deterministic, and shaped as the workloads
state (document length range, exact pack size, outlier channels)."""
import torch

from exact_tiled_attention_39_b200 import workloads


def test_tiny_deterministic_and_shaped():
    a = workloads.make_inputs("tiny")
    b = workloads.make_inputs("tiny")
    for n in ("q", "k", "v"):
        assert a[n].dtype == torch.bfloat16 and a[n].shape == (256, 2, 64)
        assert torch.equal(a[n], b[n])
    assert a["cu_seqlens"].tolist() == [0, 256]
    assert a["scale"] == 0.125


def test_packed_lengths():
    g = torch.Generator("cpu").manual_seed(2)
    L = workloads.draw_doc_lengths(g, 16384, 128, 4096)
    assert sum(L) == 16384
    assert all(128 <= x <= 4096 for x in L[:-1]) and 1 <= L[-1] <= 4096
    cu = workloads.cu_from_lengths(L)
    assert cu.dtype == torch.int32 and int(cu[-1]) == 16384


def test_outlier_channels_scaled():
    w = workloads.Workload(name="t", seed=9, heads=2, head_dim=128, causal=(True,),
                           batch=1, seq_len=64, outlier_channels=(5, 70),
                           outlier_factor=20.0)
    x = workloads.make_inputs(w)
    q = x["q"].float()
    ratio = q[:, :, 5].abs().mean() / q[:, :, 6].abs().mean()
    assert ratio > 10
    assert x["v"].float()[:, :, 5].abs().mean() < 2


def test_flop_convention():
    assert workloads.flops([4096] * 4, 16, 128, True) == 2 * 4096 ** 2 * 128 * 64
    assert workloads.flops([10, 20], 1, 8, False) == 4 * 8 * (100 + 400)

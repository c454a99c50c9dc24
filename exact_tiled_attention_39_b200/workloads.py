"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle
checks.  This module only draws random numbers and lays them out: it holds
none of the attention or quantisation arithmetic.

Recipe (the pages give no data; all inputs are synthetic):
  * RNG: ``torch.Generator('cpu').manual_seed(seed)``;
  * packed workloads first draw document lengths one at a time with
    ``torch.randint(lo, hi + 1)`` until their sum reaches the pack size, then
    cut the last document so the sum is exact (it may end up shorter than
    ``lo``);
  * then Q, K, V are drawn in that order as ``torch.randn([T, H, d])`` in
    fp32; outlier channels (when the workload has them) of Q and K are
    multiplied by their factor in fp32; finally each tensor is rounded to
    bf16 (round to nearest even).
  * the softmax scale is 1/sqrt(d) rounded to fp32.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "draw_doc_lengths",
           "cu_from_lengths", "tensor_sha256", "flops", "draw_signs"]


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    heads: int
    head_dim: int
    causal: tuple[bool, ...]
    # dense: batch docs of seq_len tokens; packed: pack_tokens split at random
    batch: int = 0
    seq_len: int = 0
    pack_tokens: int = 0
    doc_len_range: tuple[int, int] = (0, 0)
    outlier_channels: tuple[int, ...] = ()
    outlier_factor: float = 1.0
    dtype: str = "bf16"
    incoherent: bool = False      # MXFP8 with Q, K rotated by random signs + Hadamard
    description: str = ""
    extras: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", seed=0, heads=2, head_dim=64, causal=(False, True),
        batch=1, seq_len=256,
        description="B=1 H=2 N=256 d=64, N(0,1) bf16, causal and non-causal"),
    "dense_causal": Workload(
        name="dense_causal", seed=1, heads=16, head_dim=128, causal=(True,),
        batch=4, seq_len=4096,
        description="B=4 H=16 N=4096 d=128 causal bf16"),
    "packed_causal": Workload(
        name="packed_causal", seed=2, heads=32, head_dim=128, causal=(True,),
        pack_tokens=16384, doc_len_range=(128, 4096),
        description="one pack of 16384 tokens, doc lengths U[128,4096], "
                    "H=32 d=128, block-diagonal causal bf16"),
    "long_outlier": Workload(
        name="long_outlier", seed=3, heads=16, head_dim=128, causal=(True,),
        batch=1, seq_len=32768, outlier_channels=(5, 70), outlier_factor=20.0,
        description="B=1 H=16 N=32768 d=128 causal bf16, channels 5 and 70 "
                    "of Q and K x20"),
    "mxfp8_packed": Workload(
        name="mxfp8_packed", seed=4, heads=32, head_dim=128, causal=(True,),
        pack_tokens=16384, doc_len_range=(128, 4096),
        outlier_channels=(5, 70), outlier_factor=20.0, dtype="mxfp8",
        description="packed as packed_causal (seed 4) with the outlier "
                    "channels of long_outlier, MXFP8"),
    "nvfp4_packed": Workload(
        name="nvfp4_packed", seed=4, heads=32, head_dim=128, causal=(True,),
        pack_tokens=16384, doc_len_range=(128, 4096),
        outlier_channels=(5, 70), outlier_factor=20.0, dtype="nvfp4",
        description="the mxfp8_packed inputs on the mixed path: Q, K in NVFP4, "
                    "V in MXFP8"),
    "mxfp8_incoherent": Workload(
        name="mxfp8_incoherent", seed=4, heads=32, head_dim=128, causal=(True,),
        pack_tokens=16384, doc_len_range=(128, 4096),
        outlier_channels=(5, 70), outlier_factor=20.0, dtype="mxfp8", incoherent=True,
        description="the mxfp8_packed inputs with incoherent processing (Q, K "
                    "rotated by random signs and a Hadamard matrix before "
                    "quantisation; signs from seed 1004)"),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def draw_doc_lengths(g: torch.Generator, total: int, lo: int, hi: int) -> list[int]:
    lengths: list[int] = []
    s = 0
    while s < total:
        L = int(torch.randint(lo, hi + 1, (1,), generator=g).item())
        lengths.append(L)
        s += L
    lengths[-1] -= s - total
    return lengths


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def make_inputs(w: Workload | str, heads: int | None = None,
                seq_scale: float | None = None) -> dict:
    """Draw the workload's inputs on the CPU.

    ``heads`` (optional) keeps only the first heads of the drawn tensors, for
    bounded CPU timing samples; the draw itself is unchanged.
    Returns a dict with bf16 q, k, v [T, H, d], int32 cu_seqlens, the fp32
    scale as a Python float, the document lengths and the token count.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    g = torch.Generator("cpu").manual_seed(w.seed)
    if w.pack_tokens:
        lengths = draw_doc_lengths(g, w.pack_tokens, *w.doc_len_range)
    else:
        lengths = [w.seq_len] * w.batch
    T = sum(lengths)
    H, d = w.heads, w.head_dim
    out = {}
    for name in ("q", "k", "v"):
        x = torch.randn([T, H, d], generator=g, dtype=torch.float32)
        if name in ("q", "k") and w.outlier_channels:
            for c in w.outlier_channels:
                x[:, :, c] *= w.outlier_factor
        out[name] = x.to(torch.bfloat16)
    if heads is not None:
        for name in ("q", "k", "v"):
            out[name] = out[name][:, :heads, :].contiguous()
    out["cu_seqlens"] = cu_from_lengths(lengths)
    out["lengths"] = lengths
    out["tokens"] = T
    out["scale"] = float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32).item())
    out["workload"] = w
    if w.incoherent:
        out["signs"] = draw_signs(1000 + w.seed, d)
    return out


def draw_signs(seed: int, d: int) -> torch.Tensor:
    """d random signs (+1 / -1, fp32) from their own seeded generator: the
    random draw incoherent processing takes as an input."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.where(torch.rand(d, generator=g) < 0.5, -1.0, 1.0).to(torch.float32)


def tensor_sha256(t: torch.Tensor) -> str:
    return hashlib.sha256(t.contiguous().view(torch.uint8).numpy().tobytes()).hexdigest()


def flops(lengths, heads: int, head_dim: int, causal: bool) -> float:
    """Algorithmic FLOPs of the forward: 4 L^2 d per head and document,
    halved when causal (the stated counting convention, not L(L+1)/2)."""
    per_head = sum(4.0 * L * L * head_dim for L in lengths)
    if causal:
        per_head /= 2.0
    return per_head * heads

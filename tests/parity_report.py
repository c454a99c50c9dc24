"""Parity figures of the five configurations, the NVFP4 / FP8 mixed path and
incoherent processing, one JSON line each (GPU).

    python tests/parity_report.py [--bwd-only]

Runs every configuration through the C ABI and compares with the fp64 oracle
the way the GPU tests do: the tiny config element by element (causal and
non-causal), the large ones too (every (document, head) problem in a spawned
process pool), MXFP8 against the oracle on the exactly dequantised inputs.  Prints
max / mean absolute output error, max absolute lse error and the tolerance
each is held to.  Then the backward on the GPU tests' cases, every element of
dq, dk, dv against the fp64 gradient oracle, errors relative to each
gradient's largest magnitude.  Test infrastructure, like the oracle it
calls.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

from exact_tiled_attention_39_b200 import attn as A  # noqa: E402
from exact_tiled_attention_39_b200 import workloads  # noqa: E402
from oracle.attention import ref_attention  # noqa: E402
from oracle.attention_bwd import ref_attention_bwd  # noqa: E402
from oracle.mxfp8 import dequantize_mxfp8_ref, quantize_mxfp8_ref  # noqa: E402
from helpers import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_ABS, MXFP8_MAX_ABS, run_gpu  # noqa: E402
from oracle_pool import full_reference  # noqa: E402


def deq(x):
    c, s = quantize_mxfp8_ref(x.double().numpy())
    return dequantize_mxfp8_ref(c, s)


def line(name, rows, e, le, max_tol, mean_tol):
    return {"config": name, "rows_compared": int(rows), "max_abs": float(e.max()),
            "mean_abs": float(e.mean()), "lse_max_abs": float(le.max()),
            "tol": {"max_abs": max_tol, "mean_abs": mean_tol, "lse": LSE_ABS},
            "pass": bool(e.max() <= max_tol and (mean_tol is None or e.mean() <= mean_tol)
                         and le.max() <= LSE_ABS)}


def bwd_lines():
    import math
    from test_gpu_bwd import BWD_REL_MAX, BWD_REL_MEAN
    lines = []
    cases = [("bwd tiny-shape (L256 H2 d64)", [256], 2, 64),
             ("bwd ragged packed (7 docs, H2 d64)", [1, 130, 300, 129, 64, 256, 44], 2, 64),
             ("bwd ragged packed (7 docs, H2 d128)", [1, 130, 300, 129, 64, 256, 44], 2, 128),
             ("bwd one document L2048 H2 d128", [2048], 2, 128)]
    dev = torch.device("cuda:0")
    for name, lengths, H, d in cases:
        for causal in (True, False):
            g = torch.Generator().manual_seed(21)
            T = sum(lengths)
            q, k, v, do = (torch.randn((T, H, d), generator=g).to(torch.bfloat16)
                           for _ in range(4))
            scale = 1.0 / math.sqrt(d)
            cu = workloads.cu_from_lengths(lengths)
            qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
            cud = cu.to(dev)
            out = torch.empty_like(qd)
            lse = torch.empty((H, T), dtype=torch.float32, device=dev)
            A.attn_fwd(qd, kd, vd, cud, out, lse, causal, scale, max_seqlen=max(lengths))
            grads = [torch.empty_like(qd) for _ in range(3)]
            A.attn_bwd(qd, kd, vd, out, dod, lse, cud, *grads, causal, scale,
                       max_seqlen=max(lengths))
            torch.cuda.synchronize()
            ref = ref_attention_bwd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    do.double().numpy(), cu.numpy(), causal, scale)
            rec = {"config": f"{name}, {'causal' if causal else 'non-causal'}",
                   "tol_rel": {"max": BWD_REL_MAX, "mean": BWD_REL_MEAN}}
            ok = True
            for gname, got, rf in zip(("dq", "dk", "dv"), grads, ref):
                e = np.abs(got.cpu().double().numpy() - rf)
                m = float(np.abs(rf).max())
                rec[gname] = {"max_abs": float(e.max()), "mean_abs": float(e.mean()),
                              "max_ref": m, "max_rel": float(e.max()) / m,
                              "mean_rel": float(e.mean()) / m}
                ok &= e.max() <= BWD_REL_MAX * m and e.mean() <= BWD_REL_MEAN * m
            rec["pass"] = bool(ok)
            lines.append(rec)
    return lines


def main():
    if "--bwd-only" in sys.argv:
        lines = bwd_lines()
        for l_ in lines:
            print(json.dumps(l_))
        return 0 if all(l_["pass"] for l_ in lines) else 1
    out_lines = []
    inp = workloads.make_inputs("tiny")
    for causal in (False, True):
        out, lse, _ = run_gpu(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], causal,
                              inp["scale"])
        ro, rl = ref_attention(inp["q"].double().numpy(), inp["k"].double().numpy(),
                               inp["v"].double().numpy(), inp["cu_seqlens"].numpy(), causal,
                               inp["scale"])
        e = np.abs(out.double().numpy() - ro)
        le = np.abs(lse.double().numpy() - rl)
        out_lines.append(line(f"tiny ({'causal' if causal else 'non-causal'})",
                              ro.shape[0] * ro.shape[1], e, le, BF16_MAX_ABS, BF16_MEAN_ABS))
    for name in ("dense_causal", "packed_causal", "long_outlier", "mxfp8_packed"):
        inp = workloads.make_inputs(name)
        cu = inp["cu_seqlens"]
        fp8 = name.startswith("mxfp8")
        out, lse, _ = run_gpu(inp["q"], inp["k"], inp["v"], cu, True, inp["scale"],
                              dtype=A.ATTN_MXFP8 if fp8 else A.ATTN_BF16,
                              max_seqlen=max(inp["lengths"]))
        if fp8:
            q, k, v = deq(inp["q"]), deq(inp["k"]), deq(inp["v"])
        else:
            q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
        ro, rl = full_reference(q, k, v, inp["lengths"], True, inp["scale"])
        e = np.abs(out.double().numpy() - ro)
        le = np.abs(lse.double().numpy() - rl)
        out_lines.append(line(name, ro.shape[0] * ro.shape[1], e, le,
                              MXFP8_MAX_ABS if fp8 else BF16_MAX_ABS, BF16_MEAN_ABS))
    # NVFP4 Q, K with MXFP8 V, against the oracle on the exactly dequantised inputs
    from oracle.nvfp4 import dequantize_nvfp4_ref, quantize_nvfp4_ref
    inp = workloads.make_inputs("nvfp4_packed")
    out, lse, _ = run_gpu(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], True, inp["scale"],
                          dtype=A.ATTN_NVFP4, max_seqlen=max(inp["lengths"]))
    qd = dequantize_nvfp4_ref(*quantize_nvfp4_ref(inp["q"].double().numpy()))
    kd = dequantize_nvfp4_ref(*quantize_nvfp4_ref(inp["k"].double().numpy()))
    ro, rl = full_reference(qd, kd, deq(inp["v"]), inp["lengths"], True, inp["scale"])
    out_lines.append(line("nvfp4_packed", ro.shape[0] * ro.shape[1],
                          np.abs(out.double().numpy() - ro), np.abs(lse.double().numpy() - rl),
                          MXFP8_MAX_ABS, BF16_MEAN_ABS))
    # incoherent processing, against the oracle of the rotated, quantised operands
    from oracle.incoherent import incoherent_operands
    from test_gpu_incoherent import _run_incoherent
    inp = workloads.make_inputs("mxfp8_incoherent")
    out, lse = _run_incoherent(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], True,
                               inp["scale"], inp["signs"], max(inp["lengths"]))
    q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
    qd, kd, vd, s = incoherent_operands(q, k, v, inp["scale"], inp["signs"].numpy())
    ro, rl = full_reference(qd, kd, vd, inp["lengths"], True, s)
    out_lines.append(line("mxfp8_incoherent", ro.shape[0] * ro.shape[1],
                          np.abs(out.double().numpy() - ro), np.abs(lse.double().numpy() - rl),
                          MXFP8_MAX_ABS, BF16_MEAN_ABS))
    out_lines += bwd_lines()
    for l_ in out_lines:
        print(json.dumps(l_))
    return 0 if all(l_["pass"] for l_ in out_lines) else 1


if __name__ == "__main__":
    if not torch.cuda.is_available():
        print(json.dumps({"skipped": "no CUDA device"}))
        sys.exit(0)
    sys.exit(main())

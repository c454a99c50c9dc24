"""Shared helpers for the GPU tests: run the C-ABI path on seeded inputs and
compare with the oracle."""
import numpy as np
import torch

from exact_tiled_attention_39_b200 import attn as A

# Tolerances the GPU path is held to (bf16 output; fp32 log-sum-exp).
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
MXFP8_MAX_ABS = 6e-2


def run_gpu(q, k, v, cu, causal, scale, dtype=A.ATTN_BF16, max_seqlen=None, workspace=None):
    """q, k, v: CPU bf16 [T, H, d]; cu: CPU int32 or None.  Returns CPU
    (out bf16, lse fp32, workspace)."""
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    T, H, d = q.shape
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((H, T), float("nan"), dtype=torch.float32, device=dev)
    cud = cu.to(dev) if cu is not None else None
    if max_seqlen is None:
        if cu is not None:
            max_seqlen = int((cu[1:] - cu[:-1]).max()) if cu.numel() > 1 else 0
        else:
            max_seqlen = T
    ws = A.attn_fwd(qd, kd, vd, cud, out, lse, causal, scale, dtype=dtype, workspace=workspace,
                    max_seqlen=max_seqlen, num_seqs=None if cu is not None else 1)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), ws


def errors(out, lse, ref_out, ref_lse):
    o = out.double().numpy()
    e = np.abs(o - ref_out)
    le = np.abs(lse.double().numpy() - ref_lse)
    return float(e.max()), float(e.mean()), float(le.max())

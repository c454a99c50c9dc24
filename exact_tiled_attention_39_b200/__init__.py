"""Exact tiled attention forward for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libattn.so`` built from ``csrc/``
(declared in ``include/attn.h``); ``exact_tiled_attention_39_b200.attn`` is the
thin ctypes binding over it.  Importing the package does not load the
library; the first call through the binding does, and raises if it is
missing.  There is no CPU fallback.
"""

__all__ = ["attn", "workloads"]

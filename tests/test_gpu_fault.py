"""Failure detection on the GPU without a fault: a build that never sends one
"scores ready" signal (the first unit's S_A) and waits at most 50 ms per
mbarrier wait.  The waiting warps give up, raise the CTA's abort flag, every
role leaves its loop (copies and products in flight are drained, TMEM is
freed) and the call reports ATTN_ERR_TIMEOUT through the workspace's error
word.  Afterwards the normal library on the same device still gives the
oracle's answer."""
import math
import time

import numpy as np
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A
from exact_tiled_attention_39_b200 import build, workloads
from oracle.attention import ref_attention
from helpers import BF16_MAX_ABS, errors, run_gpu

pytestmark = pytest.mark.gpu

ATTN_ERR_TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def test_wait_timeout_is_reported_and_device_stays_usable():
    path = build.build_variant("fault_drop_commit", {
        "ATTN_FAULT_DROP_FIRST_SCORE_COMMIT": "1",
        "ATTN_WAIT_TIMEOUT_NS": "50000000ull",
    })
    inp = workloads.make_inputs("tiny")
    saved = (A.LIB_PATH, A._lib)
    try:
        A.LIB_PATH, A._lib = path, None
        t0 = time.time()
        out, lse, ws = run_gpu(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], True,
                               inp["scale"])
        elapsed = time.time() - t0
        assert A.attn_get_device_error(ws) == ATTN_ERR_TIMEOUT
        assert elapsed < 30.0
    finally:
        A.LIB_PATH, A._lib = saved
    # the context is intact: the normal library still matches the oracle
    out, lse, _ = run_gpu(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], True, inp["scale"])
    ro, rl = ref_attention(inp["q"].double().numpy(), inp["k"].double().numpy(),
                           inp["v"].double().numpy(), inp["cu_seqlens"].numpy(), True,
                           inp["scale"])
    mx, mean, le = errors(out, lse, ro, rl)
    assert mx <= BF16_MAX_ABS and le <= 1e-3

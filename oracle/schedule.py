"""Work list of the schedule-build step (oracle; test infrastructure only).

The packed-document workload must be balanced across the GPU's SMs: FLAMIA
("FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin
Flash Mikro-Ölçeklemeli Dikkat Mekanizması", section "FLAMIA Mimarisi ve
Temel Tasarım İlkeleri") schedules uneven per-document work without
repacking, and FlashAttention-2 ("FlashAttention, pelatihan multi-GPU, dan
kuantisasi bobot", section 1) parallelises over the sequence with the outer
loop over query blocks.  The pages fix no tile size or grouping; the reading
taken (and implemented independently on the GPU) is:

  * a query tile is 128 rows of one document, counted from the document's
    first token; a work unit is ``tiles_per_unit`` consecutive query tiles
    (1 or 2; rows [128 q t, 128 q (t + 1)) of the document, q the number of
    tiles per unit) for one head;
  * a key/value tile is 128 keys, also counted from the document start;
  * the cost of a unit is the number of (query tile, key tile) products it
    needs: for each of its query tiles qb that starts inside the document,
    min(qb + 1, n_kv) when causal, n_kv otherwise, with n_kv = ceil(L / 128);
  * entries are sorted by cost, largest first; equal costs keep document
    order, then unit order (a stable sort);
  * each entry is (doc_start, doc_len, t, cost) as four int32.
"""
from __future__ import annotations

import numpy as np

BLOCK_M = 128
BLOCK_N = 128

__all__ = ["schedule_ref", "unit_cost", "BLOCK_M", "BLOCK_N"]


def unit_cost(L: int, t: int, causal: bool, tiles_per_unit: int = 1) -> int:
    """Number of (query tile, key tile) products of unit ``t`` of a document
    of length ``L``."""
    n_kv = -(-L // BLOCK_N)
    cost = 0
    for qb in range(tiles_per_unit * t, tiles_per_unit * (t + 1)):
        if qb * BLOCK_M < L:
            cost += min(qb + 1, n_kv) if causal else n_kv
    return cost


def schedule_ref(cu_seqlens, causal: bool, tiles_per_unit: int = 1) -> np.ndarray:
    """The work list as an int32 array of shape [n_entries, 4]."""
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    entries = []
    for i in range(len(cu) - 1):
        a, L = cu[i], cu[i + 1] - cu[i]
        n_units = -(-L // (BLOCK_M * tiles_per_unit))
        for t in range(n_units):
            entries.append((a, L, t, unit_cost(L, t, causal, tiles_per_unit)))
    entries.sort(key=lambda e: -e[3])     # Python's sort is stable
    return np.asarray(entries, dtype=np.int32).reshape(-1, 4)

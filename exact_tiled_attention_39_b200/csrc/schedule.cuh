// Schedule-build kernel: validates cu_seqlens on the device and writes the
// heaviest-first work list the attention kernel walks.
//
// "FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin
// Flash Mikro-Ölçeklemeli Dikkat Mekanizması", section "FLAMIA Mimarisi ve
// Temel Tasarım İlkeleri": packed variable-length documents are used in
// place and the uneven per-document work is scheduled.  "FlashAttention,
// pelatihan multi-GPU, dan kuantisasi bobot", section 1 (FlashAttention-2):
// work is split along the sequence into query blocks.
//
// One entry per unit of `tiles_per_unit` (1 or 2) consecutive 128-row query
// tiles of one document: (doc_start, doc_len, unit index, cost), cost = the
// number of (query tile, key tile) products of its tiles (causal:
// min(qb + 1, n_kv) per query tile qb; else n_kv).  Entries are sorted by
// cost, largest first, ties in document then unit order, with a bitonic sort
// of (cost, index) keys in shared memory.
#pragma once
#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"

namespace attn {

__device__ __forceinline__ int unit_cost(int L, int t, int causal, int tiles_per_unit) {
  const int n_kv = (L + kBlockN - 1) / kBlockN;
  int cost = 0;
  for (int i = 0; i < tiles_per_unit; ++i) {
    const int qb = tiles_per_unit * t + i;
    if (qb * kBlockM < L) cost += causal ? min(qb + 1, n_kv) : n_kv;
  }
  return cost;
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  __syncthreads();
  return r;
}

// Launch: 1 block of 1024 threads; dynamic shared memory = sort_capacity * 8
// bytes (sort_capacity a power of two, or 0 to skip sorting).
__global__ void __launch_bounds__(1024, 1)
build_schedule_kernel(const int32_t* __restrict__ cu, int num_seqs, int total_tokens,
                      int max_seqlen, int dense_len, int causal, int tiles_per_unit,
                      int32_t* __restrict__ ws_header,
                      int4* __restrict__ sorted, int4* __restrict__ unsorted, int sort_capacity) {
  extern __shared__ unsigned long long keys[];
  __shared__ int warp_sums[32];
  __shared__ int chunk_total;
  const int tid = threadIdx.x, nt = blockDim.x;

  // The attention kernel queued behind this one may start its prologue now;
  // it reads the work list only after this grid has completed.
  ptx::grid_launch_dependents();

  // 0. the error word reports the most recent call only; the attention
  // kernel's unit counter starts from zero
  if (tid == 0) {
    ws_header[kWsErrorOffset / 4] = 0;
    ws_header[kWsUnitCounterOffset / 4] = 0;
  }

  // 1. validate the document offsets
  int bad = 0;
  if (cu != nullptr) {
    if (tid == 0) bad = (cu[0] != 0) || (cu[num_seqs] != total_tokens);
    for (int i = tid; i < num_seqs; i += nt) {
      const int L = cu[i + 1] - cu[i];
      bad |= (L < 0) || (L > max_seqlen);
    }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      ws_header[kWsErrorOffset / 4] = ATTN_ERR_BAD_SEQLENS;
      ws_header[kWsCountOffset / 4] = 0;
    }
    return;
  }

  // 2. enumerate (document, unit) entries in document order
  int running = 0;
  for (int base = 0; base < num_seqs; base += nt) {
    const int i = base + tid;
    int a = 0, L = 0, np = 0;
    if (i < num_seqs) {
      a = cu ? cu[i] : i * dense_len;
      L = cu ? cu[i + 1] - a : dense_len;
      np = (L + kBlockM * tiles_per_unit - 1) / (kBlockM * tiles_per_unit);
    }
    const int first = running + block_exclusive_scan(np, warp_sums, &chunk_total);
    for (int t = 0; t < np; ++t)
      unsorted[first + t] = make_int4(a, L, t, unit_cost(L, t, causal, tiles_per_unit));
    running += chunk_total;
    __syncthreads();
  }
  const int n = running;
  __syncthreads();

  // 3. stable sort by cost, largest first
  if (sort_capacity > 0 && n <= sort_capacity) {
    int n2 = 1;
    while (n2 < n) n2 <<= 1;
    for (int e = tid; e < n2; e += nt) {
      keys[e] = e < n ? (static_cast<unsigned long long>(0x7fffffff - unsorted[e].w) << 32) |
                            static_cast<unsigned>(e)
                      : ~0ull;
    }
    __syncthreads();
    for (int k = 2; k <= n2; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < n2; i += nt) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long x = keys[i], y = keys[ixj];
            const bool up = (i & k) == 0;
            if ((x > y) == up) {
              keys[i] = y;
              keys[ixj] = x;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int e = tid; e < n; e += nt) sorted[e] = unsorted[keys[e] & 0xffffffffu];
  } else {
    for (int e = tid; e < n; e += nt) sorted[e] = unsorted[e];
  }
  if (tid == 0) ws_header[kWsCountOffset / 4] = n;
}

}  // namespace attn

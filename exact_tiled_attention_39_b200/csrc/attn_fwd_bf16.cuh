// Exact attention forward, bf16, sm_100a: persistent, warp-specialised,
// TMA + tcgen05 + TMEM.
//
// The method ("FlashAttention và IO" (aihero.vn), sections "Tiling giữ công
// việc ở gần nơi tính" and "Softmax qua nhiều khối cần thống kê chạy"):
// Q, K and V are cut into tiles held on chip; for each query row the kernel
// keeps the running maximum m, the normaliser l and the weighted sum u (the
// output accumulator O), multiplies the old part by exp(m - m_new) when a
// new key tile raises the maximum, and writes u / l and the log-sum-exp at
// the end.  Scores and probabilities never leave the SM.
//
// Loop order and roles follow "FlashAttention, pelatihan multi-GPU, dan
// kuantisasi bobot" (section 1): outer loop over query blocks, inner over
// key/value blocks; a producer issues asynchronous tile copies while other
// warps run the matrix products and the softmax.  On sm_100a this becomes:
//
//   warp 0        TMA producer: the Q tile pair of a unit, then K_j, V_j into
//                 a ring of shared-memory slots (mbarrier pipelined).
//   warp 1        MMA issuer (one thread): S_i = Q_i K_j^T into TMEM and
//                 O_i += P_i V_j with P_i read from TMEM (tcgen05.mma).
//   warps 4..7    softmax of query tile 0, warps 8..11 of query tile 1: one
//                 thread per row reads its S row from TMEM, masks, updates
//                 m and l, writes P (bf16) back over S, rescales O when the
//                 maximum grew by more than 2^8 (lazy rescale), and runs the
//                 epilogue (O / l to bf16, log-sum-exp).
//
// While one softmax warpgroup works on its tile the tensor core computes
// the other tile's products (ping-pong), so the tensor pipe stays busy.
//
// TMEM (512 columns, lane = query row): S_0 at column 0, S_1 at 128,
// O_0 at 256, O_1 at 256 + D.  P_i overwrites the first 64 columns of S_i.
// Shared memory: Q_0, Q_1 and kStages K/V slots of 128 x D bf16, each stored
// as D/64 column chunks of 128 rows x 128 bytes with the 128-byte swizzle
// the TMA writes and the tensor core reads.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"

namespace attn {

struct FwdParams {
  void* out;                 // bf16 [T, H, D]
  float* lse;                // fp32 [H, T]
  const int32_t* ws_header;  // error word, work-list length
  const int4* work;          // work list
  int32_t* err;              // error word (device)
  int total_tokens;
  int num_heads;
  int causal;
  float scale_log2;          // scale * log2(e)
  unsigned long long timeout_ns;
};

template <int D>
struct FwdLayout {
  static constexpr int kChunks = D / 64;               // 128-byte chunks per row
  static constexpr int kChunkBytes = kBlockM * 128;    // one chunk of a tile
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = 4;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barrier indices
  static constexpr int kQFull = 0, kQEmpty = 1;
  static constexpr int kKVFull = 2;                    // + stage
  static constexpr int kKVEmpty = 2 + kStages;         // + stage
  static constexpr int kSFull = 2 + 2 * kStages;       // + tile
  static constexpr int kPFull = kSFull + 2;            // + tile
  static constexpr int kOFull = kPFull + 2;            // + tile
  static constexpr int kOEmpty = kOFull + 2;           // + tile
  static constexpr int kDrain = kOEmpty + 2;
  static constexpr int kNumBars = kDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAllocBytes = kBytes + 1024;    // slack for 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
};

// Bounded waits.  A wait gives up when the CTA's abort flag is raised or
// after timeout_ns; the first thread to give up records ATTN_ERR_TIMEOUT.
struct WaitCtl {
  volatile uint32_t* abort_flag;
  int32_t* err;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void raise_abort(const WaitCtl& c) {
  if (*c.abort_flag == 0) {
    *c.abort_flag = 1;
    atomicCAS(c.err, 0, (int)ATTN_ERR_TIMEOUT);
  }
}

// Single-thread bounded wait.
__device__ __noinline__ bool wait_one(uint32_t bar, uint32_t parity, const WaitCtl& c) {
  if (ptx::mbar_test(bar, parity)) return true;
  unsigned long long t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_test(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*c.abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > c.timeout_ns) {
        raise_abort(c);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: every lane probes; the warp leaves together.
__device__ __noinline__ bool wait_warp(uint32_t bar, uint32_t parity, const WaitCtl& c) {
  if (__all_sync(0xffffffffu, ptx::mbar_test(bar, parity))) return true;
  unsigned long long t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, ptx::mbar_test(bar, parity))) return true;
    if ((it & 63) == 0) {
      bool give_up = *c.abort_flag != 0;
      give_up |= ptx::globaltimer_ns() - t0 > c.timeout_ns;
      if (__any_sync(0xffffffffu, give_up)) {
        if (ptx::lane_id() == 0) raise_abort(c);
        return false;
      }
    }
  }
}

struct UnitInfo {
  int doc_start, doc_len, pair, head, n_kv_steps, kv_tiles;
  bool tile1_valid;
};

__device__ __forceinline__ UnitInfo decode_unit(const int4* work, int u, int H, int causal) {
  const int4 w = work[u / H];
  UnitInfo r;
  r.doc_start = w.x;
  r.doc_len = w.y;
  r.pair = w.z;
  r.head = u % H;
  r.kv_tiles = (w.y + kBlockN - 1) / kBlockN;
  r.n_kv_steps = causal ? min(kTilesPerUnit * w.z + kTilesPerUnit, r.kv_tiles) : r.kv_tiles;
  r.tile1_valid = (kRowsPerUnit * w.z + kBlockM) < w.y;
  return r;
}

// Is query tile `i` of the unit active at key step j?
__device__ __forceinline__ bool tile_active(const UnitInfo& ui, int i, int j, int causal) {
  if (i == 1 && !ui.tile1_valid) return false;
  return !causal || j <= kTilesPerUnit * ui.pair + i;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Lay = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBarOff + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(Lay::kQFull), 1);
    ptx::mbar_init(bar(Lay::kQEmpty), 1);
    for (int s = 0; s < Lay::kStages; ++s) {
      ptx::mbar_init(bar(Lay::kKVFull + s), 1);
      ptx::mbar_init(bar(Lay::kKVEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(Lay::kSFull + i), 1);
      ptx::mbar_init(bar(Lay::kPFull + i), 4);   // one arrival per softmax warp
      ptx::mbar_init(bar(Lay::kOFull + i), 1);
      ptx::mbar_init(bar(Lay::kOEmpty + i), 4);
    }
    ptx::mbar_init(bar(Lay::kDrain), 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_holder), Lay::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const WaitCtl ctl{abort_flag, p.err, p.timeout_ns};
  const int H = p.num_heads;
  const int causal = p.causal;
  const int n_units = p.ws_header[kWsCountOffset / 4] * H;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t q_it = 0, kv_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const UnitInfo ui = decode_unit(p.work, u, H, causal);
        if (!(ok = wait_one(bar(Lay::kQEmpty), (q_it & 1) ^ 1, ctl))) break;
        ptx::mbar_arrive_expect_tx(bar(Lay::kQFull), 2 * Lay::kTileBytes);
        for (int i = 0; i < 2; ++i) {
          const int row = ui.doc_start + kRowsPerUnit * ui.pair + kBlockM * i;
          for (int c = 0; c < Lay::kChunks; ++c)
            ptx::tma_load_3d(sbase + Lay::kQOff + i * Lay::kTileBytes + c * Lay::kChunkBytes,
                             &tm_q, bar(Lay::kQFull), c * 64, ui.head, row);
        }
        ++q_it;
        for (int j = 0; ok && j < ui.n_kv_steps; ++j) {
          const int row = ui.doc_start + kBlockN * j;
          for (int kind = 0; kind < 2; ++kind) {
            const int s = kv_it % Lay::kStages;
            if (!(ok = wait_one(bar(Lay::kKVEmpty + s), ((kv_it / Lay::kStages) & 1) ^ 1, ctl)))
              break;
            ptx::mbar_arrive_expect_tx(bar(Lay::kKVFull + s), Lay::kTileBytes);
            for (int c = 0; c < Lay::kChunks; ++c)
              ptx::tma_load_3d(sbase + Lay::kKVOff + s * Lay::kTileBytes + c * Lay::kChunkBytes,
                               kind == 0 ? static_cast<const void*>(&tm_k)
                                         : static_cast<const void*>(&tm_v),
                               bar(Lay::kKVFull + s), c * 64, ui.head, row);
            ++kv_it;
          }
        }
      }
      if (!ok) {
        // Let copies already issued land before the CTA can exit.
        WaitCtl drain = ctl;
        uint32_t zero = 0;
        drain.abort_flag = &zero;
        const uint32_t first = kv_it > (uint32_t)Lay::kStages ? kv_it - Lay::kStages : 0;
        for (uint32_t it = first; it < kv_it; ++it)
          wait_one(bar(Lay::kKVFull + it % Lay::kStages), (it / Lay::kStages) & 1, drain);
        if (q_it > 0) wait_one(bar(Lay::kQFull), (q_it - 1) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = ptx::idesc_bf16(kBlockM, kBlockN, 0);
      constexpr uint32_t kIdescO = ptx::idesc_bf16(kBlockM, D, 1);
      uint32_t q_it = 0, kv_it = 0;
      uint32_t p_cnt[2] = {0, 0}, oe_cnt[2] = {0, 0};
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const UnitInfo ui = decode_unit(p.work, u, H, causal);
        const int n = ui.n_kv_steps;
        if (!(ok = wait_one(bar(Lay::kQFull), q_it & 1, ctl))) break;
        ++q_it;
        ptx::tc_fence_after();
        bool first_pv[2] = {true, true};
        const uint32_t kv_base = kv_it;
        for (int j = 0; ok && j <= n; ++j) {
          const uint32_t idx_v = kv_base + 2 * (j - 1) + 1;
          const uint32_t idx_k = kv_base + 2 * j;
          const uint32_t slot_v = sbase + Lay::kKVOff + (idx_v % Lay::kStages) * Lay::kTileBytes;
          const uint32_t slot_k = sbase + Lay::kKVOff + (idx_k % Lay::kStages) * Lay::kTileBytes;
          if (j > 0) {
            if (!(ok = wait_one(bar(Lay::kKVFull + idx_v % Lay::kStages),
                                (idx_v / Lay::kStages) & 1, ctl)))
              break;
            ptx::tc_fence_after();
          }
          bool k_ready = false;
          for (int i = 0; ok && i < 2; ++i) {
            if (j > 0 && tile_active(ui, i, j - 1, causal)) {
              if (!(ok = wait_one(bar(Lay::kPFull + i), p_cnt[i] & 1, ctl))) break;
              ++p_cnt[i];
              if (first_pv[i]) {
                if (!(ok = wait_one(bar(Lay::kOEmpty + i), (oe_cnt[i] & 1) ^ 1, ctl))) break;
                ++oe_cnt[i];
              }
              ptx::tc_fence_after();
              const uint32_t t_o = tmem + 256 + i * D;
              const uint32_t t_p = tmem + i * 128;
#pragma unroll
              for (int kk = 0; kk < kBlockN / 16; ++kk) {
                const uint64_t bdesc = ptx::sdesc_sw128(slot_v + kk * 2048, Lay::kChunkBytes, 1024);
                ptx::mma_f16_ts(t_o, t_p + kk * 8, bdesc, kIdescO,
                                (first_pv[i] && kk == 0) ? 0u : 1u);
              }
              first_pv[i] = false;
              ptx::mma_commit(bar(Lay::kOFull + i));
            }
            if (j < n && tile_active(ui, i, j, causal)) {
              if (!k_ready) {
                if (!(ok = wait_one(bar(Lay::kKVFull + idx_k % Lay::kStages),
                                    (idx_k / Lay::kStages) & 1, ctl)))
                  break;
                ptx::tc_fence_after();
                k_ready = true;
              }
              const uint32_t t_s = tmem + i * 128;
              const uint32_t q_tile = sbase + Lay::kQOff + i * Lay::kTileBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * Lay::kChunkBytes + (kk & 3) * 32;
                const uint64_t adesc = ptx::sdesc_sw128(q_tile + off, 16, 1024);
                const uint64_t bdesc = ptx::sdesc_sw128(slot_k + off, 16, 1024);
                ptx::mma_f16_ss(t_s, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
              }
              ptx::mma_commit(bar(Lay::kSFull + i));
            }
          }
          if (!ok) break;
          if (j > 0) ptx::mma_commit(bar(Lay::kKVEmpty + idx_v % Lay::kStages));
          if (j < n) {
            if (!k_ready) {
              if (!(ok = wait_one(bar(Lay::kKVFull + idx_k % Lay::kStages),
                                  (idx_k / Lay::kStages) & 1, ctl)))
                break;
            }
            ptx::mma_commit(bar(Lay::kKVEmpty + idx_k % Lay::kStages));
          }
          if (j == n - 1) ptx::mma_commit(bar(Lay::kQEmpty));
        }
        kv_it += 2 * n;
      }
      // Every product this thread issued must be complete before TMEM is freed.
      ptx::mma_commit(bar(Lay::kDrain));
      WaitCtl drain = ctl;
      uint32_t zero = 0;
      drain.abort_flag = &zero;
      wait_one(bar(Lay::kDrain), 0, drain);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int tile = (warp - 4) >> 2;
    const int wq = warp & 3;                      // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;                 // row within the query tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_off + tile * 128;
    const uint32_t t_o = tmem + lane_off + 256 + tile * D;
    const float c = p.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const UnitInfo ui = decode_unit(p.work, u, H, causal);
      if (tile == 1 && !ui.tile1_valid) continue;
      const int qb = kTilesPerUnit * ui.pair + tile;
      const int last = causal ? min(qb, ui.kv_tiles - 1) : ui.kv_tiles - 1;
      const int row_doc = qb * kBlockM + r;
      float m_used = -INFINITY;   // running maximum in log2 units
      float l = 0.f;              // sum of the weights
      float l_round = 0.f;        // sum of the weights as rounded to bf16
      for (int j = 0; j <= last; ++j) {
        if (!(ok = wait_warp(bar(Lay::kSFull + tile), s_cnt & 1, ctl))) break;
        ++s_cnt;
        ptx::tc_fence_after();
        uint32_t sr[128];
        ptx::tmem_ld_x128(t_s, sr);
        float s[128];
#pragma unroll
        for (int k = 0; k < 128; ++k) s[k] = __uint_as_float(sr[k]);
        const bool diag = causal && j == qb;
        if (diag || (j + 1) * kBlockN > ui.doc_len) {
          int limit = ui.doc_len - j * kBlockN;
          if (diag) limit = min(limit, r + 1);
#pragma unroll
          for (int k = 0; k < 128; ++k)
            if (k >= limit) s[k] = -INFINITY;
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int k = 4; k < 128; k += 4) {
          mx0 = fmaxf(mx0, s[k]);
          mx1 = fmaxf(mx1, s[k + 1]);
          mx2 = fmaxf(mx2, s[k + 2]);
          mx3 = fmaxf(mx3, s[k + 3]);
        }
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
        if (j == 0) {
          m_used = m_tile;
        } else {
          // Rescale only rows whose maximum grew past the threshold.  TMEM
          // access is warp-wide, so the other rows of the warp take part with
          // a factor of exactly 1: a row's arithmetic never depends on other
          // rows' data.
          const bool need = m_tile > m_used + kRescaleTau;
          if (__any_sync(0xffffffffu, need)) {
            // O may only be touched once the previous P V product is done.
            if (!(ok = wait_warp(bar(Lay::kOFull + tile), (o_cnt + j - 1) & 1, ctl))) break;
            ptx::tc_fence_after();
            const float m_next = need ? m_tile : m_used;
            const float alpha = need ? ptx::ex2_approx(m_used - m_next) : 1.f;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              ptx::tmem_ld_x32(t_o + cc * 32, o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              ptx::tmem_st_x32(t_o + cc * 32, o);
            }
            ptx::tmem_wait_st();
            l *= alpha;
            l_round *= alpha;
            m_used = m_next;
          }
        }
        // Weights are rounded to bf16 for the P V product.  Two normalisers:
        // l_round sums the rounded weights, so O / l_round is an exact convex
        // combination of the values with the weights actually used (no bias
        // from the rounding, which matters when one key dominates a row);
        // l sums the unrounded weights and gives the log-sum-exp.
        const float base = m_used == -INFINITY ? 0.f : m_used;
        float se0 = 0.f, se1 = 0.f, sr0 = 0.f, sr1 = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const float p0 = ptx::ex2_approx(fmaf(s[2 * k], c, -base));
          const float p1 = ptx::ex2_approx(fmaf(s[2 * k + 1], c, -base));
          pk[k] = ptx::pack_bf16x2(p0, p1);
          se0 += p0;
          se1 += p1;
          sr0 += __uint_as_float(pk[k] << 16);
          sr1 += __uint_as_float(pk[k] & 0xFFFF0000u);
        }
        l += se0 + se1;
        l_round += sr0 + sr1;
        ptx::tmem_st_x64(t_s, pk);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kPFull + tile));
      }
      if (!ok) break;
      // epilogue: wait for the last P V product of this tile
      if (!(ok = wait_warp(bar(Lay::kOFull + tile), (o_cnt + last) & 1, ctl))) break;
      o_cnt += last + 1;
      ptx::tc_fence_after();
      const bool row_ok = row_doc < ui.doc_len;
      const long long token = static_cast<long long>(ui.doc_start) + row_doc;
      const float inv_l = 1.f / l_round;
      uint4* orow =
          reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + (token * H + ui.head) * D);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        ptx::tmem_ld_x32(t_o + cc * 32, o);
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          w[k] = ptx::pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l,
                                  __uint_as_float(o[2 * k + 1]) * inv_l);
        if (row_ok) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            orow[cc * 4 + v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (row_ok)
        p.lse[static_cast<long long>(ui.head) * p.total_tokens + token] =
            (m_used + __log2f(l)) * 0.69314718055994530942f;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(Lay::kOEmpty + tile));
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

}  // namespace attn

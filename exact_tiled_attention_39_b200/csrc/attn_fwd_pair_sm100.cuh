// Exact attention forward for sm_100a: two query tiles per CTA sharing every
// K/V tile, one softmax warpgroup per query tile.  The score product runs in
// bf16, or block-scaled on MXFP8 or NVFP4 codes (head dim 128, 112-key
// tiles); P V always runs in bf16.
//
// The method is the one of attn_fwd_sm100.cuh ("FlashAttention và IO"
// (aihero.vn), sections "Tiling giữ công việc ở gần nơi tính" and "Softmax
// qua nhiều khối cần thống kê chạy": running maximum m, normaliser l and
// weighted sum u per query row, rescale by exp(m - m_new), result u / l and
// the log-sum-exp); the loop order and roles follow "FlashAttention,
// pelatihan multi-GPU, dan kuantisasi bobot" (section 1: outer loop over
// query blocks, inner over key/value blocks, a producer issuing asynchronous
// copies, other warps running the products and the softmax).
//
// A work unit is a pair of consecutive 128-row query tiles (A = 2t, B =
// 2t + 1) of one document and head.  Both tiles use the same K_j, V_j, so
// each K/V tile is loaded once per 256 query rows, and while one tile's
// softmax works the tensor core runs the other tile's products: per key
// step the tensor pipe sees P_A V_j, S_A(j+1), P_B V_j, S_B(j+1).
//
//   warps 0..3    softmax of tile A (184 registers): one thread per query
//                 row reads its 128 scores from TMEM, masks, updates m and l,
//                 writes P (bf16) over the first 64 columns of its scores and
//                 rescales O_A when the row maximum grew by more than 2^8.
//   warps 4..7    softmax of tile B.
//   warps 8..11   epilogue (64 registers): O_t / l_round -> bf16, lse.
//   warp 12       producer (80 registers): claims units, TMA loads of Q_A,
//                 Q_B and of K_j, V_j into a ring of shared-memory slots;
//                 block-scaled forms: the whole warp stages the scale blocks.
//   warp 13       MMA issuer (one thread); block-scaled forms: copies the
//                 scale blocks into TMEM (tcgen05.cp) ahead of the products.
//   warps 14..15  idle.
//
// TMEM (512 columns, lane = query row): S_A at 0, S_B at 128, O_A at 256,
// O_B at 384.  S_t(j+1) is issued after P_t V_j has read P_t(j) (in issue
// order, which the tensor pipe keeps), and its completion also tells the
// softmax that O_t is up to date for a rescale.
#pragma once
#include "attn_fwd_sm100.cuh"

namespace attn {

// Failure-test build only: the first unit's S_A-ready signal is never sent,
// so tile A's softmax waits run out, the CTA aborts and the call reports
// ATTN_ERR_TIMEOUT (with a short ATTN_WAIT_TIMEOUT_NS).
#ifndef ATTN_FAULT_DROP_FIRST_SCORE_COMMIT
#define ATTN_FAULT_DROP_FIRST_SCORE_COMMIT 0
#endif
constexpr bool kFaultDropFirstScoreCommit = ATTN_FAULT_DROP_FIRST_SCORE_COMMIT != 0;

constexpr int kPairThreads = 512;
constexpr uint32_t kPairRegsSoftmax = 184, kPairRegsEpilogue = 64, kPairRegsOther = 80;
static_assert(2 * kPairRegsSoftmax + kPairRegsEpilogue + kPairRegsOther == 4 * 128,
              "register split must use exactly the registers the CTA is launched with");
constexpr int kPairUnitConsumers = 1 + 8 + 4;   // MMA thread + softmax warps + epilogue warps

// Score operand format kQk (attn_fwd_sm100.cuh): bf16; MXFP8 (E4M3 codes
// with one E8M0 scale per 32 elements); NVFP4 (packed E2M1 codes with one
// UE4M3 scale per 16 elements); the block-scaled formats at head dim 128.
// They use key tiles of 112: the score products are then 112 columns wide,
// which leaves the last 16 columns of each tile's score buffer for the
// scale factors (Q's of each tile, and two buffers of the K tile's).
template <int D, int kQk>
struct PairLayout {
  static constexpr bool kFp8 = kQk != kQkBf16;                // block-scaled Q, K
  static constexpr bool kNv4 = kQk == kQkNv4;
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static_assert(!kFp8 || D == 128, "block-scaled pair kernel: head dim 128");
  static constexpr int kBN = kFp8 ? 112 : 128;                // keys per K/V tile
  static constexpr int kChunks = D / 64;                      // 128-byte chunks of a bf16 row
  static constexpr int kQkChunks = kFp8 ? 1 : kChunks;        // swizzle chunks of a Q or K row
  static constexpr int kQkRowBytes = kNv4 ? 64 : 128;         // bytes of a Q or K row per chunk
  static constexpr int kQTileBytes = kQkChunks * kBlockM * kQkRowBytes;
  static constexpr int kKTileBytes = kQkChunks * kBN * kQkRowBytes;
  static constexpr int kVChunkBytes = kBN * 128;
  static constexpr int kVTileBytes = kChunks * kVChunkBytes;
  // Scale words per row (4 scale bytes each): MXFP8 1, NVFP4 2 (one per
  // K = 64 product); one 32-row x 16-byte block per word and tile.
  static constexpr int kSfWords = kNv4 ? 2 : 1;
  static constexpr int kSfBytes = kFp8 ? 512 * kSfWords : 0;  // scale blocks of a Q or K tile
  static constexpr int kSlotRaw = kVTileBytes > kKTileBytes + kSfBytes ? kVTileBytes
                                                                       : kKTileBytes + kSfBytes;
  static constexpr int kSlotBytes = (kSlotRaw + 1023) / 1024 * 1024;   // a K (+ scales) or V tile
  static constexpr int kQOff = 0;                             // Q_A, then Q_B
  static constexpr int kSfaOff = 2 * kQTileBytes;             // MXFP8: Q_A's, Q_B's scale blocks
  static constexpr int kRingOff = (kSfaOff + 2 * kSfBytes + 1023) / 1024 * 1024;
  static constexpr int kReserve = 3072;                       // stats, barriers, unit ring
  static constexpr int kStagesFit = (232448 - kRingOff - kReserve) / kSlotBytes;
  static constexpr int kStages = kStagesFit > 12 ? 12 : kStagesFit;
  static constexpr int kStatsOff = kRingOff + kStages * kSlotBytes;   // float [tile][2][128]
  static constexpr int kBarOff = kStatsOff + 2 * 2 * kBlockM * 4;
  static constexpr int kQFull = 0, kQEmpty = 1;
  static constexpr int kKVFull = 2;                           // + stage
  static constexpr int kKVEmpty = kKVFull + kStages;          // + stage
  static constexpr int kSFull = kKVEmpty + kStages;           // + tile
  static constexpr int kPFull = kSFull + 2;                   // + tile
  static constexpr int kOUnit = kPFull + 2;                   // + tile: O of a unit complete
  static constexpr int kOEmpty = kOUnit + 2;                  // + tile
  static constexpr int kStFull = kOEmpty + 2;                 // + tile
  static constexpr int kStEmpty = kStFull + 2;                // + tile
  static constexpr int kDrain = kStEmpty + 2;
  static constexpr int kUnitFull = kDrain + 1;                // + slot
  static constexpr int kUnitEmpty = kUnitFull + kUnitSlots;   // + slot
  static constexpr int kNumBars = kUnitEmpty + kUnitSlots;
  static constexpr int kMiscOff = (kBarOff + kNumBars * 8 + 15) / 16 * 16;   // tmem base, abort
  static constexpr int kUnitOff = kMiscOff + 16;              // int4 [kUnitSlots]
  static constexpr int kBytes = kUnitOff + 16 * kUnitSlots;
  static_assert(kStages >= 3, "too few K/V stages");
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory per CTA");
  static_assert(kBytes - kStatsOff <= kReserve, "reserve too small");
  static_assert(kSlotBytes % 1024 == 0 && kVChunkBytes % 1024 == 0, "swizzle alignment");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 256;                     // + 128 * tile
  // Scale factors in the unused columns 112..127 of the score buffers, 4
  // columns per scale word: Q_t's at 128 t + 112; the K tiles' two buffers
  // at 116 and 120 (MXFP8) or 120 and 248 (NVFP4, 8 columns each).
  static constexpr uint32_t kTmemSfa = 112;
  __host__ __device__ static constexpr uint32_t sfb_col(uint32_t b) {
    return kNv4 ? 120 + 128 * b : 116 + 4 * b;
  }
};

// Key steps of query tile qb (128 rows) of a document of doc_len tokens with
// key tiles of bn keys (0 if the tile starts past the document's end).
__device__ __forceinline__ int tile_steps(int qb, int doc_len, int causal, int bn = kBlockN) {
  if (qb * kBlockM >= doc_len) return 0;
  const int last = causal ? min(doc_len, (qb + 1) * kBlockM) : doc_len;   // keys seen
  return (last + bn - 1) / bn;
}

template <int D, int kQk>
__global__ void __launch_bounds__(kPairThreads, 1)
attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Lay = PairLayout<D, kQk>;
  constexpr bool kFp8 = Lay::kFp8;
  constexpr int BN = Lay::kBN;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = ptx::smem_addr(smem);
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0, (int)ATTN_ERR_UNSUPPORTED);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBarOff + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  float* stats = reinterpret_cast<float*>(smem + Lay::kStatsOff);   // [tile][lse2, 1/l_round][row]
  int4* unit_ring = reinterpret_cast<int4*>(smem + Lay::kUnitOff);

  constexpr int kWarpTma = 12, kWarpMma = 13;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(Lay::kQFull), 1);
    ptx::mbar_init(bar(Lay::kQEmpty), 1);
    for (int s = 0; s < Lay::kStages; ++s) {
      ptx::mbar_init(bar(Lay::kKVFull + s), 1);
      ptx::mbar_init(bar(Lay::kKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(bar(Lay::kSFull + t), 1);
      ptx::mbar_init(bar(Lay::kPFull + t), 4);     // the tile's softmax warps
      ptx::mbar_init(bar(Lay::kOUnit + t), 1);
      ptx::mbar_init(bar(Lay::kOEmpty + t), 4);    // epilogue warps
      ptx::mbar_init(bar(Lay::kStFull + t), 4);
      ptx::mbar_init(bar(Lay::kStEmpty + t), 4);
    }
    ptx::mbar_init(bar(Lay::kDrain), 1);
    for (int i = 0; i < kUnitSlots; ++i) {
      ptx::mbar_init(bar(Lay::kUnitFull + i), 1);
      ptx::mbar_init(bar(Lay::kUnitEmpty + i), kPairUnitConsumers);
    }
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == kWarpTma && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_holder), Lay::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // The work list is written by the schedule-build kernel launched just
  // before; everything above overlapped with its tail.
  ptx::grid_dependency_wait();

  const WaitCtl ctl{abort_flag, p.err, p.timeout_ns};
  const int H = p.num_heads;
  const int causal = p.causal;
  auto next_unit_warp = [&](uint32_t k, bool& ok) -> int4 {
    const uint32_t slot = k % kUnitSlots;
    if (!(ok = wait_warp(bar(Lay::kUnitFull + slot), (k / kUnitSlots) & 1, ctl)))
      return make_int4(0, -1, 0, 0);
    const int4 w = unit_ring[slot];   // after the wait (asm with a memory clobber)
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar(Lay::kUnitEmpty + slot));
    return w;
  };

  if (warp < 8) {
    // ------------------------------------------------------------ softmax
    ptx::regs_increase<kPairRegsSoftmax>();
    const int t = warp >> 2;                       // query tile of the pair
    const int r = (warp & 3) * 32 + lane;          // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + t * 128;
    const uint32_t t_o = tmem + lane_off + Lay::kTmemO + t * 128;
    const float c = p.scale_log2;
    const uint64_t c2 = ptx::f2_pack(c, c);
    uint32_t g = 0, st_cnt = 0;                    // this tile's key steps, units handed over
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int4 uw = next_unit_warp(k, ok);
      if (uw.y < 0) break;
      const int doc_len = uw.y;
      const int qb = 2 * uw.z + t;
      const int n = tile_steps(qb, doc_len, causal, BN);
      if (n == 0) continue;
      float m_used = -INFINITY;   // running maximum in log2 units
      float l = 0.f;              // sum of the weights
      float l_round = 0.f;        // sum of the weights as rounded to bf16
      for (int j = 0; j < n; ++j, ++g) {
        if (!(ok = wait_warp(bar(Lay::kSFull + t), g & 1, ctl))) break;
        ptx::tc_fence_after();
        float s[128];
        {
          uint32_t sa[128];
          ptx::tmem_ld_2x64(t_s, sa);     // both halves in flight, one wait
#pragma unroll
          for (int q = 0; q < 128; ++q) s[q] = __uint_as_float(sa[q]);
        }
        // Keys past the document's end or (causal) past this row: -inf.  A
        // tile needs masking if it reaches past the document or, causal,
        // past the tile's first row.
        const bool diag = causal && (j + 1) * BN - 1 > qb * kBlockM;
        if (diag || (j + 1) * BN > doc_len) {
          int limit = doc_len - j * BN;
          if (diag) limit = min(limit, qb * kBlockM + r + 1 - j * BN);
#pragma unroll
          for (int q = 0; q < BN; ++q)
            if (q >= limit) s[q] = -INFINITY;
        }
        // Weights rounded to bf16 for the P V product, written over the
        // scores; returns the sums of the weights (for the log-sum-exp) and
        // of the rounded weights (O is divided by the latter).
        auto weights = [&](float base_in, float& e_sum, float& r_sum) {
          const float base = base_in == -INFINITY ? 0.f : base_in;
          const uint64_t nb2 = ptx::f2_pack(-base, -base);
          uint64_t se[2];
          float sr[4];
#pragma unroll
          for (int a = 0; a < 2; ++a) se[a] = ptx::f2_pack(0.f, 0.f);
#pragma unroll
          for (int a = 0; a < 4; ++a) sr[a] = 0.f;
          // P in chunks of kPk key pairs (one TMEM store each)
          constexpr int kPk = BN % 32 == 0 ? 16 : 8;
#pragma unroll
          for (int ch = 0; ch < BN / (2 * kPk); ++ch) {
            uint32_t pk[kPk];
#pragma unroll
            for (int kk = 0; kk < kPk; ++kk) {
              const int q = ch * kPk + kk;
              const uint64_t x = ptx::f2_fma(ptx::f2_pack(s[2 * q], s[2 * q + 1]), c2, nb2);
              float x0, x1, p0, p1;
              ptx::f2_unpack(x, x0, x1);
              p0 = ptx::ex2_approx(x0);
              p1 = ptx::ex2_approx(x1);
              pk[kk] = ptx::pack_bf16x2(p0, p1);
              se[kk & 1] = ptx::f2_add(se[kk & 1], ptx::f2_pack(p0, p1));
              sr[(kk & 1) * 2] = ptx::add_bf16_lo(sr[(kk & 1) * 2], pk[kk]);
              sr[(kk & 1) * 2 + 1] = ptx::add_bf16_hi(sr[(kk & 1) * 2 + 1], pk[kk]);
            }
            if constexpr (kPk == 16)
              ptx::tmem_st_x16(t_s + ch * 16, pk);
            else
              ptx::tmem_st_x8(t_s + ch * 8, pk);
          }
          float e0, e1;
          ptx::f2_unpack(ptx::f2_add(se[0], se[1]), e0, e1);
          e_sum = e0 + e1;
          r_sum = (sr[0] + sr[1]) + (sr[2] + sr[3]);
        };
        // Lazy rescale: rows whose maximum grew past the threshold take the
        // new maximum and O_t's rows are multiplied by 2^(m_old - m_new)
        // (warp-wide TMEM access: other rows take part with a factor of
        // exactly 1).  S_t(j) completed after P_t V_{j-1}, so O_t is up to
        // date.
        auto rescale = [&](bool need, float m_tile) {
          const float m_next = need ? m_tile : m_used;
          const float alpha = need ? ptx::ex2_approx(m_used - m_next) : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t o[16];
            ptx::tmem_ld_x16(t_o + cc * 16, o);
#pragma unroll
            for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            ptx::tmem_st_x16(t_o + cc * 16, o);
          }
          l *= alpha;
          l_round *= alpha;
          m_used = m_next;
        };
        auto tile_max = [&]() -> float {
          float mx[8];
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = fmaxf(s[2 * a], s[2 * a + 1]);
#pragma unroll
          for (int q = 16; q < BN; q += 16)
#pragma unroll
            for (int a = 0; a < 8; ++a) mx[a] = ptx::fmax3(mx[a], s[q + 2 * a], s[q + 2 * a + 1]);
          return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                       fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * c;
        };
        const float m_tile = tile_max();
        if (j == 0) {
          m_used = m_tile;
        } else {
          const bool need = m_tile > m_used + kRescaleTau;
          if (__any_sync(0xffffffffu, need)) rescale(need, m_tile);
        }
        float e_sum, r_sum;
        weights(m_used, e_sum, r_sum);
        l += e_sum;
        l_round += r_sum;
        // bf16: a unit's first P goes to the tensor core only once the
        // epilogue has read the previous unit's O_t (its first P V
        // overwrites O_t), so the MMA thread's wait for P covers that and its
        // issue loop carries no wait of its own (measured faster; the
        // block-scaled forms keep the wait in the MMA thread, measured faster
        // there).
        if constexpr (!kFp8)
          if (j == 0 && !(ok = wait_warp(bar(Lay::kOEmpty + t), (st_cnt & 1) ^ 1, ctl))) break;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kPFull + t));
      }
      if (!ok) break;
      if (!(ok = wait_warp(bar(Lay::kStEmpty + t), (st_cnt & 1) ^ 1, ctl))) break;
      ++st_cnt;
      stats[(2 * t) * kBlockM + r] = m_used + __log2f(l);
      stats[(2 * t + 1) * kBlockM + r] = 1.f / l_round;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(Lay::kStFull + t));
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ epilogue
    ptx::regs_decrease<kPairRegsEpilogue>();
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    uint32_t st_cnt[2] = {0, 0};
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int4 uw = next_unit_warp(k, ok);
      if (uw.y < 0) break;
      for (int t = 0; t < 2 && ok; ++t) {
        const int qb = 2 * uw.z + t;
        if (tile_steps(qb, uw.y, causal, BN) == 0) continue;
        const uint32_t cnt = st_cnt[t]++;
        if (!(ok = wait_warp(bar(Lay::kStFull + t), cnt & 1, ctl))) break;
        const float lse2 = stats[(2 * t) * kBlockM + r];
        const float inv_l = stats[(2 * t + 1) * kBlockM + r];
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kStEmpty + t));
        if (!(ok = wait_warp(bar(Lay::kOUnit + t), cnt & 1, ctl))) break;
        ptx::tc_fence_after();
        const int row_doc = qb * kBlockM + r;
        const bool row_ok = row_doc < uw.y;
        const long long token = static_cast<long long>(uw.x) + row_doc;
        uint4* orow =
            reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + (token * H + uw.w) * D);
        const uint32_t t_o = tmem + (static_cast<uint32_t>(wq * 32) << 16) + Lay::kTmemO + t * 128;
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t o[16];
          ptx::tmem_ld_x16(t_o + cc * 16, o);
          if (cc == D / 16 - 1) {
            // O_t is in registers: the tensor core may overwrite it now.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(Lay::kOEmpty + t));
          }
          uint32_t w[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            w[q] = ptx::pack_bf16x2(__uint_as_float(o[2 * q]) * inv_l,
                                    __uint_as_float(o[2 * q + 1]) * inv_l);
          if (row_ok) {
            orow[cc * 2] = make_uint4(w[0], w[1], w[2], w[3]);
            orow[cc * 2 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
        if (row_ok)
          p.lse[static_cast<long long>(uw.w) * p.total_tokens + token] =
              lse2 * 0.69314718055994530942f;
      }
    }
  } else {
    ptx::regs_decrease<kPairRegsOther>();
    if (warp == kWarpTma) {
      // ---------------------------------------------------------- producer
      const int n_units = p.ws_header[kWsCountOffset / 4] * H;
      int* counter = const_cast<int*>(p.ws_header) + kWsUnitCounterOffset / 4;
      uint32_t q_it = 0, kv_it = 0;
      bool ok = true;
      // Scale block of the 128 rows from row0 (MXFP8): lane m0 writes rows
      // m0 + 32 c, c = 0..3, as 16 bytes at offset 16 m0 (the layout
      // tcgen05.cp replicates); rows past `rows` or the tensor get 0.
      auto stage_scales = [&](const uint32_t* scales, int head, int row0, int rows, int w,
                              int off) {
        uint32_t wv[4];
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {
          const int rr = lane + 32 * cq;
          const int tok = row0 + rr;
          wv[cq] = rr < rows && tok < p.total_tokens
                       ? scales[(static_cast<long long>(tok) * H + head) * Lay::kSfWords + w]
                       : 0u;
        }
        *reinterpret_cast<uint4*>(smem + off + 16 * lane) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      };
      // One K (kind 0) or V (kind 1) tile into the next ring slot.
      auto load_kv = [&](int head, int row0, int kind) -> bool {
        const uint32_t s = kv_it % Lay::kStages;
        if (!wait_warp(bar(Lay::kKVEmpty + s), ((kv_it / Lay::kStages) & 1) ^ 1, ctl)) return false;
        if (kFp8 && kind == 0) {
          for (int w = 0; w < Lay::kSfWords; ++w)
            stage_scales(p.k_scales, head, row0, BN, w,
                         Lay::kRingOff + s * Lay::kSlotBytes + Lay::kKTileBytes + 512 * w);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t slot = sbase + Lay::kRingOff + s * Lay::kSlotBytes;
          if (kind == 0) {
            ptx::mbar_arrive_expect_tx(bar(Lay::kKVFull + s), Lay::kKTileBytes);
            for (int cq = 0; cq < Lay::kQkChunks; ++cq)
              ptx::tma_load_3d(slot + cq * BN * 128, &tm_k, bar(Lay::kKVFull + s),
                               cq * 64, head, row0);
          } else {
            ptx::mbar_arrive_expect_tx(bar(Lay::kKVFull + s), Lay::kVTileBytes);
            for (int cq = 0; cq < Lay::kChunks; ++cq)
              ptx::tma_load_3d(slot + cq * Lay::kVChunkBytes, &tm_v, bar(Lay::kKVFull + s),
                               cq * 64, head, row0);
          }
        }
        __syncwarp();
        ++kv_it;
        return true;
      };
      for (uint32_t k = 0; ok; ++k) {
        int claim = 0;
        if (lane == 0)
          claim = k == 0 ? static_cast<int>(blockIdx.x)
                         : static_cast<int>(gridDim.x) + atomicAdd(counter, 1);
        claim = __shfl_sync(0xffffffffu, claim, 0);
        int4 uw = make_int4(0, -1, 0, 0);
        if (claim < n_units) {
          // Unit -> (entry, head): groups of heads one after the other, the
          // first H % n_groups groups one head larger; inside a group entry
          // major (heaviest first), head minor.
          const int n_entries = n_units / H;
          const int base = H / p.head_groups, extra = H % p.head_groups;
          const int big = n_entries * (base + 1);
          int rem, gsize, h0;
          if (claim < extra * big) {
            const int grp = claim / big;
            rem = claim - grp * big;
            gsize = base + 1;
            h0 = grp * (base + 1);
          } else {
            const int c2 = claim - extra * big;
            const int grp = c2 / (n_entries * base);
            rem = c2 - grp * (n_entries * base);
            gsize = base;
            h0 = extra * (base + 1) + grp * base;
          }
          const int4 e = p.work[rem / gsize];
          uw = make_int4(e.x, e.y, e.z, h0 + rem % gsize);
        }
        const uint32_t uslot = k % kUnitSlots;
        if (!(ok = wait_warp(bar(Lay::kUnitEmpty + uslot), ((k / kUnitSlots) & 1) ^ 1, ctl))) break;
        if (lane == 0) {
          unit_ring[uslot] = uw;
          ptx::mbar_arrive(bar(Lay::kUnitFull + uslot));
        }
        __syncwarp();
        if (uw.y < 0) break;
        const int n_max = max(tile_steps(2 * uw.z, uw.y, causal, BN),
                              tile_steps(2 * uw.z + 1, uw.y, causal, BN));
        if (!(ok = wait_warp(bar(Lay::kQEmpty), (q_it & 1) ^ 1, ctl))) break;
        const int qrow0 = uw.x + 2 * kBlockM * uw.z;
        if constexpr (kFp8) {
          for (int t = 0; t < 2; ++t)
            for (int w = 0; w < Lay::kSfWords; ++w)
              stage_scales(p.q_scales, uw.w, qrow0 + t * kBlockM, kBlockM, w,
                           Lay::kSfaOff + t * Lay::kSfBytes + 512 * w);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(bar(Lay::kQFull), 2 * Lay::kQTileBytes);
          for (int t = 0; t < 2; ++t)
            for (int cq = 0; cq < Lay::kQkChunks; ++cq)
              ptx::tma_load_3d(sbase + Lay::kQOff + t * Lay::kQTileBytes + cq * kBlockM * 128,
                               &tm_q, bar(Lay::kQFull), cq * 64, uw.w, qrow0 + t * kBlockM);
        }
        __syncwarp();
        ++q_it;
        // ring order = consumption order: K_0, then V_j, K_{j+1}
        if (!(ok = load_kv(uw.w, uw.x, 0))) break;
        for (int j = 0; ok && j < n_max; ++j) {
          if (!(ok = load_kv(uw.w, uw.x + BN * j, 1))) break;
          if (j + 1 < n_max && !(ok = load_kv(uw.w, uw.x + BN * (j + 1), 0))) break;
        }
      }
      if (!ok && lane == 0) {
        // Let copies already issued land before the CTA can exit.
        WaitCtl drain = ctl;
        uint32_t zero = 0;
        drain.abort_flag = &zero;
        const uint32_t first = kv_it > (uint32_t)Lay::kStages ? kv_it - Lay::kStages : 0;
        for (uint32_t it = first; it < kv_it; ++it)
          wait_one(bar(Lay::kKVFull + it % Lay::kStages), (it / Lay::kStages) & 1, drain);
        if (q_it > 0) wait_one(bar(Lay::kQFull), (q_it - 1) & 1, drain);
      }
    } else if (warp == kWarpMma && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescS = ptx::idesc_bf16(kBlockM, BN, 0);
      constexpr uint32_t kIdescO = ptx::idesc_bf16(kBlockM, D, 1);
      constexpr uint32_t kDescHi = ptx::sdesc_hi_sw128(1024);
      // NVFP4 Q and K rows are 64 bytes: 64-byte swizzle, 8-row groups 512 B apart
      constexpr uint32_t kQkDescHi = Lay::kNv4 ? ptx::sdesc_hi_sw64(512) : kDescHi;
      const uint32_t q_lo = ptx::sdesc_lo(sbase + Lay::kQOff, 16);
      const uint32_t ring_lo = ptx::sdesc_lo(sbase + Lay::kRingOff, 16);
      const uint32_t v_lbo = static_cast<uint32_t>(Lay::kVChunkBytes - 16) >> 4 << 16;
      uint32_t q_ph = 0;
      uint32_t g[2] = {0, 0};          // key steps of each tile so far
      uint32_t oe_cnt[2] = {0, 0};     // units of each tile so far (block-scaled)
      uint32_t cur = 0, cur_ph = 0;    // ring cursor (stage, phase)
      uint32_t k_cnt = 0;              // K tiles taken (MXFP8: scale buffer k_cnt & 1)
      bool ok = true;
      auto take = [&](uint32_t& st) -> bool {
        st = cur;
        const bool r2 = wait_one(bar(Lay::kKVFull + cur), cur_ph, ctl);
        if (++cur == static_cast<uint32_t>(Lay::kStages)) {
          cur = 0;
          cur_ph ^= 1;
        }
        return r2;
      };
      // The next K tile; block-scaled: its scale blocks into the next TMEM
      // buffer (the products that read that buffer two K tiles ago were
      // issued before, and the tensor pipe keeps issue order).
      auto take_k = [&](uint32_t& st) -> bool {
        if (!take(st)) return false;
        if constexpr (kFp8) {
          ptx::tc_fence_after();
#pragma unroll
          for (int w = 0; w < Lay::kSfWords; ++w)
            tmem_cp_32x128b_x4(tmem + Lay::sfb_col(k_cnt & 1) + 4 * w,
                               sf_copy_desc(sbase + Lay::kRingOff + st * Lay::kSlotBytes +
                                            Lay::kKTileBytes + 512 * w));
        }
        ++k_cnt;
        return true;
      };
      // S_t = Q_t K^T with K in ring stage st
      auto score = [&](int t, uint32_t st, bool commit = true) {
        const uint32_t a_lo = q_lo + ((t * Lay::kQTileBytes) >> 4);
        const uint32_t b_lo = ring_lo + st * (Lay::kSlotBytes >> 4);
        if constexpr (Lay::kNv4) {
          // block-scaled E2M1: two K = 64 products (32 bytes of packed codes
          // each, 64-byte swizzle), scale word kk of each row
          const uint32_t sfa = tmem + t * 128 + Lay::kTmemSfa;
          const uint32_t sfb = tmem + Lay::sfb_col((k_cnt - 1) & 1);
#pragma unroll
          for (int kk = 0; kk < D / 64; ++kk) {
            const uint32_t off = (kk * 32) >> 4;
            mma_nvf4_ss(tmem + t * 128, ptx::sdesc_join(a_lo + off, kQkDescHi),
                        ptx::sdesc_join(b_lo + off, kQkDescHi), idesc_nvf4(BN), sfa + 4 * kk,
                        sfb + 4 * kk, kk > 0 ? 1u : 0u);
          }
        } else if constexpr (kFp8) {
          // block-scaled E4M3: four K = 32 products, scale byte kk of each
          // row's word
          const uint32_t sfa = tmem + t * 128 + Lay::kTmemSfa;
          const uint32_t sfb = tmem + Lay::sfb_col((k_cnt - 1) & 1);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint32_t off = (kk * 32) >> 4;
            mma_mxf8_ss(tmem + t * 128, ptx::sdesc_join(a_lo + off, kDescHi),
                        ptx::sdesc_join(b_lo + off, kDescHi), idesc_mxf8(kk, BN),
                        (static_cast<uint32_t>(kk) << 30) | sfa,
                        (static_cast<uint32_t>(kk) << 30) | sfb, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * BN * 128 + (kk & 3) * 32) >> 4;
            const uint32_t a_off = ((kk >> 2) * kBlockM * 128 + (kk & 3) * 32) >> 4;
            ptx::mma_f16_ss(tmem + t * 128, ptx::sdesc_join(a_lo + a_off, kDescHi),
                            ptx::sdesc_join(b_lo + off, kDescHi), kIdescS, kk > 0 ? 1u : 0u);
          }
        }
        if (commit) ptx::mma_commit(bar(Lay::kSFull + t));
      };
      // O_t += P_t V with V in ring stage st
      auto pv = [&](int t, int j, uint32_t st) {
        const uint32_t b_lo = ring_lo + st * (Lay::kSlotBytes >> 4) + v_lbo;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          ptx::mma_f16_ts(tmem + Lay::kTmemO + t * 128, tmem + t * 128 + kk * 8,
                          ptx::sdesc_join(b_lo + kk * (2048 >> 4), kDescHi), kIdescO,
                          (j == 0 && kk == 0) ? 0u : 1u);
      };
      for (uint32_t k = 0; ok; ++k) {
        const uint32_t uslot = k % kUnitSlots;
        if (!(ok = wait_one(bar(Lay::kUnitFull + uslot), (k / kUnitSlots) & 1, ctl))) break;
        const int4 uw = unit_ring[uslot];
        ptx::mbar_arrive(bar(Lay::kUnitEmpty + uslot));
        if (uw.y < 0) break;
        const int n_t[2] = {tile_steps(2 * uw.z, uw.y, causal, BN),
                            tile_steps(2 * uw.z + 1, uw.y, causal, BN)};
        const int n_max = max(n_t[0], n_t[1]);
        if (!(ok = wait_one(bar(Lay::kQFull), q_ph, ctl))) break;
        q_ph ^= 1;
        ptx::tc_fence_after();
        if constexpr (kFp8) {
          for (int t = 0; t < 2; ++t)
            for (int w = 0; w < Lay::kSfWords; ++w)
              tmem_cp_32x128b_x4(tmem + t * 128 + Lay::kTmemSfa + 4 * w,
                                 sf_copy_desc(sbase + Lay::kSfaOff + t * Lay::kSfBytes + 512 * w));
        }
        uint32_t st_k, st_v;
        if (!(ok = take_k(st_k))) break;
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) score(t, st_k, !(kFaultDropFirstScoreCommit && k == 0 && t == 0));
        ptx::mma_commit(bar(Lay::kKVEmpty + st_k));
        if (n_max == 1) ptx::mma_commit(bar(Lay::kQEmpty));
        for (int j = 0; j < n_max && ok; ++j) {
          if (!(ok = take(st_v))) break;
          bool k_taken = false;
          for (int t = 0; t < 2; ++t) {
            if (j >= n_t[t]) continue;
            if (!(ok = wait_one(bar(Lay::kPFull + t), g[t] & 1, ctl))) break;
            if constexpr (kFp8)
              if (j == 0 && !(ok = wait_one(bar(Lay::kOEmpty + t), (oe_cnt[t] & 1) ^ 1, ctl)))
                break;
            ptx::tc_fence_after();
            pv(t, j, st_v);
            if (j == n_t[t] - 1) {
              ptx::mma_commit(bar(Lay::kOUnit + t));
              ++oe_cnt[t];
            }
            ++g[t];
            if (j + 1 < n_t[t]) {
              if (!k_taken) {
                if (!(ok = take_k(st_k))) break;
                k_taken = true;
              }
              score(t, st_k);
            }
          }
          if (!ok) break;
          ptx::mma_commit(bar(Lay::kKVEmpty + st_v));
          if (j + 1 < n_max) {
            if (!k_taken && !(ok = take_k(st_k))) break;   // unreachable: n_max's tile needs it
            ptx::mma_commit(bar(Lay::kKVEmpty + st_k));
            if (j + 2 == n_max) ptx::mma_commit(bar(Lay::kQEmpty));
          }
        }
      }
      // Every product this thread issued must be complete before TMEM is freed.
      ptx::mma_commit(bar(Lay::kDrain));
      WaitCtl drain = ctl;
      uint32_t zero = 0;
      drain.abort_flag = &zero;
      wait_one(bar(Lay::kDrain), 0, drain);
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

}  // namespace attn

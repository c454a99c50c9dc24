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
// warps run the matrix products and the softmax.  On sm_100a this becomes
// (512 threads, registers re-split per role with setmaxnreg):
//
//   warps 0..3    softmax of query tile 0, warps 4..7 of query tile 1
//                 (184 registers): one thread per row reads its S row from
//                 TMEM, masks, updates m and l, writes P (bf16) back over S,
//                 and rescales O when its maximum grew by more than 2^8
//                 (lazy rescale).
//   warps 8..11   epilogue (80 registers): O / l to bf16 and the
//                 log-sum-exp, off the softmax warps' critical path.
//   warp 12       TMA producer: the Q tile pair of a unit, then K_j, V_j into
//                 a ring of shared-memory slots (mbarrier pipelined).
//   warp 13       MMA issuer (one thread): S_i = Q_i K_j^T into TMEM and
//                 O_i += P_i V_j with P_i read from TMEM (tcgen05.mma).
//   warps 14..15  idle (64 registers, like warps 12 and 13).
//
// While one softmax warpgroup works on its tile the tensor core computes the
// other tile's products (ping-pong), so the tensor pipe stays busy.  The
// exponentials are split between the MUFU unit (ex2) and a polynomial on the
// FMA pipe, so neither pipe alone limits the softmax.
//
// TMEM (512 columns, lane = query row): S_0 at column 0, S_1 at 128,
// O_0 at 256, O_1 at 256 + D.  P_i overwrites the first 64 columns of S_i.
// Shared memory: Q_0, Q_1 and kStages K/V slots of 128 x D bf16, each stored
// as D/64 column chunks of 128 rows x 128 bytes with the 128-byte swizzle
// the TMA writes and the tensor core reads; the softmax hands each row's
// log-sum-exp and 1 / l_round to the epilogue through a small shared array.
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

constexpr int kFwdThreads = 512;
// Registers per thread: 128 at launch (65536 / 512).  Each warpgroup moves
// once, at the start of its role, to that role's count and keeps it to the
// end.  No warpgroup ever raises its count again after lowering it: in a CTA
// with little or no work a lowered-then-raised warpgroup could take back the
// registers before the softmax warpgroups' increase is served, and that
// increase would then wait forever.
constexpr uint32_t kRegsEntry = 65536 / kFwdThreads;
constexpr uint32_t kRegsSoftmax = 184, kRegsEpilogue = 80, kRegsOther = 64;
static_assert(2 * kRegsSoftmax + kRegsEpilogue + kRegsOther == 4 * kRegsEntry,
              "register split must use exactly the registers the CTA is launched with");

// Which exponentials run on the FMA pipe: pairs k of a row with
// k % period == period - 1; the rest use MUFU ex2 (0 = MUFU only).
#ifndef ATTN_POLY_PAIR_PERIOD
#define ATTN_POLY_PAIR_PERIOD 0
#endif
constexpr int kPolyPairPeriod = ATTN_POLY_PAIR_PERIOD;

// 2^f on [0, 1): 1 + f (c1 + f (c2 + f c3)), a minimax fit of the relative
// error (max 8.6e-5) made by csrc/fit_exp2_poly.py; p(0) = 1 exactly.
constexpr float kExp2C1 = 6.951168180e-01f;
constexpr float kExp2C2 = 2.276448607e-01f;
constexpr float kExp2C3 = 7.706713676e-02f;

// Work units are claimed dynamically (heaviest first, from the sorted work
// list) by the TMA warp and handed to the other roles through a small ring.
constexpr int kUnitSlots = 4;
// Arrivals that release a unit slot: the MMA thread plus one per warp of the
// two softmax warpgroups and of the epilogue warpgroup.
constexpr int kUnitConsumers = 1 + 4 + 4 + 4;

template <int D>
struct FwdLayout {
  static constexpr int kChunks = D / 64;               // 128-byte chunks per row
  static constexpr int kChunkBytes = kBlockM * 128;    // one chunk of a tile
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  // K/V ring depth: as deep as shared memory allows (a K or V tile is
  // reused two steps after its load starts, so depth hides L2 / HBM latency).
  static constexpr int kStages = D == 128 ? 5 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kStatsOff = kKVOff + kStages * kTileBytes;   // float [2][2][128]
  static constexpr int kBarOff = kStatsOff + 2 * 2 * kBlockM * 4;
  // barrier indices
  static constexpr int kQFull = 0, kQEmpty = 1;
  static constexpr int kKVFull = 2;                    // + stage
  static constexpr int kKVEmpty = 2 + kStages;         // + stage
  static constexpr int kSFull = 2 + 2 * kStages;       // + tile
  static constexpr int kPFull = kSFull + 2;            // + tile
  static constexpr int kOFull = kPFull + 2;            // + tile
  static constexpr int kOEmpty = kOFull + 2;           // + tile
  static constexpr int kStFull = kOEmpty + 2;          // + tile
  static constexpr int kStEmpty = kStFull + 2;         // + tile
  static constexpr int kDrain = kStEmpty + 2;
  static constexpr int kUnitFull = kDrain + 1;         // + slot
  static constexpr int kUnitEmpty = kUnitFull + kUnitSlots;   // + slot
  static constexpr int kNumBars = kUnitEmpty + kUnitSlots;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kUnitOff = kMiscOff + 16;           // int32 [kUnitSlots]
  static constexpr int kBytes = kUnitOff + 4 * kUnitSlots;
  static constexpr int kAllocBytes = kBytes;           // base is 1024-byte aligned
  static_assert(kAllocBytes <= 232448, "exceeds the 227 KB of shared memory per CTA");
  static constexpr uint32_t kTmemCols = 512;
};

// Bounded waits.  A wait gives up when the CTA's abort flag is raised or
// after timeout_ns; the first thread to give up records ATTN_ERR_TIMEOUT.
// They are inlined and take their control block by value: a real call with
// a stack frame cannot be register-allocated inside a setmaxnreg region.
struct WaitCtl {
  volatile uint32_t* abort_flag;
  int32_t* err;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void raise_abort(WaitCtl c) {
  if (*c.abort_flag == 0) {
    *c.abort_flag = 1;
    atomicCAS(c.err, 0, (int)ATTN_ERR_TIMEOUT);
  }
}

// Single-thread bounded wait.
__device__ __forceinline__ bool wait_one(uint32_t bar, uint32_t parity, WaitCtl c) {
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
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, WaitCtl c) {
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

// Last key step of query tile `i`.
__device__ __forceinline__ int last_step(const UnitInfo& ui, int i, int causal) {
  return causal ? min(kTilesPerUnit * ui.pair + i, ui.kv_tiles - 1) : ui.kv_tiles - 1;
}

// 2^x for a pair of x <= 8 on the FMA pipe.  x = j + f with j = floor(x)
// (taken from adding 1.5 * 2^23 rounded down, which leaves j in the low
// mantissa bits), 2^f from the polynomial, and j added to the exponent
// field.  x is clamped at -127 first, where the result is exactly +0 (the
// exponent field of p(0) = 1 cancels), so masked scores (-inf) give 0.
__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = ptx::f2_pack(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
  const float kMagic = 12582912.f;   // 1.5 * 2^23
  const uint64_t t = ptx::f2_add_rm(x, ptx::f2_pack(kMagic, kMagic));
  const uint64_t jf = ptx::f2_add(t, ptx::f2_pack(-kMagic, -kMagic));
  const uint64_t f = ptx::f2_fma(jf, ptx::f2_pack(-1.f, -1.f), x);
  uint64_t q = ptx::f2_fma(ptx::f2_pack(kExp2C3, kExp2C3), f, ptx::f2_pack(kExp2C2, kExp2C2));
  q = ptx::f2_fma(q, f, ptx::f2_pack(kExp2C1, kExp2C1));
  q = ptx::f2_fma(q, f, ptx::f2_pack(1.f, 1.f));
  float q0, q1, t0, t1;
  ptx::f2_unpack(q, q0, q1);
  ptx::f2_unpack(t, t0, t1);
  y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Lay = FwdLayout<D>;
  // The kernel has no static shared memory, so the dynamic block starts at
  // the CTA's (1024-byte aligned) shared window; the 128-byte swizzle needs
  // that alignment.  Checked anyway: a misaligned base records an error and
  // the CTA leaves before touching anything.
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
  // [tile][lse in log2 units, 1 / l_round][row]
  float* stats = reinterpret_cast<float*>(smem + Lay::kStatsOff);

  constexpr int kWarpTma = 12, kWarpMma = 13;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(Lay::kQFull), 1);
    ptx::mbar_init(bar(Lay::kQEmpty), 1);
    for (int s = 0; s < Lay::kStages; ++s) {
      ptx::mbar_init(bar(Lay::kKVFull + s), 1);
      ptx::mbar_init(bar(Lay::kKVEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(Lay::kSFull + i), 1);
      ptx::mbar_init(bar(Lay::kPFull + i), 4);    // one arrival per softmax warp
      ptx::mbar_init(bar(Lay::kOFull + i), 1);
      ptx::mbar_init(bar(Lay::kOEmpty + i), 4);   // one arrival per epilogue warp
      ptx::mbar_init(bar(Lay::kStFull + i), 4);
      ptx::mbar_init(bar(Lay::kStEmpty + i), 4);
    }
    ptx::mbar_init(bar(Lay::kDrain), 1);
    for (int i = 0; i < kUnitSlots; ++i) {
      ptx::mbar_init(bar(Lay::kUnitFull + i), 1);
      ptx::mbar_init(bar(Lay::kUnitEmpty + i), kUnitConsumers);
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
  const int n_units = p.ws_header[kWsCountOffset / 4] * H;
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + Lay::kUnitOff);
  // Consumer side of the unit ring: the k-th unit of this CTA, or -1 when the
  // work is exhausted (also -1 if the wait gave up; `ok` says which).
  auto next_unit_warp = [&](uint32_t k, bool& ok) -> int {
    const uint32_t slot = k % kUnitSlots;
    if (!(ok = wait_warp(bar(Lay::kUnitFull + slot), (k / kUnitSlots) & 1, ctl))) return -1;
    const int u = unit_ring[slot];
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar(Lay::kUnitEmpty + slot));
    return u;
  };

  if (warp < 8) {
    // ------------------------------------------------------------ softmax
    ptx::regs_increase<kRegsSoftmax>();
    const int tile = warp >> 2;
    const int wq = warp & 3;                      // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;                 // row within the query tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_off + tile * 128;
    const uint32_t t_o = tmem + lane_off + 256 + tile * D;
    const float c = p.scale_log2;
    const uint64_t c2 = ptx::f2_pack(c, c);
    uint32_t s_cnt = 0, o_cnt = 0, st_cnt = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int u = next_unit_warp(k, ok);
      if (u < 0) break;
      const UnitInfo ui = decode_unit(p.work, u, H, causal);
      if (tile == 1 && !ui.tile1_valid) continue;
      const int qb = kTilesPerUnit * ui.pair + tile;
      const int last = last_step(ui, tile, causal);
      float m_used = -INFINITY;   // running maximum in log2 units
      float l = 0.f;              // sum of the weights
      float l_round = 0.f;        // sum of the weights as rounded to bf16
      for (int j = 0; j <= last; ++j) {
        if (!(ok = wait_warp(bar(Lay::kSFull + tile), s_cnt & 1, ctl))) break;
        ++s_cnt;
        ptx::tc_fence_after();
        uint32_t sa[64], sb[64];
        ptx::tmem_ld_x64(t_s, sa);
        ptx::tmem_ld_x64(t_s + 64, sb);
        float s[128];
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          s[k] = __uint_as_float(sa[k]);
          s[64 + k] = __uint_as_float(sb[k]);
        }
        const bool diag = causal && j == qb;
        if (diag || (j + 1) * kBlockN > ui.doc_len) {
          int limit = ui.doc_len - j * kBlockN;
          if (diag) limit = min(limit, r + 1);
#pragma unroll
          for (int k = 0; k < 128; ++k)
            if (k >= limit) s[k] = -INFINITY;
        }
        float mx0 = ptx::fmax3(s[0], s[1], s[2]);
        float mx1 = ptx::fmax3(s[3], s[4], s[5]);
        float mx2 = ptx::fmax3(s[6], s[7], s[8]);
        float mx3 = ptx::fmax3(s[9], s[10], s[11]);
#pragma unroll
        for (int k = 12; k < 124; k += 8) {
          mx0 = ptx::fmax3(mx0, s[k], s[k + 1]);
          mx1 = ptx::fmax3(mx1, s[k + 2], s[k + 3]);
          mx2 = ptx::fmax3(mx2, s[k + 4], s[k + 5]);
          mx3 = ptx::fmax3(mx3, s[k + 6], s[k + 7]);
        }
        mx0 = ptx::fmax3(mx0, s[124], s[125]);
        mx1 = ptx::fmax3(mx1, s[126], s[127]);
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
        const uint64_t nb2 = ptx::f2_pack(-base, -base);
        uint64_t se[2], sq[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) se[a] = sq[a] = ptx::f2_pack(0.f, 0.f);
        // Four chunks of 32 keys: exponentiate, round, and store each chunk
        // of P to TMEM before starting the next, so only one chunk of packed
        // weights is live at a time.
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const int k = ch * 16 + kk;
            const uint64_t x = ptx::f2_fma(ptx::f2_pack(s[2 * k], s[2 * k + 1]), c2, nb2);
            float x0, x1, p0, p1;
            ptx::f2_unpack(x, x0, x1);
            if (kPolyPairPeriod > 0 && k % (kPolyPairPeriod > 0 ? kPolyPairPeriod : 1) == kPolyPairPeriod - 1) {
              exp2_poly_pair(x0, x1, p0, p1);
            } else {
              p0 = ptx::ex2_approx(x0);
              p1 = ptx::ex2_approx(x1);
            }
            pk[kk] = ptx::pack_bf16x2(p0, p1);
            se[kk & 1] = ptx::f2_add(se[kk & 1], ptx::f2_pack(p0, p1));
            sq[kk & 1] = ptx::f2_add(sq[kk & 1], ptx::f2_pack(__uint_as_float(pk[kk] << 16),
                                                              __uint_as_float(pk[kk] & 0xFFFF0000u)));
          }
          ptx::tmem_st_x16(t_s + ch * 16, pk);
        }
        const uint64_t se_all = ptx::f2_add(se[0], se[1]);
        const uint64_t sq_all = ptx::f2_add(sq[0], sq[1]);
        float e0, e1, q0, q1;
        ptx::f2_unpack(se_all, e0, e1);
        ptx::f2_unpack(sq_all, q0, q1);
        l += e0 + e1;
        l_round += q0 + q1;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kPFull + tile));
      }
      if (!ok) break;
      o_cnt += last + 1;
      // hand the row's statistics to the epilogue warps
      if (!(ok = wait_warp(bar(Lay::kStEmpty + tile), (st_cnt & 1) ^ 1, ctl))) break;
      ++st_cnt;
      float* st = stats + tile * 2 * kBlockM;
      st[r] = m_used + __log2f(l);
      st[kBlockM + r] = 1.f / l_round;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(Lay::kStFull + tile));
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ epilogue
    ptx::regs_decrease<kRegsEpilogue>();
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint32_t sf_cnt[2] = {0, 0}, o_cnt[2] = {0, 0};
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int u = next_unit_warp(k, ok);
      if (u < 0) break;
      const UnitInfo ui = decode_unit(p.work, u, H, causal);
#pragma unroll
      for (int tile = 0; tile < 2; ++tile) {
        if (!ok || (tile == 1 && !ui.tile1_valid)) continue;
        const int qb = kTilesPerUnit * ui.pair + tile;
        const int last = last_step(ui, tile, causal);
        if (!(ok = wait_warp(bar(Lay::kStFull + tile), sf_cnt[tile] & 1, ctl))) break;
        ++sf_cnt[tile];
        const float* st = stats + tile * 2 * kBlockM;
        const float lse2 = st[r], inv_l = st[kBlockM + r];
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kStEmpty + tile));
        if (!(ok = wait_warp(bar(Lay::kOFull + tile), (o_cnt[tile] + last) & 1, ctl))) break;
        o_cnt[tile] += last + 1;
        ptx::tc_fence_after();
        const int row_doc = qb * kBlockM + r;
        const bool row_ok = row_doc < ui.doc_len;
        const long long token = static_cast<long long>(ui.doc_start) + row_doc;
        uint4* orow =
            reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + (token * H + ui.head) * D);
        const uint32_t t_o = tmem + lane_off + 256 + tile * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          ptx::tmem_ld_x32(t_o + cc * 32, o);
          if (cc == D / 32 - 1) {
            // O is in registers: the tensor core may overwrite it now.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(Lay::kOEmpty + tile));
          }
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
              lse2 * 0.69314718055994530942f;
      }
    }
  } else {
    // One setmaxnreg for the whole warpgroup (warps 12..15), as required.
    ptx::regs_decrease<kRegsOther>();
    if (warp == kWarpTma && lane == 0) {
    // ------------------------------------------------------------ producer
      uint32_t q_it = 0, kv_it = 0;
      bool ok = true;
      int* counter = const_cast<int*>(p.ws_header) + kWsUnitCounterOffset / 4;
      for (uint32_t k = 0; ok; ++k) {
        // Claim the next unit: the first one statically, the rest from the
        // shared counter, so each CTA takes the heaviest unit left whenever
        // it runs out of work (the list is sorted by cost).
        const int claim = k == 0 ? static_cast<int>(blockIdx.x)
                                 : static_cast<int>(gridDim.x) + atomicAdd(counter, 1);
        const int u = claim < n_units ? claim : -1;
        const uint32_t slot = k % kUnitSlots;
        if (!(ok = wait_one(bar(Lay::kUnitEmpty + slot), ((k / kUnitSlots) & 1) ^ 1, ctl))) break;
        unit_ring[slot] = u;
        ptx::mbar_arrive(bar(Lay::kUnitFull + slot));
        if (u < 0) break;
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
    } else if (warp == kWarpMma && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
      // The issuing thread sits on the critical path between a softmax
      // warpgroup's P and its next S, so the loop is kept lean: descriptors
      // are precomputed 32-bit halves (advancing along K only adds to the low
      // half) and the per-tile state lives in registers (no runtime-indexed
      // arrays, which would go to local memory).
      constexpr uint32_t kIdescS = ptx::idesc_bf16(kBlockM, kBlockN, 0);
      constexpr uint32_t kIdescO = ptx::idesc_bf16(kBlockM, D, 1);
      constexpr uint32_t kDescHi = ptx::sdesc_hi_sw128(1024);
      const uint32_t q_lo0 = ptx::sdesc_lo(sbase + Lay::kQOff, 16);
      const uint32_t q_lo1 = ptx::sdesc_lo(sbase + Lay::kQOff + Lay::kTileBytes, 16);
      const uint32_t kv_lo = ptx::sdesc_lo(sbase + Lay::kKVOff, 16);
      const uint32_t v_lbo = static_cast<uint32_t>(Lay::kChunkBytes - 16) >> 4 << 16;
      uint32_t q_it = 0, kv_it = 0;
      uint32_t p_cnt0 = 0, p_cnt1 = 0, oe_cnt0 = 0, oe_cnt1 = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const uint32_t slot = k % kUnitSlots;
        if (!(ok = wait_one(bar(Lay::kUnitFull + slot), (k / kUnitSlots) & 1, ctl))) break;
        const int u = unit_ring[slot];
        ptx::mbar_arrive(bar(Lay::kUnitEmpty + slot));
        if (u < 0) break;
        const UnitInfo ui = decode_unit(p.work, u, H, causal);
        const int n = ui.n_kv_steps;
        if (!(ok = wait_one(bar(Lay::kQFull), q_it & 1, ctl))) break;
        ++q_it;
        ptx::tc_fence_after();
        bool first_pv0 = true, first_pv1 = true;
        const uint32_t kv_base = kv_it;
        for (int j = 0; ok && j <= n; ++j) {
          const uint32_t idx_v = kv_base + 2 * (j - 1) + 1;
          const uint32_t idx_k = kv_base + 2 * j;
          const uint32_t st_v = idx_v % Lay::kStages, st_k = idx_k % Lay::kStages;
          bool v_ready = false, k_ready = false;
          // P_i V_{j-1} into O_i (A operand = P_i from TMEM)
          auto pv = [&](const int i, uint32_t& p_cnt, uint32_t& oe_cnt, bool& first) -> bool {
            if (!v_ready) {
              if (!wait_one(bar(Lay::kKVFull + st_v), (idx_v / Lay::kStages) & 1, ctl)) return false;
              v_ready = true;
            }
            if (!wait_one(bar(Lay::kPFull + i), p_cnt & 1, ctl)) return false;
            ++p_cnt;
            if (first) {
              if (!wait_one(bar(Lay::kOEmpty + i), (oe_cnt & 1) ^ 1, ctl)) return false;
              ++oe_cnt;
            }
            ptx::tc_fence_after();
            const uint32_t t_o = tmem + 256 + i * D;
            const uint32_t t_p = tmem + i * 128;
            const uint32_t b_lo = (kv_lo + st_v * (Lay::kTileBytes >> 4)) + v_lbo;
#pragma unroll
            for (int kk = 0; kk < kBlockN / 16; ++kk)
              ptx::mma_f16_ts(t_o, t_p + kk * 8, ptx::sdesc_join(b_lo + kk * (2048 >> 4), kDescHi),
                              kIdescO, (first && kk == 0) ? 0u : 1u);
            first = false;
            ptx::mma_commit(bar(Lay::kOFull + i));
            return true;
          };
          // S_i = Q_i K_j^T
          auto qk = [&](const int i) -> bool {
            if (!k_ready) {
              if (!wait_one(bar(Lay::kKVFull + st_k), (idx_k / Lay::kStages) & 1, ctl)) return false;
              ptx::tc_fence_after();
              k_ready = true;
            }
            const uint32_t a_lo = i == 0 ? q_lo0 : q_lo1;
            const uint32_t b_lo = kv_lo + st_k * (Lay::kTileBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * Lay::kChunkBytes + (kk & 3) * 32) >> 4;
              ptx::mma_f16_ss(tmem + i * 128, ptx::sdesc_join(a_lo + off, kDescHi),
                              ptx::sdesc_join(b_lo + off, kDescHi), kIdescS, kk > 0 ? 1u : 0u);
            }
            ptx::mma_commit(bar(Lay::kSFull + i));
            return true;
          };
          if (j > 0 && tile_active(ui, 0, j - 1, causal))
            if (!(ok = pv(0, p_cnt0, oe_cnt0, first_pv0))) break;
          if (j < n && tile_active(ui, 0, j, causal))
            if (!(ok = qk(0))) break;
          if (j > 0 && tile_active(ui, 1, j - 1, causal))
            if (!(ok = pv(1, p_cnt1, oe_cnt1, first_pv1))) break;
          if (j < n && tile_active(ui, 1, j, causal))
            if (!(ok = qk(1))) break;
          if (j > 0) {
            if (!v_ready && !(ok = wait_one(bar(Lay::kKVFull + st_v), (idx_v / Lay::kStages) & 1, ctl)))
              break;
            ptx::mma_commit(bar(Lay::kKVEmpty + st_v));
          }
          if (j < n) {
            if (!k_ready && !(ok = wait_one(bar(Lay::kKVFull + st_k), (idx_k / Lay::kStages) & 1, ctl)))
              break;
            ptx::mma_commit(bar(Lay::kKVEmpty + st_k));
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

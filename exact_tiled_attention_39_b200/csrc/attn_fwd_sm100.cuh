// Exact attention forward for sm_100a, MXFP8: persistent, warp-specialised,
// TMA + tcgen05 + TMEM, with the score product block-scaled (E4M3 operands,
// E8M0 scales) and P V in bf16 on the exactly dequantised values.  Also the
// helpers (bounded waits, unit decode, exponentials) the bf16 kernel in
// attn_fwd_pair_sm100.cuh uses.  The host instantiates it for head dim 128
// with MXFP8 operands; the template keeps a bf16 mode (kFp8 = false).
//
// The method ("FlashAttention và IO" (aihero.vn), sections "Tiling giữ công
// việc ở gần nơi tính" and "Softmax qua nhiều khối cần thống kê chạy"):
// Q, K and V are cut into tiles held on chip; for each query row the kernel
// keeps the running maximum m, the normaliser l and the weighted sum u (the
// output accumulator O), multiplies the old part by exp(m - m_new) when a new
// key tile raises the maximum, and writes u / l and the log-sum-exp at the
// end.  Scores and probabilities never leave the SM.
//
// Loop order and roles follow "FlashAttention, pelatihan multi-GPU, dan
// kuantisasi bobot" (section 1): outer loop over query blocks, inner over
// key/value blocks; a producer issues asynchronous tile copies while other
// warps run the products and the softmax.  The MXFP8 products follow
// "FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin
// Flash Mikro-Ölçeklemeli Dikkat Mekanizması" (section "FLAMIA Mimarisi ve
// Temel Tasarım İlkeleri"): block-scaled low-precision products whose scales
// (one per token, head and 32 head-dim elements) never span two tokens.
//
// A work unit is one 128-row query tile of one document and head (the scale
// factors take the TMEM a second query tile would need).  On sm_100a (512
// threads, registers re-split per warpgroup with setmaxnreg):
//
//   warps 0..7    softmax (168 registers), two warpgroups on the same rows:
//                 warpgroup h takes keys [64 h, 64 h + 64) of every score
//                 tile.  Each thread reads its half row from TMEM and masks
//                 it; the two halves swap their maxima through shared memory,
//                 so both use the same running maximum m; each writes its
//                 half of P (bf16) back over its own scores, keeps its part of
//                 l, and rescales its half of O when the row maximum grew by
//                 more than 2^8 (lazy rescale).
//   warps 8..11   epilogue (96 registers): O / l to bf16 and the log-sum-exp.
//   warp 12       producer (80 registers): claims units, TMA loads of Q and of
//                 K_j, V_j into a ring of shared-memory slots; the whole warp
//                 also stages the E8M0 scale blocks.
//   warp 13       MMA issuer (one thread): S = Q K_j^T into one of two TMEM
//                 score buffers, O += P V_j with P read from TMEM.
//   warps 14..15  idle.
//
// The score buffers alternate between key steps, so while the softmax works
// on step j the tensor core computes P_{j-1} V_{j-1} and S_{j+1}.  Splitting
// a row between two warps halves the softmax latency of a step and puts two
// softmax warps on every SM sub-partition.
//
// TMEM (512 columns, lane = query row): S buffers at columns 0 and 128 (the
// P half of warpgroup h overwrites columns [64 h, 64 h + 32) of its buffer),
// O at 256, the scale factors of Q at 384 and of the current K tile at
// 388 / 392.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"

namespace attn {

struct FwdParams {
  void* out;                 // bf16 [T, H, D]
  float* lse;                // fp32 [H, T]
  const int32_t* ws_header;  // error word, work-list length, unit counter
  const int4* work;          // work list
  int32_t* err;              // error word (device)
  const uint32_t* q_scales;  // MXFP8: E8M0 words [T, H] (4 scales per word);
  const uint32_t* k_scales;  // NVFP4: UE4M3 words [T, H, 2] (4 scales per word)
  int total_tokens;
  int num_heads;
  int head_groups;           // unit order: heads in this many groups (see common.cuh)
  int causal;
  float scale_log2;          // scale * log2(e)
  unsigned long long timeout_ns;
};

constexpr int kFwdThreads = 512;
// Registers per thread at launch: 65536 / 512.  Each warpgroup moves once, at
// the start of its role, and keeps that count: a warpgroup that lowered its
// count and raised it again could take back registers before the softmax
// warpgroups' increase is served.
constexpr uint32_t kRegsEntry = 128;
constexpr uint32_t kRegsSoftmax = 168, kRegsEpilogue = 96, kRegsOther = 80;
static_assert(2 * kRegsSoftmax + kRegsEpilogue + kRegsOther == 4 * kRegsEntry,
              "register split must use exactly the registers the CTA is launched with");

constexpr int kSoftmaxWarps = 8;            // two warpgroups, one per half of the keys
constexpr int kHalfKeys = kBlockN / 2;
constexpr int kUnitSlots = 4;
constexpr int kUnitConsumers = 1 + kSoftmaxWarps + 4;   // MMA thread + softmax + epilogue warps


// Operand format of the score product Q K^T: bf16, MXFP8 (E4M3 codes, one
// E8M0 scale per 32 elements) or NVFP4 (E2M1 codes two per byte, one
// unsigned E4M3 scale per 16 elements).
constexpr int kQkBf16 = 0, kQkMx8 = 1, kQkNv4 = 2;

template <int D, int kQk>
struct FwdLayout {
  static constexpr bool kFp8 = kQk != kQkBf16;                // Q, K as block-scaled codes
  static constexpr bool kNv4 = kQk == kQkNv4;
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static_assert(!kFp8 || D == 128, "the block-scaled kernel is built for head dim 128");
  static constexpr int kQKChunks = kFp8 ? 1 : D / 64;         // swizzle-wide chunks per Q/K row
  static constexpr int kQKRowBytes = kNv4 ? 64 : 128;         // bytes of a row in one chunk
  static constexpr int kVChunks = D / 64;                     // V is bf16
  static constexpr int kChunkBytes = kBlockM * 128;           // 128 rows x 128 bytes
  static constexpr int kQKChunkBytes = kBlockM * kQKRowBytes;
  static constexpr int kQBytes = kQKChunks * kQKChunkBytes;
  static constexpr int kKBytes = kQKChunks * kQKChunkBytes;
  static constexpr int kVBytes = kVChunks * kChunkBytes;
  // Scale blocks of a tile: 32 rows x 16 bytes each, one per 32-bit scale
  // word of a row (MXFP8: 4 E8M0 bytes cover the 128 elements; NVFP4: two
  // words of 4 UE4M3 bytes, one per 64 elements).
  static constexpr int kSfWords = kNv4 ? 2 : 1;
  static constexpr int kSfBytes = 512 * kSfWords;
  static constexpr int kSlotBytes = kVBytes;                  // a V tile, or a K tile + scales
  static_assert(kKBytes + (kFp8 ? kSfBytes : 0) <= kSlotBytes, "K tile must fit a slot");
  static constexpr int kQOff = 0;
  static constexpr int kSfaOff = kQBytes;                     // MXFP8 only
  static constexpr int kRingOff = ((kQBytes + (kFp8 ? kSfBytes : 0)) + 1023) / 1024 * 1024;
  static constexpr int kReserve = 6144;                       // stats, maxima, barriers, units
  static constexpr int kStagesFit = (232448 - kRingOff - kReserve) / kSlotBytes;
  static constexpr int kStages = kStagesFit > 10 ? 10 : kStagesFit;
  // Unit statistics handed to the epilogue: float [5][128] = m, then l and
  // the rounded l of each half.  Half-row maxima: float [2 steps][2][128].
  static constexpr int kStatsOff = kRingOff + kStages * kSlotBytes;
  static constexpr int kXmaxOff = kStatsOff + 5 * kBlockM * 4;
  static constexpr int kBarOff = kXmaxOff + 2 * 2 * kBlockM * 4;
  static constexpr int kQFull = 0, kQEmpty = 1;
  static constexpr int kKVFull = 2;                           // + stage
  static constexpr int kKVEmpty = kKVFull + kStages;          // + stage
  static constexpr int kSFull = kKVEmpty + kStages;           // + buffer
  static constexpr int kPFull = kSFull + 2;                   // + buffer
  // O of a unit complete (one phase per unit: a waiter is never more than one
  // phase behind, which a parity wait needs)
  static constexpr int kOUnit = kPFull + 2;
  static constexpr int kOEmpty = kOUnit + 1;
  static constexpr int kStFull = kOEmpty + 1;
  static constexpr int kStEmpty = kStFull + 1;
  static constexpr int kXFull = kStEmpty + 1;                // + step parity
  static constexpr int kPFree = kXFull + 2;                   // + buffer: P V of that buffer done
  static constexpr int kDrain = kPFree + 2;
  static constexpr int kUnitFull = kDrain + 1;                // + slot
  static constexpr int kUnitEmpty = kUnitFull + kUnitSlots;   // + slot
  static constexpr int kNumBars = kUnitEmpty + kUnitSlots;
  static constexpr int kMiscOff = (kBarOff + kNumBars * 8 + 15) / 16 * 16;   // tmem base, abort flag
  static constexpr int kUnitOff = kMiscOff + 16;              // int4 [kUnitSlots]
  static constexpr int kBytes = kUnitOff + 16 * kUnitSlots;
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory per CTA");
  static_assert(kBytes - kStatsOff <= kReserve, "reserve too small");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 256, kTmemSfa = 384;
  static constexpr uint32_t kTmemSfb = kTmemSfa + 4 * kSfWords;   // + 4 * kSfWords * buffer
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
  int doc_start, doc_len, qb, head, kv_tiles, n;   // n = key steps of this tile
};

// Unit from its ring entry (doc_start, doc_len, query block, head).
__device__ __forceinline__ UnitInfo decode_unit(int4 w, int causal) {
  UnitInfo r;
  r.doc_start = w.x;
  r.doc_len = w.y;
  r.qb = w.z;
  r.head = w.w;
  r.kv_tiles = (w.y + kBlockN - 1) / kBlockN;
  r.n = causal ? min(w.z + 1, r.kv_tiles) : r.kv_tiles;
  return r;
}

// Shared-memory descriptor of a 32-row x 16-byte block of E8M0 scales for
// tcgen05.cp (K-major, no swizzle: 8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_copy_desc(uint32_t saddr) {
  return ptx::sdesc_join(ptx::sdesc_lo(saddr, 512), ((128u >> 4) & 0x3FFFu) | (1u << 14));
}

// Instruction descriptor for the block-scaled E4M3 x E4M3 product (fp32
// accumulate, E8M0 scales, M = 128, N = n, K = 32); sf_id picks the scale
// byte (the 32-element block) inside each 32-bit scale column.
__host__ __device__ constexpr uint32_t idesc_mxf8(uint32_t sf_id, int n = kBlockN) {
  return (sf_id << 4)                         // B scale id
         | (0u << 7) | (0u << 10)             // A, B format: E4M3
         | (static_cast<uint32_t>(n >> 3) << 17)
         | (1u << 23)                         // scale format: E8M0
         | (static_cast<uint32_t>(kBlockM >> 4) << 24)
         | (sf_id << 29);                     // A scale id
}

// Instruction descriptor for the block-scaled E2M1 x E2M1 product (fp32
// accumulate, unsigned E4M3 scales, one per 16 elements, M = N = 128,
// K = 64): the scale ids are 0, each instruction reads a whole 32-bit scale
// word per row.
__host__ __device__ constexpr uint32_t idesc_nvf4() {
  return (1u << 7) | (1u << 10)               // A, B format: E2M1
         | (static_cast<uint32_t>(kBlockN >> 3) << 17)
         | (0u << 23)                         // scale format: UE4M3
         | (static_cast<uint32_t>(kBlockM >> 4) << 24);
}

__device__ __forceinline__ void mma_nvf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void mma_mxf8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Copy a 32-row x 128-bit block from shared memory to TMEM lanes 0..31 and
// replicate it into the other three lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D, int kQk>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Lay = FwdLayout<D, kQk>;
  constexpr bool kFp8 = Lay::kFp8;
  constexpr bool kNv4 = Lay::kNv4;
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
  float* stats = reinterpret_cast<float*>(smem + Lay::kStatsOff);   // [m, l0, lr0, l1, lr1][row]
  float* xmax = reinterpret_cast<float*>(smem + Lay::kXmaxOff);     // [step & 1][half][row]
  // Units handed from the producer to the other roles, decoded (doc_len < 0
  // marks the end of the work).
  int4* unit_ring = reinterpret_cast<int4*>(smem + Lay::kUnitOff);

  constexpr int kWarpTma = 12, kWarpMma = 13;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(Lay::kQFull), 1);
    ptx::mbar_init(bar(Lay::kQEmpty), 1);
    for (int s = 0; s < Lay::kStages; ++s) {
      ptx::mbar_init(bar(Lay::kKVFull + s), 1);
      ptx::mbar_init(bar(Lay::kKVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(Lay::kSFull + b), 1);
      ptx::mbar_init(bar(Lay::kPFull + b), kSoftmaxWarps);   // one arrival per softmax warp
      ptx::mbar_init(bar(Lay::kXFull + b), kSoftmaxWarps);
      ptx::mbar_init(bar(Lay::kPFree + b), 1);
    }
    ptx::mbar_init(bar(Lay::kOUnit), 1);
    ptx::mbar_init(bar(Lay::kOEmpty), 4);         // one arrival per epilogue warp
    ptx::mbar_init(bar(Lay::kStFull), kSoftmaxWarps);
    ptx::mbar_init(bar(Lay::kStEmpty), 4);
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
  // Consumer side of the unit ring: the k-th unit of this CTA; doc_len < 0
  // when the work is exhausted (also if the wait gave up; `ok` says which).
  auto next_unit_warp = [&](uint32_t k, bool& ok) -> int4 {
    const uint32_t slot = k % kUnitSlots;
    if (!(ok = wait_warp(bar(Lay::kUnitFull + slot), (k / kUnitSlots) & 1, ctl)))
      return make_int4(0, -1, 0, 0);
    const int4 w = unit_ring[slot];   // after the wait (asm with a memory clobber)
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar(Lay::kUnitEmpty + slot));
    return w;
  };

  if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax
    ptx::regs_increase<kRegsSoftmax>();
    const int h = warp >> 2;                      // which half of the keys
    const int r = (warp & 3) * 32 + lane;         // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_off + Lay::kTmemO + h * (D / 2);
    const float c = p.scale_log2;
    const uint64_t c2 = ptx::f2_pack(c, c);
    uint32_t g = 0, st_cnt = 0;                   // global key step, units handed over
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int4 uw = next_unit_warp(k, ok);
      if (uw.y < 0) break;
      const UnitInfo ui = decode_unit(uw, causal);
      float m_used = -INFINITY;   // running maximum in log2 units (same in both halves)
      float l = 0.f;              // this half's sum of the weights
      float l_round = 0.f;        // the same, of the weights as rounded to bf16
      for (int j = 0; j < ui.n; ++j, ++g) {
        const uint32_t buf = g & 1;
        const uint32_t t_s = tmem + lane_off + buf * 128 + h * kHalfKeys;
        if (!(ok = wait_warp(bar(Lay::kSFull + buf), (g >> 1) & 1, ctl))) break;
        ptx::tc_fence_after();
        uint32_t sa[64];
        ptx::tmem_ld_x64(t_s, sa);
        float s[64];
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] = __uint_as_float(sa[q]);
        const bool diag = causal && j == ui.qb;
        if (diag || (j + 1) * kBlockN > ui.doc_len) {
          int limit = ui.doc_len - j * kBlockN;
          if (diag) limit = min(limit, r + 1);
          limit -= h * kHalfKeys;
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if (q >= limit) s[q] = -INFINITY;
        }
        // Maximum of this half (8 independent chains), then of the row: the
        // two halves swap theirs through shared memory.
        float mx[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmaxf(s[2 * a], s[2 * a + 1]);
#pragma unroll
        for (int q = 16; q < 64; q += 16)
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = ptx::fmax3(mx[a], s[q + 2 * a], s[q + 2 * a + 1]);
        const float m_half = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        float* xm = xmax + buf * 2 * kBlockM;
        xm[h * kBlockM + r] = m_half;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kXFull + buf));
        if (!(ok = wait_warp(bar(Lay::kXFull + buf), (g >> 1) & 1, ctl))) break;
        const float m_tile = fmaxf(m_half, xm[(h ^ 1) * kBlockM + r]) * c;
        if (j == 0) {
          m_used = m_tile;
        } else {
          // Rescale only rows whose maximum grew past the threshold.  TMEM
          // access is warp-wide, so the other rows of the warp take part with
          // a factor of exactly 1: a row's arithmetic never depends on other
          // rows' data.  Both halves of a row take the same decision.
          const bool need = m_tile > m_used + kRescaleTau;
          if (__any_sync(0xffffffffu, need)) {
            // O may only be touched once the previous P V product is done.
            // Its buffer's barrier has one phase per two steps and this warp
            // has seen the phase before (P V two steps further back) complete
            // already, so the parity names exactly P_{j-1} V_{j-1}.
            if (!(ok = wait_warp(bar(Lay::kPFree + ((g - 1) & 1)), ((g - 1) >> 1) & 1, ctl))) break;
            ptx::tc_fence_after();
            const float m_next = need ? m_tile : m_used;
            const float alpha = need ? ptx::ex2_approx(m_used - m_next) : 1.f;
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
              uint32_t o[32];
              ptx::tmem_ld_x32(t_o + cc * 32, o);
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
              ptx::tmem_st_x32(t_o + cc * 32, o);
            }
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
        // P of this step goes over this half's scores.  The P V product two
        // steps back has read that buffer already (these scores came after
        // it); the wait on its barrier, after the weights are formed, keeps
        // this warp at most one phase behind each buffer's barrier.
        const uint32_t t_p = t_s;
        {
          const float base = m_used == -INFINITY ? 0.f : m_used;
          const uint64_t nb2 = ptx::f2_pack(-base, -base);
          uint64_t se[2];
          float sr[4];
#pragma unroll
          for (int a = 0; a < 2; ++a) se[a] = ptx::f2_pack(0.f, 0.f);
#pragma unroll
          for (int a = 0; a < 4; ++a) sr[a] = 0.f;
          uint32_t pk[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const uint64_t x = ptx::f2_fma(ptx::f2_pack(s[2 * q], s[2 * q + 1]), c2, nb2);
            float x0, x1, p0, p1;
            ptx::f2_unpack(x, x0, x1);
            p0 = ptx::ex2_approx(x0);
            p1 = ptx::ex2_approx(x1);
            pk[q] = ptx::pack_bf16x2(p0, p1);
            se[q & 1] = ptx::f2_add(se[q & 1], ptx::f2_pack(p0, p1));
            sr[(q & 1) * 2] = ptx::add_bf16_lo(sr[(q & 1) * 2], pk[q]);
            sr[(q & 1) * 2 + 1] = ptx::add_bf16_hi(sr[(q & 1) * 2 + 1], pk[q]);
          }
          float e0, e1;
          ptx::f2_unpack(ptx::f2_add(se[0], se[1]), e0, e1);
          l += e0 + e1;
          l_round += (sr[0] + sr[1]) + (sr[2] + sr[3]);
          if (!(ok = wait_warp(bar(Lay::kPFree + buf), ((g >> 1) & 1) ^ 1, ctl))) break;
          ptx::tc_fence_after();
          ptx::tmem_st_x32(t_p, pk);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kPFull + buf));
      }
      if (!ok) break;
      // hand the row's statistics to the epilogue warps
      if (!(ok = wait_warp(bar(Lay::kStEmpty), (st_cnt & 1) ^ 1, ctl))) break;
      ++st_cnt;
      if (h == 0) stats[r] = m_used;
      stats[(1 + 2 * h) * kBlockM + r] = l;
      stats[(2 + 2 * h) * kBlockM + r] = l_round;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(Lay::kStFull));
    }
  } else if (warp < kSoftmaxWarps + 4) {
    // ------------------------------------------------------------ epilogue
    ptx::regs_decrease<kRegsEpilogue>();
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t t_o = tmem + (static_cast<uint32_t>(wq * 32) << 16) + Lay::kTmemO;
    uint32_t st_cnt = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int4 uw = next_unit_warp(k, ok);
      if (uw.y < 0) break;
      const UnitInfo ui = decode_unit(uw, causal);
      if (!(ok = wait_warp(bar(Lay::kStFull), st_cnt & 1, ctl))) break;
      ++st_cnt;
      const float lse2 = stats[r] + __log2f(stats[kBlockM + r] + stats[3 * kBlockM + r]);
      const float inv_l = 1.f / (stats[2 * kBlockM + r] + stats[4 * kBlockM + r]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(Lay::kStEmpty));
      if (!(ok = wait_warp(bar(Lay::kOUnit), k & 1, ctl))) break;
      ptx::tc_fence_after();
      const int row_doc = ui.qb * kBlockM + r;
      const bool row_ok = row_doc < ui.doc_len;
      const long long token = static_cast<long long>(ui.doc_start) + row_doc;
      uint4* orow =
          reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + (token * H + ui.head) * D);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        ptx::tmem_ld_x32(t_o + cc * 32, o);
        if (cc == D / 32 - 1) {
          // O is in registers: the tensor core may overwrite it now.
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bar(Lay::kOEmpty));
        }
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          w[q] = ptx::pack_bf16x2(__uint_as_float(o[2 * q]) * inv_l,
                                  __uint_as_float(o[2 * q + 1]) * inv_l);
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
  } else {
    // One setmaxnreg for the whole warpgroup (warps 12..15), as required.
    ptx::regs_decrease<kRegsOther>();
    if (warp == kWarpTma) {
      // ---------------------------------------------------------- producer
      // Lane 0 issues the copies; for MXFP8 every lane stages scale words.
      const int n_units = p.ws_header[kWsCountOffset / 4] * H;
      int* counter = const_cast<int*>(p.ws_header) + kWsUnitCounterOffset / 4;
      uint32_t q_it = 0, kv_it = 0;
      bool ok = true;
      // One tile into the next ring slot: kind 0 = K (rows start at row0),
      // kind 1 = V.
      auto load_kv = [&](const UnitInfo& ui, int j, int kind) -> bool {
        const uint32_t s = kv_it % Lay::kStages;
        if (!wait_warp(bar(Lay::kKVEmpty + s), ((kv_it / Lay::kStages) & 1) ^ 1, ctl)) return false;
        const uint32_t slot = sbase + Lay::kRingOff + s * Lay::kSlotBytes;
        const int row0 = ui.doc_start + kBlockN * j;
        if (kFp8 && kind == 0) {
          // Scale blocks of the K tile, one per scale word w of a row: lane
          // m0 writes keys m0 + 32 c, c = 0..3, as 16 bytes at offset
          // 512 w + 16 m0 (the layout tcgen05.cp replicates).
#pragma unroll
          for (int w = 0; w < Lay::kSfWords; ++w) {
            uint32_t wv[4];
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
              const int tok = row0 + lane + 32 * cq;
              wv[cq] = tok < p.total_tokens
                           ? p.k_scales[(static_cast<long long>(tok) * H + ui.head) * Lay::kSfWords + w]
                           : 0u;
            }
            *reinterpret_cast<uint4*>(smem + Lay::kRingOff + s * Lay::kSlotBytes + Lay::kKBytes +
                                      512 * w + 16 * lane) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          const int chunks = kind == 0 ? Lay::kQKChunks : Lay::kVChunks;
          const int bytes = kind == 0 ? Lay::kKBytes : Lay::kVBytes;
          ptx::mbar_arrive_expect_tx(bar(Lay::kKVFull + s), bytes);
          for (int cq = 0; cq < chunks; ++cq)
            ptx::tma_load_3d(slot + cq * (kind == 0 ? Lay::kQKChunkBytes : Lay::kChunkBytes),
                             kind == 0 ? static_cast<const void*>(&tm_k)
                                       : static_cast<const void*>(&tm_v),
                             bar(Lay::kKVFull + s), kind == 0 ? cq * Lay::kQKRowBytes / (kFp8 ? 1 : 2) : cq * 64,
                             ui.head, row0);
        }
        __syncwarp();
        ++kv_it;
        return true;
      };
      for (uint32_t k = 0; ok; ++k) {
        // Claim the next unit: the first one statically, the rest from the
        // shared counter, so each CTA takes the heaviest unit left whenever it
        // runs out of work (the list is sorted by cost).
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
        const UnitInfo ui = decode_unit(uw, causal);
        if (!(ok = wait_warp(bar(Lay::kQEmpty), (q_it & 1) ^ 1, ctl))) break;
        const int qrow0 = ui.doc_start + kBlockM * ui.qb;
        if constexpr (kFp8) {
#pragma unroll
          for (int w = 0; w < Lay::kSfWords; ++w) {
            uint32_t wv[4];
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
              const int tok = qrow0 + lane + 32 * cq;
              wv[cq] = tok < p.total_tokens
                           ? p.q_scales[(static_cast<long long>(tok) * H + ui.head) * Lay::kSfWords + w]
                           : 0u;
            }
            *reinterpret_cast<uint4*>(smem + Lay::kSfaOff + 512 * w + 16 * lane) =
                make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(bar(Lay::kQFull), Lay::kQBytes);
          for (int cq = 0; cq < Lay::kQKChunks; ++cq)
            ptx::tma_load_3d(sbase + Lay::kQOff + cq * Lay::kQKChunkBytes, &tm_q, bar(Lay::kQFull),
                             cq * Lay::kQKRowBytes / (kFp8 ? 1 : 2), ui.head, qrow0);
        }
        __syncwarp();
        ++q_it;
        // ring order = consumption order: K_0, K_1, then per step V_j and
        // K_{j+2}
        if (!(ok = load_kv(ui, 0, 0))) break;
        if (ui.n > 1 && !(ok = load_kv(ui, 1, 0))) break;
        for (int j = 0; ok && j < ui.n; ++j) {
          if (!(ok = load_kv(ui, j, 1))) break;
          if (j + 2 < ui.n && !(ok = load_kv(ui, j + 2, 0))) break;
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
      // Descriptors are precomputed 32-bit halves (advancing along K only adds
      // to the low half); per-buffer state is selected, never indexed.
      constexpr uint32_t kIdescS = ptx::idesc_bf16(kBlockM, kBlockN, 0);
      constexpr uint32_t kIdescO = ptx::idesc_bf16(kBlockM, D, 1);
      constexpr uint32_t kDescHi = ptx::sdesc_hi_sw128(1024);
      // NVFP4 Q and K rows are 64 bytes: 64-byte swizzle, 8-row groups 512 B apart
      constexpr uint32_t kQkDescHi = kNv4 ? ptx::sdesc_hi_sw64(512) : kDescHi;
      const uint32_t q_lo = ptx::sdesc_lo(sbase + Lay::kQOff, 16);
      const uint32_t ring_lo = ptx::sdesc_lo(sbase + Lay::kRingOff, 16);
      const uint32_t v_lbo = static_cast<uint32_t>(Lay::kChunkBytes - 16) >> 4 << 16;
      uint32_t q_ph = 0, oe_cnt = 0, g = 0;
      uint32_t cur = 0, cur_ph = 0;    // ring cursor (stage, phase)
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const uint32_t uslot = k % kUnitSlots;
        if (!(ok = wait_one(bar(Lay::kUnitFull + uslot), (k / kUnitSlots) & 1, ctl))) break;
        const int4 uw = unit_ring[uslot];
        ptx::mbar_arrive(bar(Lay::kUnitEmpty + uslot));
        if (uw.y < 0) break;
        const UnitInfo ui = decode_unit(uw, causal);
        const int n = ui.n;
        if (!(ok = wait_one(bar(Lay::kQFull), q_ph, ctl))) break;
        q_ph ^= 1;
        ptx::tc_fence_after();
        if constexpr (kFp8) {
#pragma unroll
          for (int w = 0; w < Lay::kSfWords; ++w)
            tmem_cp_32x128b_x4(tmem + Lay::kTmemSfa + 4 * w,
                               sf_copy_desc(sbase + Lay::kSfaOff + 512 * w));
        }
        // S for global step gs from the K tile in ring stage st.  It
        // overwrites P_{gs-2}, so it is issued after P_{gs-2} V_{gs-2} (the
        // tensor pipe keeps issue order).
        auto score = [&](uint32_t gs, uint32_t st) -> bool {
          const uint32_t buf = gs & 1;
          const uint32_t b_lo = ring_lo + st * (Lay::kSlotBytes >> 4);
          if constexpr (kNv4) {
            const uint32_t sfb = tmem + Lay::kTmemSfb + 4 * Lay::kSfWords * buf;
#pragma unroll
            for (int w = 0; w < Lay::kSfWords; ++w)
              tmem_cp_32x128b_x4(sfb + 4 * w,
                                 sf_copy_desc(sbase + Lay::kRingOff + st * Lay::kSlotBytes +
                                              Lay::kKBytes + 512 * w));
            // two K = 64 products (32 bytes of packed E2M1 each) per tile
#pragma unroll
            for (int kk = 0; kk < D / 64; ++kk) {
              const uint32_t off = (kk * 32) >> 4;
              mma_nvf4_ss(tmem + buf * 128, ptx::sdesc_join(q_lo + off, kQkDescHi),
                          ptx::sdesc_join(b_lo + off, kQkDescHi), idesc_nvf4(),
                          tmem + Lay::kTmemSfa + 4 * kk, sfb + 4 * kk, kk > 0 ? 1u : 0u);
            }
          } else if constexpr (kFp8) {
            const uint32_t sfb = tmem + Lay::kTmemSfb + 4 * buf;
            tmem_cp_32x128b_x4(sfb, sf_copy_desc(sbase + Lay::kRingOff + st * Lay::kSlotBytes +
                                                 Lay::kKBytes));
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
              const uint32_t off = (kk * 32) >> 4;
              mma_mxf8_ss(tmem + buf * 128, ptx::sdesc_join(q_lo + off, kDescHi),
                          ptx::sdesc_join(b_lo + off, kDescHi), idesc_mxf8(kk),
                          (static_cast<uint32_t>(kk) << 30) | (tmem + Lay::kTmemSfa),
                          (static_cast<uint32_t>(kk) << 30) | sfb, kk > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * Lay::kChunkBytes + (kk & 3) * 32) >> 4;
              ptx::mma_f16_ss(tmem + buf * 128, ptx::sdesc_join(q_lo + off, kDescHi),
                              ptx::sdesc_join(b_lo + off, kDescHi), kIdescS, kk > 0 ? 1u : 0u);
            }
          }
          ptx::mma_commit(bar(Lay::kSFull + buf));
          ptx::mma_commit(bar(Lay::kKVEmpty + st));
          return true;
        };
        // Next ring tile (in load order); false if the wait gave up.
        auto take = [&](uint32_t& st) -> bool {
          st = cur;
          const bool r2 = wait_one(bar(Lay::kKVFull + cur), cur_ph, ctl);
          if (++cur == static_cast<uint32_t>(Lay::kStages)) {
            cur = 0;
            cur_ph ^= 1;
          }
          return r2;
        };
        // O += P_j V_j with P_j in TMEM over the scores: keys 64 h + k of
        // half h at column 64 h + k / 2 of the buffer
        auto pv = [&](int j, uint32_t st_v, uint32_t buf) {
          const uint32_t b_lo = ring_lo + st_v * (Lay::kSlotBytes >> 4) + v_lbo;
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk) {
            const uint32_t a_col = buf * 128 + (kk >> 2) * kHalfKeys + (kk & 3) * 8;
            ptx::mma_f16_ts(tmem + Lay::kTmemO, tmem + a_col,
                            ptx::sdesc_join(b_lo + kk * (2048 >> 4), kDescHi), kIdescO,
                            (j == 0 && kk == 0) ? 0u : 1u);
          }
          ptx::mma_commit(bar(Lay::kKVEmpty + st_v));
          ptx::mma_commit(bar(Lay::kPFree + buf));
          if (j == n - 1) ptx::mma_commit(bar(Lay::kOUnit));
        };
        uint32_t st_k, st_v;
        if (!(ok = take(st_k)) || !(ok = score(g, st_k))) break;
        if (n > 1) {
          if (!(ok = take(st_k)) || !(ok = score(g + 1, st_k))) break;
        }
        if (n <= 2) ptx::mma_commit(bar(Lay::kQEmpty));
        for (int j = 0; j < n; ++j) {
          const uint32_t gs = g + j;
          const uint32_t buf = gs & 1;
          if (!(ok = take(st_v))) break;
          if (!(ok = wait_one(bar(Lay::kPFull + buf), (gs >> 1) & 1, ctl))) break;
          if (j == 0 && !(ok = wait_one(bar(Lay::kOEmpty), (oe_cnt++ & 1) ^ 1, ctl))) break;
          ptx::tc_fence_after();
          pv(j, st_v, buf);
          // S_{j+2} overwrites P_j, so it follows P_j V_j
          if (j + 2 < n) {
            if (!(ok = take(st_k)) || !(ok = score(gs + 2, st_k))) break;
            if (j + 2 == n - 1) ptx::mma_commit(bar(Lay::kQEmpty));
          }
        }
        if (!ok) break;
        g += n;
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

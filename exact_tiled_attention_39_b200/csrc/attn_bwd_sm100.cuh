// Exact attention backward for sm_100a, bf16 (head dim 64 or 128): dQ, dK
// and dV from Q, K, V, the forward's output O and log-sum-exp, and dO.
//
// The gradients are the derivatives of the forward definition ("FlashAttention
// và IO" (aihero.vn), section "Ma trận trung gian là một khoản chi phí":
// S = scale Q K^T, P = row-softmax(S), O = P V), per document and head:
//
//   P   = exp(scale S - lse)            recomputed tile by tile from the lse
//                                       the forward saved, never stored
//   dV  = P^T dO
//   dP  = dO V^T
//   D_i = dO_i . O_i                    (= sum_j P_ij dP_ij)
//   dS  = P * (dP - D)                  (elementwise, D broadcast along rows)
//   dQ  = scale dS K,   dK = scale dS^T Q
//
// The pages measure forward and backward together (FLAMIA: "Blackwell
// Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin Flash
// Mikro-Ölçeklemeli Dikkat Mekanizması", section "Performans Sonuçları") and
// print no backward formulas; the tiling keeps the forward's rule that no
// score or probability tile reaches device memory ("Tiling giữ công việc ở
// gần nơi tính").
//
// A work unit is one 128-key tile K_j, V_j of one document and head.  The
// CTA keeps dK_j and dV_j in TMEM while it walks the query tiles that see
// K_j (causal: from the diagonal tile on).  dQ_i gets one partial product
// per (i, j); it is added in fp32 to a device accumulator by TMA tensor
// reductions (staged in shared memory, 32 rows x 32 columns per copy), and a
// last small kernel scales and rounds it.
//
// Orientation: TMEM lane = key.  S^T = K_j Q_i^T and dP^T = V_j dO_i^T give
// each thread one key row of 128 query columns; P^T and dS^T go back over
// them as bf16 and feed dV += P^T dO_i and dK += dS^T Q_i directly from
// TMEM.  dQ_i = dS K_j reads dS from shared memory, stored MN-major (a key
// row of dS^T is a column of dS).
//
//   warps 0..7    compute, two warpgroups on the same key rows: warpgroup g
//                 takes query columns [64 g, 64 g + 64).  P^T from S^T, lse
//                 and the masks; dS^T from dP^T and D.  Each half writes its
//                 bf16 values over the first 32 columns of its own 64, so
//                 neither overwrites what the other has still to read.
//   warps 8..11   dQ_i read-out (176 registers): TMEM -> registers -> shared
//                 memory (the ring stage of Q_i and dO_i, free once dK_i and
//                 dV_i have read them; the producer refills it only after
//                 these reductions have read it) -> TMA reduce-add into the
//                 accumulator; at the end of a unit the dK_j, dV_j epilogue.
//   warp 12       producer (80 registers): claims units; TMA loads of K_j,
//                 V_j and of Q_i, dO_i into a two-stage ring, with the tile's
//                 lse and D rows.
//   warp 13       MMA issuer (one thread).
//   warps 14..15  idle.
//
// TMEM (512 columns): S^T / P^T at 0; dP^T / dS^T at 128, where dQ_i lands
// once dK's product has read dS^T (the tensor pipe runs products in issue
// order); dV at 256, dK at 256 + D.  The bf16 P^T and dS^T of query columns
// [64 g, 64 g + 64) sit in TMEM columns [64 g, 64 g + 32) of their block.
//
// A 128-row query tile may run past its document's end into the next
// document.  Those rows have P = 0, hence dS = 0 and a dQ_i row of exact
// zeros, so the reduction copies cover whole 32-row boxes: they add +-0 to
// the next document's rows (rows past the tensor's end are clipped by TMA).
#pragma once
#include <cuda.h>

#include <cstdint>

#include "attn_fwd_sm100.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace attn {

struct BwdParams {
  const float* lse;          // fp32 [H, T], natural log (the forward's)
  const float* delta;        // fp32 [H, T]: D = rowsum(dO * O)
  float* dq_acc;             // fp32 [T, H, D]
  void* dk;                  // bf16 [T, H, D]
  void* dv;                  // bf16 [T, H, D]
  const int32_t* ws_header;  // error word, work-list length, unit counter
  const int4* work;          // work list (one query-tile entry per key tile, see decode)
  int32_t* err;
  int total_tokens;
  int num_heads;
  int head_groups;
  int causal;
  float scale;               // softmax scale: dK = scale dS^T Q
  float scale_log2;          // scale * log2(e)
  unsigned long long timeout_ns;
};

constexpr int kBwdThreads = 512;
constexpr int kBwdComputeWarps = 8;
constexpr int kBwdUnitConsumers = 1 + kBwdComputeWarps + 4;   // MMA thread, compute, read-out warps
// Registers per thread at launch: 65536 / 512 = 128.  The compute
// warpgroups keep 128; the read-out warpgroup takes what the producer / MMA
// warpgroup gives up.
constexpr uint32_t kBwdRegsCompute = 128, kBwdRegsReadout = 176, kBwdRegsOther = 80;
static_assert(2 * kBwdRegsCompute + kBwdRegsReadout + kBwdRegsOther == 4 * 128,
              "register split must use exactly the registers the CTA is launched with");

template <int D>
struct BwdLayout {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static constexpr int kChunks = D / 64;                      // 128-byte chunks per row
  static constexpr int kChunkBytes = 128 * 128;               // 128 rows x 128 bytes
  static constexpr int kTileBytes = kChunks * kChunkBytes;    // one K, V, Q or dO tile
  static constexpr int kStages = 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;          // Q_i, then dO_i
  static constexpr int kRingOff = 2 * kTileBytes;
  // dS (bf16, 128 queries x 128 keys), MN-major: row = key, 64 queries per
  // 128-byte chunk row, two chunks of 16 KB.
  static constexpr int kDsOff = kRingOff + kStages * kStageBytes;
  // dQ_i staging, in ring stage i's Q_i (and, at head dim 64, dO_i) once
  // dK_i and dV_i have read them: per read-out warp two 4 KB buffers of 32
  // rows x 32 fp32 in the 128-byte swizzle.
  static constexpr int kStageBufBytes = 32 * 128;
  static constexpr int kDsBytes = 2 * kChunkBytes;
  static constexpr int kVecOff = kDsOff + kDsBytes;           // float [stage][lse2, D][128]
  static constexpr int kBarOff = kVecOff + kStages * 2 * 128 * 4;
  static constexpr int kKVFull = 0, kKVEmpty = 1;
  static constexpr int kQFull = 2;                            // + stage
  static constexpr int kQEmpty = kQFull + kStages;            // + stage
  static constexpr int kSFull = kQEmpty + kStages;
  static constexpr int kPFull = kSFull + 1;
  static constexpr int kDPFull = kPFull + 1;
  static constexpr int kDSFull = kDPFull + 1;
  static constexpr int kDQFull = kDSFull + 1;
  static constexpr int kDQEmpty = kDQFull + 1;
  static constexpr int kDKVFull = kDQEmpty + 1;
  static constexpr int kDKVEmpty = kDKVFull + 1;
  static constexpr int kDrain = kDKVEmpty + 1;
  static constexpr int kUnitFull = kDrain + 1;                // + slot
  static constexpr int kUnitEmpty = kUnitFull + kUnitSlots;   // + slot
  static constexpr int kNumBars = kUnitEmpty + kUnitSlots;
  static constexpr int kMiscOff = (kBarOff + kNumBars * 8 + 15) / 16 * 16;   // tmem base, abort
  static constexpr int kUnitOff = kMiscOff + 16;              // int4 [kUnitSlots]
  static constexpr int kBytes = kUnitOff + 16 * kUnitSlots;
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory per CTA");
  static_assert(4 * 2 * kStageBufBytes <= kStageBytes, "dQ staging must fit a ring stage");
  static constexpr uint32_t kTmemS = 0;
  static constexpr uint32_t kTmemDP = 128;
  static constexpr uint32_t kTmemDV = 256;
  static constexpr uint32_t kTmemDK = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
};

// TMA tensor reduce-add of a shared-memory box into global memory (element
// type and box from the tensor map), tracked by the issuing thread's bulk
// async-group.
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, uint32_t src, int32_t c0,
                                                  int32_t c1, int32_t c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// D = rowsum(dO * O) per (token, head) into [H, T], and the dQ accumulator
// row cleared.  d / 8 threads per row, 8 elements each.
__global__ void __launch_bounds__(256)
attn_bwd_prep_kernel(const uint4* __restrict__ out, const uint4* __restrict__ dout,
                     float* __restrict__ delta, float4* __restrict__ dq_acc, long long rows,
                     int head_dim, int num_heads, int total_tokens) {
  ptx::grid_launch_dependents();
  const int g = head_dim / 8;                     // threads per row (8 or 16)
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = tid / g;
  const int part = static_cast<int>(tid % g);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = out[row * g + part];
    const uint4 b = dout[row * g + part];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(aw[i] << 16), __uint_as_float(bw[i] << 16), acc);
      acc = fmaf(__uint_as_float(aw[i] & 0xffff0000u), __uint_as_float(bw[i] & 0xffff0000u), acc);
    }
    dq_acc[(row * g + part) * 2] = make_float4(0.f, 0.f, 0.f, 0.f);
    dq_acc[(row * g + part) * 2 + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // groups of g lanes are aligned inside the warp (g divides 32)
  for (int o = g / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (row < rows && part == 0) {
    const long long t = row / num_heads;
    const int h = static_cast<int>(row % num_heads);
    delta[static_cast<long long>(h) * total_tokens + t] = acc;
  }
}

// dQ = scale * accumulator, rounded to bf16, four elements per thread;
// nothing is written if the call recorded an error (dq is then left as it
// was, like the forward's outputs).
__global__ void __launch_bounds__(256)
attn_bwd_dq_kernel(const int32_t* __restrict__ err, const float4* __restrict__ acc,
                   uint2* __restrict__ dq, long long n4, float scale) {
  if (*err != 0) return;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 a = acc[i];
  dq[i] = make_uint2(ptx::pack_bf16x2(a.x * scale, a.y * scale),
                     ptx::pack_bf16x2(a.z * scale, a.w * scale));
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using Lay = BwdLayout<D>;
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
  float* vecs = reinterpret_cast<float*>(smem + Lay::kVecOff);
  int4* unit_ring = reinterpret_cast<int4*>(smem + Lay::kUnitOff);

  constexpr int kWarpTma = 12, kWarpMma = 13;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(Lay::kKVFull), 1);
    ptx::mbar_init(bar(Lay::kKVEmpty), 1);
    for (int s = 0; s < Lay::kStages; ++s) {
      ptx::mbar_init(bar(Lay::kQFull + s), 1);
      // MMA (dK_i's product done) + compute warps (lse, D read) + read-out
      // warps (dQ_i's staging read by its reductions)
      ptx::mbar_init(bar(Lay::kQEmpty + s), 1 + kBwdComputeWarps + 4);
    }
    ptx::mbar_init(bar(Lay::kSFull), 1);
    ptx::mbar_init(bar(Lay::kPFull), kBwdComputeWarps);
    ptx::mbar_init(bar(Lay::kDPFull), 1);
    ptx::mbar_init(bar(Lay::kDSFull), kBwdComputeWarps);
    ptx::mbar_init(bar(Lay::kDQFull), 1);
    ptx::mbar_init(bar(Lay::kDQEmpty), 4);
    ptx::mbar_init(bar(Lay::kDKVFull), 1);
    ptx::mbar_init(bar(Lay::kDKVEmpty), 4);
    ptx::mbar_init(bar(Lay::kDrain), 1);
    for (int i = 0; i < kUnitSlots; ++i) {
      ptx::mbar_init(bar(Lay::kUnitFull + i), 1);
      ptx::mbar_init(bar(Lay::kUnitEmpty + i), kBwdUnitConsumers);
    }
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == kWarpTma && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_do);
    ptx::prefetch_tmap(&tm_dq);
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_holder), Lay::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // The work list, D and the cleared accumulator come from the kernels
  // launched just before.
  ptx::grid_dependency_wait();

  const WaitCtl ctl{abort_flag, p.err, p.timeout_ns};
  const int H = p.num_heads;
  const int causal = p.causal;
  auto next_unit_warp = [&](uint32_t k, bool& ok) -> int4 {
    const uint32_t slot = k % kUnitSlots;
    if (!(ok = wait_warp(bar(Lay::kUnitFull + slot), (k / kUnitSlots) & 1, ctl)))
      return make_int4(0, -1, 0, 0);
    const int4 w = unit_ring[slot];
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar(Lay::kUnitEmpty + slot));
    return w;
  };
  // Ring entry (doc_start, doc_len, key tile kb, head): the query tiles that
  // see key tile kb are [qb0, n_tiles).
  auto query_tiles = [&](int4 uw, int& qb0) -> int {
    const int n_tiles = (uw.y + kBlockM - 1) / kBlockM;
    qb0 = causal ? uw.z : 0;
    return n_tiles - qb0;
  };

  if (warp < 8) {
    // ------------------------------------------------------------ compute
    const int g = warp >> 2;                       // query-column half
    const int r = (warp & 3) * 32 + lane;          // key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + Lay::kTmemS + 64 * g;
    const uint32_t t_dp = tmem + lane_off + Lay::kTmemDP + 64 * g;
    const float c = p.scale_log2;
    uint8_t* const ds_row = smem + Lay::kDsOff + g * Lay::kChunkBytes + r * 128;
    uint32_t q_cnt = 0;                            // query steps so far (all units)
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int4 uw = next_unit_warp(k, ok);
      if (uw.y < 0) break;
      int qb0;
      const int n = query_tiles(uw, qb0);
      const int kb = uw.z;
      const bool key_ok = kb * kBlockN + r < uw.y;
      for (int ii = 0; ii < n; ++ii, ++q_cnt) {
        const int qb = qb0 + ii;
        const uint32_t s = q_cnt % Lay::kStages;
        if (!(ok = wait_warp(bar(Lay::kQFull + s), (q_cnt / Lay::kStages) & 1, ctl))) break;
        const float* lse2 = vecs + (s * 2) * 128 + 64 * g;
        const float* dd = vecs + (s * 2 + 1) * 128 + 64 * g;
        // visible query columns q (relative to this half): 64 g + q < q_end,
        // and 64 g + q >= r on the diagonal tile
        const int q_end = (key_ok ? min(uw.y - qb * kBlockM, kBlockM) : 0) - 64 * g;
        const int q_begin = ((causal && qb == kb) ? r : 0) - 64 * g;
        if (!(ok = wait_warp(bar(Lay::kSFull), q_cnt & 1, ctl))) break;
        ptx::tc_fence_after();
        uint32_t pk[32];   // this half of the P^T row as bf16 pairs
        {
          uint32_t sa[64];
          ptx::tmem_ld_x64(t_s, sa);
#pragma unroll
          for (int a = 0; a < 32; ++a) {
            const int q = 2 * a;
            const float2 l2 = *reinterpret_cast<const float2*>(lse2 + q);
            float p0 = ptx::ex2_approx(__uint_as_float(sa[2 * a]) * c - l2.x);
            float p1 = ptx::ex2_approx(__uint_as_float(sa[2 * a + 1]) * c - l2.y);
            if (q < q_begin || q >= q_end) p0 = 0.f;
            if (q + 1 < q_begin || q + 1 >= q_end) p1 = 0.f;
            pk[a] = ptx::pack_bf16x2(p0, p1);
          }
        }
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t w[16];
#pragma unroll
          for (int a = 0; a < 16; ++a) w[a] = pk[16 * ch + a];
          ptx::tmem_st_x16(t_s + 16 * ch, w);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kPFull));
        // dS^T = P^T * (dP^T - D), 32 query columns at a time, written over
        // this half's dP^T in TMEM and as chunk g of the key's row of the
        // MN-major dS tile in shared memory
        if (!(ok = wait_warp(bar(Lay::kDPFull), q_cnt & 1, ctl))) break;
        ptx::tc_fence_after();
        // the dS buffer is free: dP^T of this step was issued after the
        // previous dQ (the product that read dS) had left TMEM
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t dp[32];
          ptx::tmem_ld_x32(t_dp + 32 * ch, dp);
          uint32_t ds[16];
#pragma unroll
          for (int a = 0; a < 16; ++a) {
            const int q = 32 * ch + 2 * a;
            const float2 d2 = *reinterpret_cast<const float2*>(dd + q);
            const uint32_t pw = pk[16 * ch + a];
            const float p0 = __uint_as_float(pw << 16), p1 = __uint_as_float(pw & 0xffff0000u);
            ds[a] = ptx::pack_bf16x2(p0 * (__uint_as_float(dp[2 * a]) - d2.x),
                                     p1 * (__uint_as_float(dp[2 * a + 1]) - d2.y));
          }
          // columns 16 ch .. 16 ch + 15 of this half: dP^T values already read
          ptx::tmem_st_x16(t_dp + 16 * ch, ds);
          // queries 32 ch .. 32 ch + 31 of the half: 16-byte units
          // 4 ch .. 4 ch + 3 of the chunk row, swizzled by r % 8
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const int u = 4 * ch + uu;
            *reinterpret_cast<uint4*>(ds_row + ((u ^ (r & 7)) << 4)) =
                make_uint4(ds[4 * uu], ds[4 * uu + 1], ds[4 * uu + 2], ds[4 * uu + 3]);
          }
        }
        ptx::tmem_wait_st();
        fence_proxy_async_smem();   // the tensor core reads dS through the async proxy
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(bar(Lay::kDSFull));
          ptx::mbar_arrive(bar(Lay::kQEmpty + s));   // done with this stage's lse and D
        }
      }
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ dQ read-out, dK / dV epilogue
    ptx::regs_increase<kBwdRegsReadout>();
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t warp_stage_off = wq * 2 * Lay::kStageBufBytes;
    uint32_t q_cnt = 0, u_cnt = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int4 uw = next_unit_warp(k, ok);
      if (uw.y < 0) break;
      int qb0;
      const int n = query_tiles(uw, qb0);
      for (int ii = 0; ii < n; ++ii, ++q_cnt) {
        const int qb = qb0 + ii;
        if (!(ok = wait_warp(bar(Lay::kDQFull), q_cnt & 1, ctl))) break;
        ptx::tc_fence_after();
        uint32_t acc[D];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t t[32];
          ptx::tmem_ld_x32(tmem + lane_off + Lay::kTmemDP + 32 * cc, t);
#pragma unroll
          for (int a = 0; a < 32; ++a) acc[32 * cc + a] = t[a];
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kDQEmpty));
        // 32 columns per copy: this warp's 32 rows in a 4 KB buffer (row =
        // lane, 16-byte unit u at u ^ (lane % 8)), two buffers in turn
        const int qrow0 = uw.x + qb * kBlockM + 32 * wq;
        // (a warp whose 32 rows all lie past the document end has only zeros)
        const bool any_row = qb * kBlockM + 32 * wq < uw.y;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          if (!any_row) break;
          if (c >= 2) {
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
          }
          const uint32_t buf = sbase + Lay::kRingOff + (q_cnt % Lay::kStages) * Lay::kStageBytes +
                               warp_stage_off + (c & 1) * Lay::kStageBufBytes;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t addr = buf + lane * 128 + ((u ^ (lane & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(acc[32 * c + 4 * u]), "r"(acc[32 * c + 4 * u + 1]),
                         "r"(acc[32 * c + 4 * u + 2]), "r"(acc[32 * c + 4 * u + 3])
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&tm_dq, buf, 32 * c, uw.w, qrow0);
            bulk_commit_group();
          }
        }
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        // the stage's staging has been read: the producer may refill it
        if (lane == 0) ptx::mbar_arrive(bar(Lay::kQEmpty + q_cnt % Lay::kStages));
      }
      if (!ok) break;
      // dK_j, dV_j of the unit (key rows)
      if (!(ok = wait_warp(bar(Lay::kDKVFull), u_cnt & 1, ctl))) break;
      ptx::tc_fence_after();
      ++u_cnt;
      const int key = uw.z * kBlockN + r;
      const bool row_ok = key < uw.y;
      const long long off = (static_cast<long long>(uw.x + key) * H + uw.w) * D;
      uint4* dv_row = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dv) + off);
      uint4* dk_row = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dk) + off);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint32_t col = m == 0 ? Lay::kTmemDV : Lay::kTmemDK;
        const float f = m == 0 ? 1.f : p.scale;
        uint4* dst = m == 0 ? dv_row : dk_row;
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t o[16];
          ptx::tmem_ld_x16(tmem + lane_off + col + 16 * cc, o);
          if (m == 1 && cc == D / 16 - 1) {
            // dK and dV are in registers: the next unit may overwrite them.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(Lay::kDKVEmpty));
          }
          uint32_t w[8];
#pragma unroll
          for (int a = 0; a < 8; ++a)
            w[a] = ptx::pack_bf16x2(__uint_as_float(o[2 * a]) * f, __uint_as_float(o[2 * a + 1]) * f);
          if (row_ok) {
            dst[2 * cc] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[2 * cc + 1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
      }
    }
  } else {
    ptx::regs_decrease<kBwdRegsOther>();
  }
  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    const int n_units = p.ws_header[kWsCountOffset / 4] * H;
    int* counter = const_cast<int*>(p.ws_header) + kWsUnitCounterOffset / 4;
    const float kLog2e = 1.4426950408889634f;
    uint32_t q_it = 0, kv_it = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      int claim = 0;
      if (lane == 0)
        claim = k == 0 ? static_cast<int>(blockIdx.x)
                       : static_cast<int>(gridDim.x) + atomicAdd(counter, 1);
      claim = __shfl_sync(0xffffffffu, claim, 0);
      int4 uw = make_int4(0, -1, 0, 0);
      if (claim < n_units) {
        // Unit -> (entry, head) as in the forward: groups of heads one after
        // the other, inside a group entry major (heaviest first), head minor.
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
        // The list entry of query tile t of a document has the cost of key
        // tile n_tiles - 1 - t (causal: n_tiles - kb query tiles see key tile
        // kb), so the same heaviest-first list serves, read backwards.
        const int4 e = p.work[rem / gsize];
        const int n_tiles = (e.y + kBlockM - 1) / kBlockM;
        uw = make_int4(e.x, e.y, n_tiles - 1 - e.z, h0 + rem % gsize);
      }
      const uint32_t uslot = k % kUnitSlots;
      if (!(ok = wait_warp(bar(Lay::kUnitEmpty + uslot), ((k / kUnitSlots) & 1) ^ 1, ctl))) break;
      if (lane == 0) {
        unit_ring[uslot] = uw;
        ptx::mbar_arrive(bar(Lay::kUnitFull + uslot));
      }
      __syncwarp();
      if (uw.y < 0) break;
      // K_j, V_j (one buffer each: the previous unit's products must be done)
      if (!(ok = wait_warp(bar(Lay::kKVEmpty), (kv_it & 1) ^ 1, ctl))) break;
      const int krow0 = uw.x + uw.z * kBlockN;
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar(Lay::kKVFull), 2 * Lay::kTileBytes);
        for (int cq = 0; cq < Lay::kChunks; ++cq) {
          ptx::tma_load_3d(sbase + Lay::kKOff + cq * Lay::kChunkBytes, &tm_k, bar(Lay::kKVFull),
                           cq * 64, uw.w, krow0);
          ptx::tma_load_3d(sbase + Lay::kVOff + cq * Lay::kChunkBytes, &tm_v, bar(Lay::kKVFull),
                           cq * 64, uw.w, krow0);
        }
      }
      __syncwarp();
      ++kv_it;
      int qb0;
      const int n = query_tiles(uw, qb0);
      for (int ii = 0; ii < n; ++ii) {
        const int qb = qb0 + ii;
        const uint32_t s = q_it % Lay::kStages;
        // lse (in log2 units) and D of the tile's 128 query rows, read before
        // the stage is free so their latency overlaps the wait; rows past the
        // document end get 0 (their columns are masked)
        float lr[4], dr[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int row = qb * kBlockM + 4 * lane + a;
          const bool valid = row < uw.y;
          const long long idx = static_cast<long long>(uw.w) * p.total_tokens + uw.x + row;
          lr[a] = valid ? p.lse[idx] * kLog2e : 0.f;
          dr[a] = valid ? p.delta[idx] : 0.f;
        }
        if (!(ok = wait_warp(bar(Lay::kQEmpty + s), ((q_it / Lay::kStages) & 1) ^ 1, ctl))) break;
        *reinterpret_cast<float4*>(vecs + (s * 2) * 128 + 4 * lane) =
            make_float4(lr[0], lr[1], lr[2], lr[3]);
        *reinterpret_cast<float4*>(vecs + (s * 2 + 1) * 128 + 4 * lane) =
            make_float4(dr[0], dr[1], dr[2], dr[3]);
        __syncwarp();
        const uint32_t stage = sbase + Lay::kRingOff + s * Lay::kStageBytes;
        const int qrow0 = uw.x + qb * kBlockM;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(bar(Lay::kQFull + s), 2 * Lay::kTileBytes);
          for (int cq = 0; cq < Lay::kChunks; ++cq) {
            ptx::tma_load_3d(stage + cq * Lay::kChunkBytes, &tm_q, bar(Lay::kQFull + s), cq * 64,
                             uw.w, qrow0);
            ptx::tma_load_3d(stage + Lay::kTileBytes + cq * Lay::kChunkBytes, &tm_do,
                             bar(Lay::kQFull + s), cq * 64, uw.w, qrow0);
          }
        }
        __syncwarp();
        ++q_it;
      }
    }
    if (!ok && lane == 0) {
      // Let copies already issued land before the CTA can exit.
      WaitCtl drain = ctl;
      uint32_t zero = 0;
      drain.abort_flag = &zero;
      if (kv_it > 0) wait_one(bar(Lay::kKVFull), (kv_it - 1) & 1, drain);
      const uint32_t first = q_it > (uint32_t)Lay::kStages ? q_it - Lay::kStages : 0;
      for (uint32_t it = first; it < q_it; ++it)
        wait_one(bar(Lay::kQFull + it % Lay::kStages), (it / Lay::kStages) & 1, drain);
    }
  } else if (warp == kWarpMma && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdescT = ptx::idesc_bf16(128, 128, 0);            // S^T, dP^T
    constexpr uint32_t kIdescG = ptx::idesc_bf16(128, D, 1);              // dV, dK (A in TMEM)
    constexpr uint32_t kIdescQ = ptx::idesc_bf16(128, D, 1) | (1u << 15); // dQ: A MN-major too
    constexpr uint32_t kDescHi = ptx::sdesc_hi_sw128(1024);
    // MN-major operands: 64-element chunks 16 KB apart (leading byte offset)
    const uint32_t mn_lbo = static_cast<uint32_t>(Lay::kChunkBytes - 16) >> 4 << 16;
    const uint32_t k_lo = ptx::sdesc_lo(sbase + Lay::kKOff, 16);
    const uint32_t v_lo = ptx::sdesc_lo(sbase + Lay::kVOff, 16);
    const uint32_t ring_lo = ptx::sdesc_lo(sbase + Lay::kRingOff, 16);
    const uint32_t ds_lo = ptx::sdesc_lo(sbase + Lay::kDsOff, 16);
    uint32_t kv_ph = 0, q_cnt = 0, u_cnt = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const uint32_t uslot = k % kUnitSlots;
      if (!(ok = wait_one(bar(Lay::kUnitFull + uslot), (k / kUnitSlots) & 1, ctl))) break;
      const int4 uw = unit_ring[uslot];
      ptx::mbar_arrive(bar(Lay::kUnitEmpty + uslot));
      if (uw.y < 0) break;
      int qb0;
      const int n = query_tiles(uw, qb0);
      if (!(ok = wait_one(bar(Lay::kKVFull), kv_ph, ctl))) break;
      kv_ph ^= 1;
      ptx::tc_fence_after();
      for (int ii = 0; ii < n; ++ii, ++q_cnt) {
        const uint32_t s = q_cnt % Lay::kStages;
        if (!(ok = wait_one(bar(Lay::kQFull + s), (q_cnt / Lay::kStages) & 1, ctl))) break;
        ptx::tc_fence_after();
        const uint32_t q_lo = ring_lo + ((s * Lay::kStageBytes) >> 4);
        const uint32_t do_lo = q_lo + (Lay::kTileBytes >> 4);
        // S^T = K_j Q_i^T (P^T of the step before was read by its dV product,
        // issued earlier)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Lay::kChunkBytes + (kk & 3) * 32) >> 4;
          ptx::mma_f16_ss(tmem + Lay::kTmemS, ptx::sdesc_join(k_lo + off, kDescHi),
                          ptx::sdesc_join(q_lo + off, kDescHi), kIdescT, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(Lay::kSFull));
        // dP^T = V_j dO_i^T, once the previous dQ has left those columns
        if (q_cnt > 0 && !(ok = wait_one(bar(Lay::kDQEmpty), (q_cnt - 1) & 1, ctl))) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Lay::kChunkBytes + (kk & 3) * 32) >> 4;
          ptx::mma_f16_ss(tmem + Lay::kTmemDP, ptx::sdesc_join(v_lo + off, kDescHi),
                          ptx::sdesc_join(do_lo + off, kDescHi), kIdescT, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(Lay::kDPFull));
        // dV += P^T dO_i (the first product of a unit waits for the previous
        // unit's epilogue to have read dK and dV)
        if (!(ok = wait_one(bar(Lay::kPFull), q_cnt & 1, ctl))) break;
        if (ii == 0 && u_cnt > 0 && !(ok = wait_one(bar(Lay::kDKVEmpty), (u_cnt - 1) & 1, ctl)))
          break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlockM / 16; ++kk)
          ptx::mma_f16_ts(tmem + Lay::kTmemDV, tmem + Lay::kTmemS + kk * 8 + (kk >= 4 ? 32 : 0),
                          ptx::sdesc_join(do_lo + mn_lbo + kk * (2048 >> 4), kDescHi), kIdescG,
                          (ii > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q_i, then dQ_i = dS K_j over dS^T's columns
        if (!(ok = wait_one(bar(Lay::kDSFull), q_cnt & 1, ctl))) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlockM / 16; ++kk)
          ptx::mma_f16_ts(tmem + Lay::kTmemDK, tmem + Lay::kTmemDP + kk * 8 + (kk >= 4 ? 32 : 0),
                          ptx::sdesc_join(q_lo + mn_lbo + kk * (2048 >> 4), kDescHi), kIdescG,
                          (ii > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(bar(Lay::kQEmpty + s));   // Q_i and dO_i: last read by dK's product
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          ptx::mma_f16_ss(tmem + Lay::kTmemDP,
                          ptx::sdesc_join(ds_lo + mn_lbo + kk * (2048 >> 4), kDescHi),
                          ptx::sdesc_join(k_lo + mn_lbo + kk * (2048 >> 4), kDescHi), kIdescQ,
                          kk > 0 ? 1u : 0u);
        ptx::mma_commit(bar(Lay::kDQFull));
      }
      if (!ok) break;
      ptx::mma_commit(bar(Lay::kDKVFull));
      ptx::mma_commit(bar(Lay::kKVEmpty));
      ++u_cnt;
    }
    // Every product this thread issued must be complete before TMEM is freed.
    ptx::mma_commit(bar(Lay::kDrain));
    WaitCtl drain = ctl;
    uint32_t zero = 0;
    drain.abort_flag = &zero;
    wait_one(bar(Lay::kDrain), 0, drain);
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

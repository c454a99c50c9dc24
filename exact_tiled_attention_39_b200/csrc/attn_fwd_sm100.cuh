// Pieces of the exact attention forward for sm_100a that the kernels share:
// the kernel parameters, the bounded mbarrier waits, and the block-scaled
// tcgen05 forms (instruction descriptors, the MXFP8 and NVFP4 score
// products, the tcgen05.cp copy of scale blocks into TMEM).  The kernel
// itself is attn_fwd_pair_sm100.cuh; the backward uses the waits.
//
// The method ("FlashAttention và IO" (aihero.vn), sections "Tiling giữ công
// việc ở gần nơi tính" and "Softmax qua nhiều khối cần thống kê chạy"):
// Q, K and V are cut into tiles held on chip; for each query row the kernel
// keeps the running maximum m, the normaliser l and the weighted sum u (the
// output accumulator O), multiplies the old part by exp(m - m_new) when a new
// key tile raises the maximum, and writes u / l and the log-sum-exp at the
// end.  Scores and probabilities never leave the SM.
//
// The block-scaled products follow "FLAMIA: Blackwell Üzerinde Hızlı ve
// Nedensel Olarak Güvenli Eğitim İçin Flash Mikro-Ölçeklemeli Dikkat
// Mekanizması" (section "FLAMIA Mimarisi ve Temel Tasarım İlkeleri"):
// low-precision products whose scales (one per token, head and 32 (MXFP8)
// or 16 (NVFP4) head-dim elements) run along the contraction and never span
// two tokens.
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
  const uint32_t* q_scales;  // scale words of Q: MXFP8 [T, H] (4 E8M0 bytes each),
                             // NVFP4 [T, H, 2] (4 UE4M3 bytes each)
  const uint32_t* k_scales;  // scale words of K, as q_scales
  int total_tokens;
  int num_heads;
  int head_groups;           // unit order: heads in this many groups (see common.cuh)
  int causal;
  float scale_log2;          // scale * log2(e)
  unsigned long long timeout_ns;
};

constexpr int kUnitSlots = 4;                // ring of claimed work units

// Operand format of the score product Q K^T: bf16, MXFP8 (E4M3 codes, one
// E8M0 scale per 32 elements) or NVFP4 (E2M1 codes two per byte, one
// unsigned E4M3 scale per 16 elements).
constexpr int kQkBf16 = 0, kQkMx8 = 1, kQkNv4 = 2;

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
// accumulate, unsigned E4M3 scales, one per 16 elements, M = 128, N = n,
// K = 64): the scale ids are 0, each instruction reads a whole 32-bit scale
// word per row.
__host__ __device__ constexpr uint32_t idesc_nvf4(int n = kBlockN) {
  return (1u << 7) | (1u << 10)               // A, B format: E2M1
         | (static_cast<uint32_t>(n >> 3) << 17)
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

}  // namespace attn

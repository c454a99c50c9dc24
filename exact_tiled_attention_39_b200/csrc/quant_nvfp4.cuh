// NVFP4 quantisation pre-pass for the mixed NVFP4 / FP8 path: bf16 -> E2M1
// element codes (two per byte, the lower-indexed element in the low nibble)
// and one unsigned E4M3 scale per 16 contiguous elements of a row.  For
// attention operands a row is one token of one head, so no scale spans two
// tokens, and there is no per-tensor scale (one computed over the whole
// tensor would make every token's codes depend on future tokens).
//
// FLAMIA ("FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli
// Eğitim İçin Flash Mikro-Ölçeklemeli Dikkat Mekanizması", section "FLAMIA
// Mimarisi ve Temel Tasarım İlkeleri") names the mixed NVFP4 / FP8 path
// beside MXFP8, with fused quantisation and scales that never carry
// information across a causal or document boundary.
//
// Scale rule: S = the smallest positive E4M3 value with amax <= 6 S (448
// past 6 * 448; 1 for a block of zeros).  The hardware's round-to-nearest
// E4M3 conversion of amax / 6 lands on S or a neighbour; the exact test
// 6 v >= amax (6 v is exact in fp32: v has a 4-bit significand) moves it to
// S.  Elements: the IEEE fp32 quotient x / S, converted by the hardware's
// round-to-nearest-even, saturating E2M1 conversion.
//
// HBM-bound: per 16-element block 32 bytes read; 8 bytes of codes and one
// scale byte and/or 32 bytes of exact dequantised bf16 written.
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

#include "quant_mxfp8.cuh"

namespace attn {

// Value of a positive E4M3 code (exact, through f16).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  float lo, hi;
  e4m3x2_to_f32(static_cast<uint16_t>(code & 0xFFu), lo, hi);
  return lo;
}

__device__ __forceinline__ uint32_t nvfp4_scale_code(float amax) {
  if (amax == 0.f) return 0x38u;                                   // 1.0
  uint32_t code = cvt_e4m3x2(__fdiv_rn(amax, 6.f), 0.f) & 0xFFu;   // saturates at 448
  if (code == 0u) code = 1u;                                       // below 2^-9: the smallest
  if (code < 0x7Eu && 6.f * e4m3_value(code) < amax) ++code;
  if (code > 1u && 6.f * e4m3_value(code - 1u) >= amax) --code;
  return code;
}

// Two fp32 -> one byte of E2M1 codes (lo in bits 0-3, hi in bits 4-7).
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// E2M1 code (4 bits) -> fp32 value.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  // 0, 0.5, 1, 1.5, 2, 3, 4, 6
  const float mag = m < 2u ? 0.5f * static_cast<float>(m)
                           : __uint_as_float((126u + (m >> 1)) << 23) * (1.f + 0.5f * (m & 1u));
  return (c & 8u) ? -mag : mag;
}

// One 16-element block b of a row-major bf16 tensor, given as its two
// 16-byte halves v0, v1: codes (8 bytes), scale byte and/or exact
// dequantised bf16 (32 bytes); any output may be null.
__device__ __forceinline__ void quantize_block_nvfp4_values(uint4 v0, uint4 v1,
                                                            uint2* __restrict__ codes,
                                                            uint8_t* __restrict__ scales,
                                                            uint4* __restrict__ deq, long long b) {
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float f[16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = bf16_lo(w[i]);
    f[2 * i + 1] = bf16_hi(w[i]);
    amax = fmaxf(amax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
  }
  const uint32_t scode = nvfp4_scale_code(amax);
  const float s = e4m3_value(scode);
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t byte = cvt_e2m1x2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
    packed[i >> 2] |= byte << (8 * (i & 3));
  }
  if (codes != nullptr) codes[b] = make_uint2(packed[0], packed[1]);
  if (scales != nullptr) scales[b] = static_cast<uint8_t>(scode);
  if (deq != nullptr) {
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte = packed[i >> 2] >> (8 * (i & 3));
      const float a = e2m1_value(byte & 15u) * s, c = e2m1_value((byte >> 4) & 15u) * s;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[i]) : "f"(c), "f"(a));
    }
    deq[2 * b] = make_uint4(o[0], o[1], o[2], o[3]);
    deq[2 * b + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

__device__ __forceinline__ void quantize_block_nvfp4(const uint4* __restrict__ x,
                                                     uint2* __restrict__ codes,
                                                     uint8_t* __restrict__ scales,
                                                     uint4* __restrict__ deq, long long b) {
  quantize_block_nvfp4_values(x[2 * b], x[2 * b + 1], codes, scales, deq, b);
}

// One thread per 16-element block; n_blocks = rows * cols / 16.
__global__ void __launch_bounds__(256)
quantize_nvfp4_kernel(const uint4* __restrict__ x, uint2* __restrict__ codes,
                      uint8_t* __restrict__ scales, uint4* __restrict__ deq, long long n_blocks) {
  const long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= n_blocks) return;
  quantize_block_nvfp4(x, codes, scales, deq, b);
}

// The pre-pass of the mixed path in one launch: blockIdx.y 0 and 1 take Q
// and K to NVFP4 (one thread per two consecutive 16-element blocks, both
// loaded before either is worked on), 2 takes V to MXFP8 (one thread per
// 32-element block, exact dequantised bf16 only): one thread per 32
// elements and 64 bytes in flight in every part.
struct MixedQuantJobs {
  const uint4* x[3];
  uint2* codes[2];        // packed E2M1 of Q, K (null: not written)
  uint8_t* scales[2];     // UE4M3 of Q, K (null: not written)
  uint4* deq[3];          // exact dequantised bf16 (null: not written)
  long long n16;          // 16-element blocks per tensor (even: rows of 64 or 128)
};

__global__ void __launch_bounds__(256)
quantize_nvfp4_qk_mxfp8_v_kernel(const __grid_constant__ MixedQuantJobs jobs) {
  const long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (b >= jobs.n16 / 2) return;
  if (t < 2) {
    const uint4* x = jobs.x[t];
    const uint4 v0 = x[4 * b], v1 = x[4 * b + 1], v2 = x[4 * b + 2], v3 = x[4 * b + 3];
    quantize_block_nvfp4_values(v0, v1, jobs.codes[t], jobs.scales[t], jobs.deq[t], 2 * b);
    quantize_block_nvfp4_values(v2, v3, jobs.codes[t], jobs.scales[t], jobs.deq[t], 2 * b + 1);
  } else {
    quantize_block(jobs.x[2], nullptr, nullptr, jobs.deq[2], b);
  }
}

}  // namespace attn

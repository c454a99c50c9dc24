// MXFP8 quantisation pre-pass: bf16 -> E4M3 element codes + one E8M0 scale
// per 32 contiguous elements of a row (for attention operands a row is one
// token of one head, so no scale spans two tokens and hence never a document
// or causal boundary).
//
// FLAMIA ("FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli
// Eğitim İçin Flash Mikro-Ölçeklemeli Dikkat Mekanizması", section "FLAMIA
// Mimarisi ve Temel Tasarım İlkeleri") fuses quantisation into its kernels
// and keeps scales from carrying information from future tokens to past ones;
// FlashAttention-3 ("FlashAttention, pelatihan multi-GPU, dan kuantisasi
// bobot", section 1) scales small blocks independently against outliers.
//
// Scale rule: X = the smallest integer with amax <= 448 * 2^X, found from the
// exponent and fraction bits of amax (exact, no division); code X + 127
// clamped to [0, 254]; amax == 0 -> 127.  Elements: x * 2^-(code - 127)
// (an exact power-of-two product) converted by the hardware's
// round-to-nearest-even, saturating E4M3 conversion.
//
// HBM-bound: each thread reads one 64-byte block and writes what the
// consumer needs: 32 + 1 bytes of codes and scale and/or 64 bytes of exact
// dequantised bf16.
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

namespace attn {

__device__ __forceinline__ uint32_t e8m0_code_from_amax(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  if (bits == 0u) return 127u;
  uint32_t exp_field = bits >> 23;
  uint32_t frac = bits & 0x7FFFFFu;
  int e;  // floor(log2(amax))
  if (exp_field == 0u) {  // subnormal: normalise the fraction
    const int shift = __clz(frac) - 8;
    frac = (frac << shift) & 0x7FFFFFu;
    e = -126 - shift;
  } else {
    e = static_cast<int>(exp_field) - 127;
  }
  // 448 = 1.75 * 2^8: amax = f * 2^e fits under 448 * 2^(e-8) iff f <= 1.75
  const int x = e - 8 + (frac > 0x600000u ? 1 : 0);
  return static_cast<uint32_t>(min(max(x + 127, 0), 254));
}

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 pair -> two fp32 (exact: through f16, which holds every E4M3 value).
__device__ __forceinline__ void e4m3x2_to_f32(uint16_t v, float& lo, float& hi) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// One 32-element block: E4M3 codes and the E8M0 scale, and/or the exact
// dequantised values (E4M3 value * 2^(code - 127)) as bf16: a 4-bit
// significand times a power of two is exact in bf16 over the whole range the
// scale rule produces.  Any of codes, scales and deq may be null (not
// written).
__device__ __forceinline__ void quantize_block(const uint4* __restrict__ x, uint4* __restrict__ codes,
                                               uint8_t* __restrict__ scales, uint4* __restrict__ deq,
                                               long long b) {
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = x[4 * b + i];
  const uint32_t* w = reinterpret_cast<const uint32_t*>(v);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  const uint32_t code = e8m0_code_from_amax(amax);
  // 2^-(code - 127) as an fp32 bit pattern; code 254 needs 2^-127 (subnormal).
  const int xexp = static_cast<int>(code) - 127;
  const float inv = xexp == 127 ? __uint_as_float(0x00400000u)
                                : __uint_as_float(static_cast<uint32_t>(127 - xexp) << 23);
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint16_t a = cvt_e4m3x2(bf16_lo(w[2 * i]) * inv, bf16_hi(w[2 * i]) * inv);
    const uint16_t c = cvt_e4m3x2(bf16_lo(w[2 * i + 1]) * inv, bf16_hi(w[2 * i + 1]) * inv);
    out[i] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(c) << 16);
  }
  if (codes != nullptr) {
    codes[2 * b] = make_uint4(out[0], out[1], out[2], out[3]);
    codes[2 * b + 1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
  if (scales != nullptr) scales[b] = static_cast<uint8_t>(code);
  if (deq != nullptr) {
    // 2^(code - 127); code 0 needs 2^-127 (subnormal)
    const float mul = code == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
    uint32_t y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float f0, f1, f2, f3;
      e4m3x2_to_f32(static_cast<uint16_t>(out[i] & 0xFFFFu), f0, f1);
      e4m3x2_to_f32(static_cast<uint16_t>(out[i] >> 16), f2, f3);
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(y[2 * i]) : "f"(f1 * mul), "f"(f0 * mul));
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(y[2 * i + 1]) : "f"(f3 * mul), "f"(f2 * mul));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) deq[4 * b + i] = make_uint4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
  }
}

// One thread per 32-element block; n_blocks = rows * cols / 32.
__global__ void __launch_bounds__(256)
quantize_mxfp8_kernel(const uint4* __restrict__ x, uint4* __restrict__ codes,
                      uint8_t* __restrict__ scales, uint4* __restrict__ deq, long long n_blocks) {
  const long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= n_blocks) return;
  quantize_block(x, codes, scales, deq, b);
}

// The operands of one attention call in one launch (blockIdx.y picks the
// tensor: Q, K, V, and dO for the backward), each with the outputs its
// consumer reads.
struct QuantJob {
  const uint4* x;
  uint4* codes;
  uint8_t* scales;
  uint4* deq;
};
struct QuantJobs {
  QuantJob t[4];
  long long n_blocks;   // per tensor
};

__global__ void __launch_bounds__(256)
quantize_mxfp8_qkv_kernel(const __grid_constant__ QuantJobs jobs) {
  const long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= jobs.n_blocks) return;
  const QuantJob& j = jobs.t[blockIdx.y];
  quantize_block(j.x, j.codes, j.scales, j.deq, b);
}

}  // namespace attn

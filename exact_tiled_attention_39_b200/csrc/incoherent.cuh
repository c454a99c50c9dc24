// Incoherent processing before MXFP8 quantisation: each row x (one token of
// one head, d = 64 or 128 bf16 values) becomes (x * s) H_d in fp32 and is
// then quantised to E4M3 codes with one E8M0 scale per 32 elements.
//
// "FlashAttention, pelatihan multi-GPU, dan kuantisasi bobot", section 1
// (FlashAttention-3's FP8 support): Q and K are multiplied by a random
// orthogonal matrix before quantisation so that outlier channels are spread
// over the whole head dimension; the scores are unchanged because the
// matrix is orthogonal.  Here the matrix is diag(s) H_d with H_d the
// Sylvester Hadamard matrix and s the caller's random signs, unnormalised
// (M M^T = d I; the caller divides the softmax scale by d).
//
// The rotation is the fast Walsh-Hadamard butterfly in registers, one thread
// per row: for span h = 1, 2, 4, ..., d/2 every pair (a, b) at distance h in
// a block of 2h becomes (a + b, a - b), each an fp32 add rounded to nearest.
// The quantiser then takes its E4M3 decisions on those fp32 values, so the
// codes can be checked bit for bit against a CPU restatement of the same
// order.  HBM-bound: 2 d bytes read, d + d / 32 bytes written per row.
#pragma once
#include <cstdint>

#include "quant_mxfp8.cuh"

namespace attn {

// 32 fp32 values -> 32 E4M3 codes (eight words) and the E8M0 scale code,
// by the scale rule of quantize_block.
__device__ __forceinline__ uint32_t quantize_block_f32(const float* v, uint32_t (&out)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t code = e8m0_code_from_amax(amax);
  const int xexp = static_cast<int>(code) - 127;
  const float inv = xexp == 127 ? __uint_as_float(0x00400000u)
                                : __uint_as_float(static_cast<uint32_t>(127 - xexp) << 23);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint16_t a = cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv);
    const uint16_t c = cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv);
    out[i] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(c) << 16);
  }
  return code;
}

// The rows of one tensor for the incoherent pre-pass of an attention call:
// any of codes, scales and deq may be null (not written).
struct RowQuantJob {
  const uint4* x;       // bf16 [rows][D]
  uint4* codes;         // E4M3 [rows][D]
  uint8_t* scales;      // E8M0 [rows][D / 32]
  uint4* deq;           // bf16 [rows][D]: exact dequantised values
  int rotate;           // 1: (x * s) H_d before quantisation; 0: x as it is
};
struct RowQuantJobs {
  RowQuantJob t[3];
  long long rows;       // per tensor
};

// One row: load, optionally rotate, quantise each 32-element block and write
// what the job asks for.
template <int D>
__device__ __forceinline__ void quantize_row(const RowQuantJob& j, const float* __restrict__ signs,
                                             long long row) {
  float y[D];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const uint4 w = j.x[row * (D / 8) + i];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      y[8 * i + 2 * q] = bf16_lo(ws[q]);
      y[8 * i + 2 * q + 1] = bf16_hi(ws[q]);
    }
  }
  if (j.rotate) {
#pragma unroll
    for (int i = 0; i < D; ++i) y[i] *= signs[i];          // exact: +-1
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
      for (int b0 = 0; b0 < D; b0 += 2 * h) {
#pragma unroll
        for (int q = 0; q < h; ++q) {
          const float a = y[b0 + q], b = y[b0 + q + h];
          y[b0 + q] = __fadd_rn(a, b);
          y[b0 + q + h] = __fsub_rn(a, b);
        }
      }
    }
  }
  uint32_t sc = 0;
#pragma unroll
  for (int blk = 0; blk < D / 32; ++blk) {
    uint32_t out[8];
    const uint32_t code = quantize_block_f32(y + 32 * blk, out);
    sc |= code << (8 * blk);
    if (j.codes != nullptr) {
      j.codes[row * (D / 16) + 2 * blk] = make_uint4(out[0], out[1], out[2], out[3]);
      j.codes[row * (D / 16) + 2 * blk + 1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
    if (j.deq != nullptr) {
      // E4M3 value * 2^(code - 127): exact in bf16 (code 0 needs 2^-127)
      const float mul = code == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
      uint32_t o[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float f0, f1, f2, f3;
        e4m3x2_to_f32(static_cast<uint16_t>(out[i] & 0xFFFFu), f0, f1);
        e4m3x2_to_f32(static_cast<uint16_t>(out[i] >> 16), f2, f3);
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[2 * i]) : "f"(f1 * mul), "f"(f0 * mul));
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[2 * i + 1]) : "f"(f3 * mul), "f"(f2 * mul));
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        j.deq[row * (D / 8) + 4 * blk + i] =
            make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
  }
  if (j.scales != nullptr) {
    if (D == 128) {
      reinterpret_cast<uint32_t*>(j.scales)[row] = sc;
    } else {
      reinterpret_cast<uint16_t*>(j.scales)[row] = static_cast<uint16_t>(sc);
    }
  }
}

// One thread per row of D bf16 values: codes [rows][D] (E4M3), scales
// [rows][D / 32] (E8M0), signs: D fp32 values (+-1).
template <int D>
__global__ void __launch_bounds__(128)
quantize_mxfp8_rotated_kernel(const uint4* __restrict__ x, const float* __restrict__ signs,
                              uint4* __restrict__ codes, uint8_t* __restrict__ scales,
                              long long rows) {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  const RowQuantJob j{x, codes, scales, nullptr, 1};
  quantize_row<D>(j, signs, row);
}

// The pre-pass of an attention call with incoherent processing: Q and K
// rotated then quantised, V quantised as it is, all three in one launch
// (blockIdx.y picks the tensor).
template <int D>
__global__ void __launch_bounds__(128)
quantize_mxfp8_incoherent_qkv_kernel(const __grid_constant__ RowQuantJobs jobs,
                                     const float* __restrict__ signs) {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= jobs.rows) return;
  quantize_row<D>(jobs.t[blockIdx.y], signs, row);
}

}  // namespace attn

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
// The rotation is the fast Walsh-Hadamard butterfly in registers, a row
// spread over d / 8 lanes: for span h = 1, 2, 4, ..., d/2 every pair (a, b)
// at distance h in a block of 2h becomes (a + b, a - b), each an fp32 add
// rounded to nearest.  The quantiser then takes its E4M3 decisions on those
// fp32 values, so the codes can be checked bit for bit against a CPU
// restatement of the same order.  HBM-bound: 2 d bytes read, d + d / 32
// bytes written per row.
#pragma once
#include <cstdint>

#include "quant_mxfp8.cuh"

namespace attn {

// The rows of one tensor for the incoherent pre-pass of an attention call:
// any of codes, scales and deq may be null (not written).
struct RowQuantJob {
  const uint4* x;       // bf16 [rows][D]
  uint2* codes;         // E4M3 [rows][D], 8 bytes per lane
  uint8_t* scales;      // E8M0 [rows][D / 32]
  uint4* deq;           // bf16 [rows][D]: exact dequantised values
  int rotate;           // 1: (x * s) H_d before quantisation; 0: x as it is
};
struct RowQuantJobs {
  RowQuantJob t[3];
  long long rows;       // per tensor
};

// One row spread over D / 8 consecutive lanes (8 elements each, one 16-byte
// load: the lanes of a warp read contiguous memory).  The butterfly's spans
// 1, 2, 4 pair elements inside a lane; spans 8 .. D/2 pair lane l with lane
// l ^ (span / 8), which receives its partner's value by a shuffle: the lower
// element of a pair becomes a + b, the upper a - b, the same fp32 additions
// in the same order as one thread per row would make.  A 32-element
// quantisation block is four lanes; its maximum comes from two shuffles.
// Every lane of the warp must call this (rows past the end pass valid = 0);
// w is the lane's 16 bytes of the row (loaded by the caller, so that several
// rows' loads are in flight at once), sg the lane's 8 signs.
template <int D>
__device__ __forceinline__ void quantize_row_lanes(const RowQuantJob& j, const float (&sg)[8],
                                                   long long row, bool valid, uint4 w) {
  constexpr int kLanes = D / 8;
  const int sub = static_cast<int>(threadIdx.x) & (kLanes - 1);
  float y[8];
  {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      y[2 * q] = bf16_lo(ws[q]);
      y[2 * q + 1] = bf16_hi(ws[q]);
    }
  }
  if (j.rotate) {
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] *= sg[e];                      // exact: +-1
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (e & h) continue;
        const float a = y[e], b = y[e + h];
        y[e] = __fadd_rn(a, b);
        y[e + h] = __fsub_rn(a, b);
      }
    }
#pragma unroll
    for (int hl = 1; hl < kLanes; hl <<= 1) {
      const bool upper = (sub & hl) != 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float other = __shfl_xor_sync(0xffffffffu, y[e], hl);
        y[e] = upper ? __fsub_rn(other, y[e]) : __fadd_rn(y[e], other);
      }
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  if (!valid) return;
  const uint32_t code = e8m0_code_from_amax(amax);
  const int xexp = static_cast<int>(code) - 127;
  const float inv = xexp == 127 ? __uint_as_float(0x00400000u)
                                : __uint_as_float(static_cast<uint32_t>(127 - xexp) << 23);
  uint32_t out[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint16_t a = cvt_e4m3x2(y[4 * i] * inv, y[4 * i + 1] * inv);
    const uint16_t c = cvt_e4m3x2(y[4 * i + 2] * inv, y[4 * i + 3] * inv);
    out[i] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(c) << 16);
  }
  if (j.codes != nullptr) j.codes[row * kLanes + sub] = make_uint2(out[0], out[1]);
  if (j.scales != nullptr && (sub & 3) == 0)
    j.scales[row * (D / 32) + (sub >> 2)] = static_cast<uint8_t>(code);
  if (j.deq != nullptr) {
    // E4M3 value * 2^(code - 127): exact in bf16 (code 0 needs 2^-127)
    const float mul = code == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float f0, f1, f2, f3;
      e4m3x2_to_f32(static_cast<uint16_t>(out[i] & 0xFFFFu), f0, f1);
      e4m3x2_to_f32(static_cast<uint16_t>(out[i] >> 16), f2, f3);
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[2 * i]) : "f"(f1 * mul), "f"(f0 * mul));
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[2 * i + 1]) : "f"(f3 * mul), "f"(f2 * mul));
    }
    j.deq[row * kLanes + sub] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Rows per thread of the rotating kernels: a 256-thread block takes
// kRotRowsPerThread groups of 256 / (D / 8) consecutive rows, and each
// thread loads its rows' 16 bytes before working on the first, so that
// several loads per thread are in flight (one is too few to keep HBM busy).
constexpr int kRotRowsPerThread = 4;

template <int D>
__device__ __forceinline__ void quantize_rows_block(const RowQuantJob& j,
                                                    const float* __restrict__ signs,
                                                    long long rows) {
  constexpr int kLanes = D / 8;
  constexpr int kRowsPerPass = 256 / kLanes;
  const int sub = static_cast<int>(threadIdx.x) & (kLanes - 1);
  const long long row0 = static_cast<long long>(blockIdx.x) * (kRowsPerPass * kRotRowsPerThread) +
                         static_cast<int>(threadIdx.x) / kLanes;
  float sg[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sg[e] = j.rotate ? signs[8 * sub + e] : 1.f;
  uint4 w[kRotRowsPerThread];
#pragma unroll
  for (int i = 0; i < kRotRowsPerThread; ++i) {
    const long long row = row0 + i * kRowsPerPass;
    w[i] = row < rows ? j.x[row * kLanes + sub] : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < kRotRowsPerThread; ++i) {
    const long long row = row0 + i * kRowsPerPass;
    quantize_row_lanes<D>(j, sg, row, row < rows, w[i]);
  }
}

// Rows of D bf16 values, D / 8 lanes each: codes [rows][D] (E4M3), scales
// [rows][D / 32] (E8M0), signs: D fp32 values (+-1).
template <int D>
__global__ void __launch_bounds__(256)
quantize_mxfp8_rotated_kernel(const uint4* __restrict__ x, const float* __restrict__ signs,
                              uint2* __restrict__ codes, uint8_t* __restrict__ scales,
                              long long rows) {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  const RowQuantJob j{x, codes, scales, nullptr, 1};
  quantize_rows_block<D>(j, signs, rows);
}

// The pre-pass of an attention call with incoherent processing: Q and K
// rotated then quantised, V quantised as it is, all three in one launch
// (blockIdx.y picks the tensor).
template <int D>
__global__ void __launch_bounds__(256)
quantize_mxfp8_incoherent_qkv_kernel(const __grid_constant__ RowQuantJobs jobs,
                                     const float* __restrict__ signs) {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  quantize_rows_block<D>(jobs.t[blockIdx.y], signs, jobs.rows);
}

}  // namespace attn

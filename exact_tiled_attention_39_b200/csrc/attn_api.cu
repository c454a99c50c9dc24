// Host side of the C ABI declared in include/attn.h: argument checks,
// workspace carving, TMA tensor-map encoding and the kernel launches.
// Everything is asynchronous on the caller's stream; nothing is allocated.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_fwd_pair_sm100.cuh"
#include "attn_fwd_sm100.cuh"
#include "common.cuh"
#include "incoherent.cuh"
#include "quant_mxfp8.cuh"
#include "quant_nvfp4.cuh"
#include "schedule.cuh"

namespace attn {
namespace {

// Events of the timed call (attn_timing_enable / attn_timing_read).
struct CallTiming {
  std::mutex mu;
  bool enabled = false;
  bool recorded = false;
  int device = -1;
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};   // call start, kernel start, kernel end
};
CallTiming g_timing;

// Records event i of the timed call on `strm` when timing is enabled.
void timing_mark(int i, cudaStream_t strm) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (!g_timing.enabled) return;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  if (dev != g_timing.device) {
    for (auto& e : g_timing.ev)
      if (e != nullptr) {
        cudaEventDestroy(e);
        e = nullptr;
      }
    g_timing.device = dev;
    g_timing.recorded = false;
  }
  if (g_timing.ev[i] == nullptr && cudaEventCreate(&g_timing.ev[i]) != cudaSuccess) {
    g_timing.ev[i] = nullptr;
    return;
  }
  if (cudaEventRecord(g_timing.ev[i], strm) == cudaSuccess && i == 2) g_timing.recorded = true;
}

constexpr int kMaxDevices = 64;
constexpr int kScheduleThreads = 1024;
constexpr int kSortCapacityMax = 16384;                   // 128 KB of keys
// Limit of every mbarrier wait in the kernels (a build for the failure tests
// sets a short one).
#ifndef ATTN_WAIT_TIMEOUT_NS
#define ATTN_WAIT_TIMEOUT_NS 1000000000ull
#endif
constexpr unsigned long long kWaitTimeoutNs = ATTN_WAIT_TIMEOUT_NS;  // 1 s per wait by default

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t sort_capacity_for(int64_t max_entries) {
  int64_t c = 1;
  while (c < max_entries) c <<= 1;
  return c > kSortCapacityMax ? 0 : c;
}

struct WsLayout {
  size_t sorted_off, unsorted_off, mx_off, total;
  // MXFP8 / NVFP4: per operand (q, k, v) codes, scales, bf16 dequantised copy
  size_t codes_off[3], scales_off[3], deq_off[3];
  int64_t max_entries;
};

bool valid_fwd_dtype(attn_dtype_t dtype) {
  return dtype == ATTN_BF16 || dtype == ATTN_MXFP8 || dtype == ATTN_NVFP4;
}

WsLayout ws_layout(const attn_shape_t& s, attn_dtype_t dtype) {
  WsLayout w{};
  w.max_entries = max_work_entries(s.total_tokens, s.num_seqs);
  w.sorted_off = kWsListOffset;
  w.unsorted_off = align_up(w.sorted_off + 16 * static_cast<size_t>(w.max_entries), kWsAlign);
  w.mx_off = align_up(w.unsorted_off + 16 * static_cast<size_t>(w.max_entries), kWsAlign);
  w.total = w.mx_off;
  if (dtype == ATTN_MXFP8 || dtype == ATTN_NVFP4) {
    const size_t elems = static_cast<size_t>(s.total_tokens) * s.num_heads * s.head_dim;
    // MXFP8: one E4M3 byte per element, one E8M0 scale per 32; NVFP4 (q and
    // k): half a byte per element, one UE4M3 scale per 16
    const bool nv = dtype == ATTN_NVFP4;
    for (int i = 0; i < 3; ++i) {
      w.codes_off[i] = w.total;
      w.total = align_up(w.total + (nv ? elems / 2 : elems), kWsAlign);
      w.scales_off[i] = w.total;
      w.total = align_up(w.total + (nv ? elems / 16 : elems / 32), kWsAlign);
      w.deq_off[i] = w.total;
      w.total = align_up(w.total + 2 * elems, kWsAlign);
    }
  }
  return w;
}

attn_status_t check_shape(const attn_shape_t* s) {
  if (s == nullptr) return ATTN_ERR_INVALID_ARG;
  if (s->total_tokens < 0 || s->num_seqs < 0 || s->num_heads < 1 || s->max_seqlen < 0)
    return ATTN_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (s->total_tokens > 0 && s->num_seqs < 1) return ATTN_ERR_INVALID_ARG;
  const int64_t elems = static_cast<int64_t>(s->total_tokens) * s->num_heads;
  if (elems > (int64_t(1) << 31)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

attn_status_t device_info(int* dev_out, DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return ATTN_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaFuncSetAttribute(attn_fwd_pair_kernel<128, kQkNv4>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairLayout<128, kQkNv4>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_pair_kernel<64, kQkBf16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairLayout<64, kQkBf16>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_pair_kernel<128, kQkBf16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairLayout<128, kQkBf16>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_pair_kernel<128, kQkMx8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairLayout<128, kQkMx8>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(build_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSortCapacityMax * 8) != cudaSuccess)
      return ATTN_ERR_CUDA;
    d.ready = true;
  }
  *dev_out = dev;
  *info = d;
  return ATTN_OK;
}

// 3-D map over a [T, H, d] tensor of `elem` bytes per element: box = 128
// bytes of head dim (the swizzle span) x 1 head x box_rows tokens, 128-byte
// swizzle, zero fill outside the tensor.
bool encode_qkv_map(CUtensorMap* m, const void* base, int T, int H, int d, int elem,
                    int box_rows = kBlockM) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem,
                                 static_cast<cuuint64_t>(H) * d * elem};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), 1,
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                  3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over packed E2M1 codes [T, H, d / 2 bytes]: box = the d / 2 bytes
// of a row (64 for d = 128) x 1 head x box_rows tokens, 64-byte swizzle.
bool encode_fp4_map(CUtensorMap* m, const void* base, int T, int H, int d,
                    int box_rows = kBlockM) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d / 2), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d / 2),
                                 static_cast<cuuint64_t>(H) * (d / 2)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(d / 2), 1,
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

int32_t attn_abi_version(void) { return ATTN_ABI_VERSION; }

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_ALIGNMENT: return "ATTN_ERR_ALIGNMENT";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_BAD_SEQLENS: return "ATTN_ERR_BAD_SEQLENS";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
  }
  return "ATTN_ERR_UNKNOWN";
}

size_t attn_workspace_size(const attn_shape_t* shape, attn_dtype_t dtype) {
  if (check_shape(shape) != ATTN_OK) return 0;
  if (!valid_fwd_dtype(dtype)) return 0;
  return ws_layout(*shape, dtype).total;
}

attn_status_t attn_quantize_mxfp8(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows,
                                  int32_t cols, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return ATTN_ERR_INVALID_ARG;
  if (rows == 0) return ATTN_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes)) return ATTN_ERR_ALIGNMENT;
  const long long n_blocks = rows * static_cast<long long>(cols / 32);
  const int threads = 256;
  const long long grid = (n_blocks + threads - 1) / threads;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  quantize_mxfp8_kernel<<<static_cast<unsigned>(grid), threads, 0,
                          static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(x), reinterpret_cast<uint4*>(codes), scales, nullptr, n_blocks);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

namespace attn {
namespace {

// The forward of attn_fwd and attn_fwd_incoherent.  signs != nullptr (MXFP8
// only) selects incoherent processing: Q and K rotated by diag(signs) H_d
// in the pre-pass, the softmax scale divided by d.
attn_status_t fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                       void* out, float* lse, int causal, float scale, attn_dtype_t dtype,
                       const float* signs, void* stream, const attn_shape_t* shape,
                       void* workspace, size_t workspace_bytes) {
  const attn_status_t st = check_shape(shape);
  if (st != ATTN_OK) return st;
  if (!valid_fwd_dtype(dtype)) return ATTN_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  const attn_shape_t s = *shape;
  if (cu_seqlens == nullptr &&
      static_cast<int64_t>(s.num_seqs) * s.max_seqlen != static_cast<int64_t>(s.total_tokens))
    return ATTN_ERR_INVALID_ARG;
  if (s.total_tokens == 0) return ATTN_OK;
  if (!q || !k || !v || !out || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return ATTN_ERR_ALIGNMENT;
  const WsLayout wl = ws_layout(s, dtype);
  if (workspace == nullptr || workspace_bytes < wl.total) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;

  int dev = 0;
  DeviceInfo info;
  if (device_info(&dev, &info) != ATTN_OK) return ATTN_ERR_CUDA;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* header = reinterpret_cast<int32_t*>(ws);

  // Every path runs the two-query-tile kernel; the block-scaled forms
  // (MXFP8, NVFP4 at d = 128) with 112-key tiles.
  const bool nv4 = dtype == ATTN_NVFP4;
  const bool fp8_kernel = (dtype == ATTN_MXFP8 || nv4) && s.head_dim == 128;
  const int kv_rows = fp8_kernel ? PairLayout<128, kQkMx8>::kBN : kBlockN;
  timing_mark(0, strm);
  // 1. schedule (validates cu_seqlens, writes the work list and its length)
  const int64_t cap = sort_capacity_for(wl.max_entries);
  build_schedule_kernel<<<1, kScheduleThreads, static_cast<size_t>(cap) * 8, strm>>>(
      cu_seqlens, s.num_seqs, s.total_tokens, s.max_seqlen, s.max_seqlen, causal,
      2, header,
      reinterpret_cast<int4*>(ws + wl.sorted_off), reinterpret_cast<int4*>(ws + wl.unsorted_off),
      static_cast<int>(cap));
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

  // 2. MXFP8: quantise q, k, v (E4M3 + one E8M0 scale per token, head and 32
  // head-dim elements).  With d = 128 the score product runs block-scaled on
  // the E4M3 codes of q and k, and P V on the exact bf16 dequantisation of v;
  // with d = 64 all three products run on the dequantised values.
  const void* qk_src[2] = {q, k};
  if (dtype == ATTN_MXFP8 && signs != nullptr) {
    // Incoherent processing: one launch for the three tensors, one thread per
    // (token, head) row; Q and K rotated, V quantised as it is.  Outputs as
    // for the plain pre-pass below.
    RowQuantJobs jobs;
    jobs.rows = static_cast<long long>(s.total_tokens) * s.num_heads;
    const void* src[3] = {q, k, v};
    for (int i = 0; i < 3; ++i) {
      const bool use_codes = fp8_kernel && i < 2;
      jobs.t[i].x = static_cast<const uint4*>(src[i]);
      jobs.t[i].codes = use_codes ? reinterpret_cast<uint2*>(ws + wl.codes_off[i]) : nullptr;
      jobs.t[i].scales = use_codes ? ws + wl.scales_off[i] : nullptr;
      jobs.t[i].deq = use_codes ? nullptr : reinterpret_cast<uint4*>(ws + wl.deq_off[i]);
      jobs.t[i].rotate = i < 2 ? 1 : 0;
    }
    // D / 8 lanes per row, 256 threads per block, kRotRowsPerThread rows a thread
    const long long rows_per_block = 256 / (s.head_dim / 8) * kRotRowsPerThread;
    const long long qgrid = (jobs.rows + rows_per_block - 1) / rows_per_block;
    if (qgrid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (s.head_dim == 128)
      quantize_mxfp8_incoherent_qkv_kernel<128>
          <<<dim3(static_cast<unsigned>(qgrid), 3), 256, 0, strm>>>(jobs, signs);
    else
      quantize_mxfp8_incoherent_qkv_kernel<64>
          <<<dim3(static_cast<unsigned>(qgrid), 3), 256, 0, strm>>>(jobs, signs);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    for (int i = 0; i < 2; ++i) qk_src[i] = ws + (fp8_kernel ? wl.codes_off[i] : wl.deq_off[i]);
    v = ws + wl.deq_off[2];
    // (Q M)(K M)^T = d Q K^T: exact division by the power of two d
    scale /= static_cast<float>(s.head_dim);
  } else if (nv4) {
    // Mixed NVFP4 / FP8 path: Q and K to NVFP4 (packed E2M1 codes and UE4M3
    // scales for the block-scaled kernel; the exact dequantised values for
    // head dim 64), V to MXFP8 (exact dequantised bf16), one launch.
    MixedQuantJobs jobs;
    const void* src[3] = {q, k, v};
    for (int i = 0; i < 3; ++i) {
      jobs.x[i] = static_cast<const uint4*>(src[i]);
      jobs.deq[i] = (i == 2 || !fp8_kernel) ? reinterpret_cast<uint4*>(ws + wl.deq_off[i]) : nullptr;
    }
    for (int i = 0; i < 2; ++i) {
      jobs.codes[i] = fp8_kernel ? reinterpret_cast<uint2*>(ws + wl.codes_off[i]) : nullptr;
      jobs.scales[i] = fp8_kernel ? ws + wl.scales_off[i] : nullptr;
    }
    jobs.n16 = static_cast<long long>(s.total_tokens) * s.num_heads * (s.head_dim / 16);
    const long long qgrid = (jobs.n16 / 2 + 255) / 256;     // one thread per 32 elements
    if (qgrid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    quantize_nvfp4_qk_mxfp8_v_kernel<<<dim3(static_cast<unsigned>(qgrid), 3), 256, 0, strm>>>(jobs);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    for (int i = 0; i < 2; ++i) qk_src[i] = ws + (fp8_kernel ? wl.codes_off[i] : wl.deq_off[i]);
    v = ws + wl.deq_off[2];
  } else if (dtype == ATTN_MXFP8) {
    // One launch for all three tensors.  The block-scaled kernel reads the
    // codes and scales of Q and K and the exact dequantised V; the head-dim
    // 64 fallback reads dequantised Q, K and V.
    const void* src[3] = {q, k, v};
    const long long n_blocks =
        static_cast<long long>(s.total_tokens) * s.num_heads * (s.head_dim / 32);
    QuantJobs jobs;
    jobs.n_blocks = n_blocks;
    for (int i = 0; i < 3; ++i) {
      const bool use_codes = fp8_kernel && i < 2;
      jobs.t[i].x = static_cast<const uint4*>(src[i]);
      jobs.t[i].codes = use_codes ? reinterpret_cast<uint4*>(ws + wl.codes_off[i]) : nullptr;
      jobs.t[i].scales = use_codes ? ws + wl.scales_off[i] : nullptr;
      jobs.t[i].deq = use_codes ? nullptr : reinterpret_cast<uint4*>(ws + wl.deq_off[i]);
    }
    const long long qgrid = (n_blocks + 255) / 256;
    if (qgrid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    quantize_mxfp8_qkv_kernel<<<dim3(static_cast<unsigned>(qgrid), 3), 256, 0, strm>>>(jobs);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    for (int i = 0; i < 2; ++i) qk_src[i] = ws + (fp8_kernel ? wl.codes_off[i] : wl.deq_off[i]);
    v = ws + wl.deq_off[2];
  }

  // 3. attention
  const int qk_elem = fp8_kernel ? 1 : 2;
  CUtensorMap tq, tk, tv;
  if (fp8_kernel && nv4) {
    if (!encode_fp4_map(&tq, qk_src[0], s.total_tokens, s.num_heads, s.head_dim) ||
        !encode_fp4_map(&tk, qk_src[1], s.total_tokens, s.num_heads, s.head_dim, kv_rows))
      return ATTN_ERR_CUDA;
  } else if (!encode_qkv_map(&tq, qk_src[0], s.total_tokens, s.num_heads, s.head_dim, qk_elem) ||
             !encode_qkv_map(&tk, qk_src[1], s.total_tokens, s.num_heads, s.head_dim, qk_elem,
                             kv_rows)) {
    return ATTN_ERR_CUDA;
  }
  if (!encode_qkv_map(&tv, v, s.total_tokens, s.num_heads, s.head_dim, 2, kv_rows))
    return ATTN_ERR_CUDA;
  FwdParams fp;
  fp.out = out;
  fp.lse = lse;
  fp.ws_header = header;
  fp.work = reinterpret_cast<const int4*>(ws + wl.sorted_off);
  fp.err = header + kWsErrorOffset / 4;
  fp.q_scales = fp8_kernel ? reinterpret_cast<const uint32_t*>(ws + wl.scales_off[0]) : nullptr;
  fp.k_scales = fp8_kernel ? reinterpret_cast<const uint32_t*>(ws + wl.scales_off[1]) : nullptr;
  fp.total_tokens = s.total_tokens;
  fp.num_heads = s.num_heads;
  fp.head_groups = head_group_count(s.total_tokens, s.num_heads, s.head_dim, fp8_kernel ? 3 : 4);
  fp.causal = causal;
  fp.scale_log2 = scale * 1.4426950408889634f;
  fp.timeout_ns = kWaitTimeoutNs;
  const int64_t max_units = wl.max_entries * s.num_heads;
  const int grid = static_cast<int>(max_units < info.num_sms ? max_units : info.num_sms);
  // Programmatic dependent launch: the attention kernel's prologue (barrier
  // set-up, TMEM allocation, tensor-map prefetch) overlaps the schedule
  // kernel; it waits for the work list with griddepcontrol.wait.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kPairThreads);
  cfg.stream = strm;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  timing_mark(1, strm);
  if (fp8_kernel && nv4) {
    cfg.dynamicSmemBytes = PairLayout<128, kQkNv4>::kBytes;
    e = cudaLaunchKernelEx(&cfg, attn_fwd_pair_kernel<128, kQkNv4>, tq, tk, tv, fp);
  } else if (fp8_kernel) {
    cfg.dynamicSmemBytes = PairLayout<128, kQkMx8>::kBytes;
    e = cudaLaunchKernelEx(&cfg, attn_fwd_pair_kernel<128, kQkMx8>, tq, tk, tv, fp);
  } else if (s.head_dim == 128) {
    cfg.dynamicSmemBytes = PairLayout<128, kQkBf16>::kBytes;
    e = cudaLaunchKernelEx(&cfg, attn_fwd_pair_kernel<128, kQkBf16>, tq, tk, tv, fp);
  } else {
    cfg.dynamicSmemBytes = PairLayout<64, kQkBf16>::kBytes;
    e = cudaLaunchKernelEx(&cfg, attn_fwd_pair_kernel<64, kQkBf16>, tq, tk, tv, fp);
  }
  timing_mark(2, strm);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace attn

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                       void* out, float* lse, int causal, float scale, attn_dtype_t dtype,
                       void* stream, const attn_shape_t* shape, void* workspace,
                       size_t workspace_bytes) {
  return fwd_impl(q, k, v, cu_seqlens, out, lse, causal, scale, dtype, nullptr, stream, shape,
                  workspace, workspace_bytes);
}

attn_status_t attn_fwd_incoherent(const void* q, const void* k, const void* v,
                                  const int32_t* cu_seqlens, void* out, float* lse, int causal,
                                  float scale, const float* signs, void* stream,
                                  const attn_shape_t* shape, void* workspace,
                                  size_t workspace_bytes) {
  if (shape != nullptr && shape->total_tokens > 0) {
    if (signs == nullptr) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(signs) & 3u) != 0) return ATTN_ERR_ALIGNMENT;
  }
  return fwd_impl(q, k, v, cu_seqlens, out, lse, causal, scale, ATTN_MXFP8,
                  signs != nullptr ? signs : nullptr, stream, shape, workspace, workspace_bytes);
}

attn_status_t attn_timing_enable(int32_t enable) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  g_timing.enabled = enable != 0;
  g_timing.recorded = false;
  return ATTN_OK;
}

attn_status_t attn_timing_read(float* attention_ms, float* prepass_ms) {
  if (attention_ms == nullptr || prepass_ms == nullptr) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (!g_timing.recorded) return ATTN_ERR_INVALID_ARG;
  if (cudaEventSynchronize(g_timing.ev[2]) != cudaSuccess ||
      cudaEventElapsedTime(attention_ms, g_timing.ev[1], g_timing.ev[2]) != cudaSuccess ||
      cudaEventElapsedTime(prepass_ms, g_timing.ev[0], g_timing.ev[1]) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status_t attn_get_device_error(const void* workspace, void* stream, int32_t* device_status) {
  if (workspace == nullptr || device_status == nullptr) return ATTN_ERR_INVALID_ARG;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(strm) != cudaSuccess) return ATTN_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpy(const_cast<void*>(workspace), &zero, sizeof(zero), cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return ATTN_ERR_CUDA;
  *device_status = v;
  return ATTN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// attn_fwd_noalloc: the bf16 forward for callers that cannot allocate device
// memory (see include/attn.h).  Its scratch - the error word and the two
// work lists the schedule-build kernel writes and the attention kernel reads
// - is this fixed array, part of the library's device image: every GPU that
// loads the library holds it until the process exits.  All calls share it.
// ---------------------------------------------------------------------------
namespace attn {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, looked up once per device with that device
// current.  In host code `g_noalloc_scratch` names a host-side stand-in, not
// device memory, so it is never passed to a kernel directly.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

}  // namespace
}  // namespace attn

extern "C" attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                          const int32_t* cu_seqlens, void* out, float* lse,
                                          int causal, float scale, void* stream,
                                          const attn_shape_t* shape) {
  const attn_status_t st = check_shape(shape);
  if (st != ATTN_OK) return st;
  // Reject problems whose work lists do not fit the fixed scratch.
  if (ws_layout(*shape, ATTN_BF16).total > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return ATTN_ERR_CUDA;
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  // The schedule-build kernel rewrites the error word, the list length and
  // both lists on every call, so nothing left by an earlier call is read.
  return attn_fwd(q, k, v, cu_seqlens, out, lse, causal, scale, ATTN_BF16, stream, shape,
                  scratch, kNoAllocScratchBytes);
}

// ===========================================================================
// Backward (bf16): attn_bwd_workspace_size, attn_bwd.  The forward's sources
// end above this line.
// ===========================================================================
#include "attn_bwd_sm100.cuh"

namespace attn {
namespace {

struct BwdWsLayout {
  size_t sorted_off, unsorted_off, delta_off, dq_off, total;
  size_t deq_off[4];   // MXFP8: exact dequantised q, k, v, dout (bf16 [T, H, d])
  int64_t max_entries;
};

BwdWsLayout bwd_ws_layout(const attn_shape_t& s, attn_dtype_t dtype) {
  BwdWsLayout w{};
  w.max_entries = max_work_entries(s.total_tokens, s.num_seqs);
  w.sorted_off = kWsListOffset;
  w.unsorted_off = align_up(w.sorted_off + 16 * static_cast<size_t>(w.max_entries), kWsAlign);
  w.delta_off = align_up(w.unsorted_off + 16 * static_cast<size_t>(w.max_entries), kWsAlign);
  const size_t rows = static_cast<size_t>(s.total_tokens) * s.num_heads;
  w.dq_off = align_up(w.delta_off + 4 * rows, kWsAlign);
  w.total = align_up(w.dq_off + 4 * rows * s.head_dim, kWsAlign);
  if (dtype == ATTN_MXFP8) {
    for (int i = 0; i < 4; ++i) {
      w.deq_off[i] = w.total;
      w.total = align_up(w.total + 2 * rows * s.head_dim, kWsAlign);
    }
  }
  return w;
}

bool g_bwd_ready[kMaxDevices] = {};

// 3-D map over the fp32 dQ accumulator [T, H, d] for the kernel's reduce-add
// copies: box = 32 fp32 of head dim (128 bytes, the swizzle span) x 1 head x
// 32 tokens, 128-byte swizzle.
bool encode_dq_map(CUtensorMap* m, void* base, int T, int H, int d) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(H) * d * 4};
  const cuuint32_t box[3] = {32, 1, 32};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

attn_status_t bwd_kernel_attributes(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_bwd_ready[dev]) return ATTN_OK;
  if (cudaFuncSetAttribute(attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           BwdLayout<64>::kBytes) != cudaSuccess ||
      cudaFuncSetAttribute(attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           BwdLayout<128>::kBytes) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_bwd_ready[dev] = true;
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

extern "C" {

size_t attn_bwd_workspace_size(const attn_shape_t* shape, attn_dtype_t dtype) {
  if (check_shape(shape) != ATTN_OK) return 0;
  if (dtype != ATTN_BF16 && dtype != ATTN_MXFP8) return 0;
  return bwd_ws_layout(*shape, dtype).total;
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, const int32_t* cu_seqlens, void* dq,
                       void* dk, void* dv, int causal, float scale, attn_dtype_t dtype,
                       void* stream, const attn_shape_t* shape, void* workspace,
                       size_t workspace_bytes) {
  const attn_status_t st = check_shape(shape);
  if (st != ATTN_OK) return st;
  if (dtype != ATTN_BF16 && dtype != ATTN_MXFP8) return ATTN_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  const attn_shape_t s = *shape;
  if (cu_seqlens == nullptr &&
      static_cast<int64_t>(s.num_seqs) * s.max_seqlen != static_cast<int64_t>(s.total_tokens))
    return ATTN_ERR_INVALID_ARG;
  if (s.total_tokens == 0) return ATTN_OK;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  const void* ptrs[9] = {q, k, v, out, dout, lse, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return ATTN_ERR_ALIGNMENT;
  const BwdWsLayout wl = bwd_ws_layout(s, dtype);
  if (workspace == nullptr || workspace_bytes < wl.total) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGNMENT;

  int dev = 0;
  DeviceInfo info;
  if (device_info(&dev, &info) != ATTN_OK) return ATTN_ERR_CUDA;
  if (bwd_kernel_attributes(dev) != ATTN_OK) return ATTN_ERR_CUDA;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* header = reinterpret_cast<int32_t*>(ws);
  float* delta = reinterpret_cast<float*>(ws + wl.delta_off);
  float* dq_acc = reinterpret_cast<float*>(ws + wl.dq_off);

  // 1. schedule: one entry per 128-token tile of each document, heaviest
  //    first (validates cu_seqlens)
  const int64_t cap = sort_capacity_for(wl.max_entries);
  build_schedule_kernel<<<1, kScheduleThreads, static_cast<size_t>(cap) * 8, strm>>>(
      cu_seqlens, s.num_seqs, s.total_tokens, s.max_seqlen, s.max_seqlen, causal, 1, header,
      reinterpret_cast<int4*>(ws + wl.sorted_off), reinterpret_cast<int4*>(ws + wl.unsorted_off),
      static_cast<int>(cap));
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

  // 1b. MXFP8: Q, K, V and dO quantised (E4M3, one E8M0 scale per token,
  //     head and 32 head-dim elements) and exactly dequantised in one
  //     launch; every product below reads these values, in whichever
  //     orientation it needs them, so the forward (which quantises Q, K, V
  //     the same way) and the backward see one set of operands.
  if (dtype == ATTN_MXFP8) {
    const void* src[4] = {q, k, v, dout};
    QuantJobs jobs;
    jobs.n_blocks = static_cast<long long>(s.total_tokens) * s.num_heads * (s.head_dim / 32);
    for (int i = 0; i < 4; ++i) {
      jobs.t[i].x = static_cast<const uint4*>(src[i]);
      jobs.t[i].codes = nullptr;
      jobs.t[i].scales = nullptr;
      jobs.t[i].deq = reinterpret_cast<uint4*>(ws + wl.deq_off[i]);
    }
    const long long qgrid = (jobs.n_blocks + 255) / 256;
    if (qgrid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    quantize_mxfp8_qkv_kernel<<<dim3(static_cast<unsigned>(qgrid), 4), 256, 0, strm>>>(jobs);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    q = ws + wl.deq_off[0];
    k = ws + wl.deq_off[1];
    v = ws + wl.deq_off[2];
    dout = ws + wl.deq_off[3];
  }

  // 2. D = rowsum(dO * O), dQ accumulator cleared
  const long long rows = static_cast<long long>(s.total_tokens) * s.num_heads;
  const long long prep_threads = rows * (s.head_dim / 8);
  const long long prep_grid = (prep_threads + 255) / 256;
  if (prep_grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  attn_bwd_prep_kernel<<<static_cast<unsigned>(prep_grid), 256, 0, strm>>>(
      static_cast<const uint4*>(out), static_cast<const uint4*>(dout), delta,
      reinterpret_cast<float4*>(dq_acc), rows, s.head_dim, s.num_heads, s.total_tokens);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

  // 3. dK, dV and the dQ partial sums, one key tile per unit
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (!encode_qkv_map(&tq, q, s.total_tokens, s.num_heads, s.head_dim, 2) ||
      !encode_qkv_map(&tk, k, s.total_tokens, s.num_heads, s.head_dim, 2) ||
      !encode_qkv_map(&tv, v, s.total_tokens, s.num_heads, s.head_dim, 2) ||
      !encode_qkv_map(&tdo, dout, s.total_tokens, s.num_heads, s.head_dim, 2) ||
      !encode_dq_map(&tdq, dq_acc, s.total_tokens, s.num_heads, s.head_dim))
    return ATTN_ERR_CUDA;
  BwdParams bp;
  bp.lse = lse;
  bp.delta = delta;
  bp.dq_acc = dq_acc;
  bp.dk = dk;
  bp.dv = dv;
  bp.ws_header = header;
  bp.work = reinterpret_cast<const int4*>(ws + wl.sorted_off);
  bp.err = header + kWsErrorOffset / 4;
  bp.total_tokens = s.total_tokens;
  bp.num_heads = s.num_heads;
  // Q and dO of a head are what every key tile of it reads again.
  bp.head_groups = head_group_count(s.total_tokens, s.num_heads, s.head_dim, 4);
  bp.causal = causal;
  bp.scale = scale;
  bp.scale_log2 = scale * 1.4426950408889634f;
  bp.timeout_ns = kWaitTimeoutNs;
  const int64_t max_units = wl.max_entries * s.num_heads;
  const int grid = static_cast<int>(max_units < info.num_sms ? max_units : info.num_sms);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kBwdThreads);
  cfg.stream = strm;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (s.head_dim == 128) {
    cfg.dynamicSmemBytes = BwdLayout<128>::kBytes;
    e = cudaLaunchKernelEx(&cfg, attn_bwd_kernel<128>, tq, tk, tv, tdo, tdq, bp);
  } else {
    cfg.dynamicSmemBytes = BwdLayout<64>::kBytes;
    e = cudaLaunchKernelEx(&cfg, attn_bwd_kernel<64>, tq, tk, tv, tdo, tdq, bp);
  }
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

  // 4. dQ = scale * accumulator in bf16
  const long long n4 = rows * s.head_dim / 4;
  attn_bwd_dq_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, strm>>>(
      bp.err, reinterpret_cast<const float4*>(dq_acc), static_cast<uint2*>(dq), n4, scale);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

// ===========================================================================
// Incoherent processing: attn_quantize_mxfp8_rotated.  The forward's and the
// backward's sources end above this line.
// ===========================================================================

extern "C" attn_status_t attn_quantize_mxfp8_rotated(const void* x, const float* signs,
                                                     uint8_t* codes, uint8_t* scales,
                                                     int64_t rows, int32_t cols, void* stream) {
  if (rows < 0 || (cols != 64 && cols != 128)) return rows < 0 ? ATTN_ERR_INVALID_ARG
                                                               : ATTN_ERR_UNSUPPORTED;
  if (rows == 0) return ATTN_OK;
  if (x == nullptr || signs == nullptr || codes == nullptr || scales == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u) != 0)
    return ATTN_ERR_ALIGNMENT;
  const long long rows_per_block = 256 / (cols / 8) * kRotRowsPerThread;
  const long long grid = (rows + rows_per_block - 1) / rows_per_block;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  if (cols == 128)
    quantize_mxfp8_rotated_kernel<128><<<static_cast<unsigned>(grid), 256, 0, strm>>>(
        static_cast<const uint4*>(x), signs, reinterpret_cast<uint2*>(codes), scales, rows);
  else
    quantize_mxfp8_rotated_kernel<64><<<static_cast<unsigned>(grid), 256, 0, strm>>>(
        static_cast<const uint4*>(x), signs, reinterpret_cast<uint2*>(codes), scales, rows);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ===========================================================================
// NVFP4 quantisation pre-pass on its own: attn_quantize_nvfp4.
// ===========================================================================

extern "C" attn_status_t attn_quantize_nvfp4(const void* x, uint8_t* codes, uint8_t* scales,
                                             int64_t rows, int32_t cols, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return ATTN_ERR_INVALID_ARG;
  if (rows == 0) return ATTN_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(codes) & 7u) != 0) return ATTN_ERR_ALIGNMENT;
  const long long n_blocks = rows * static_cast<long long>(cols / 16);
  const long long grid = (n_blocks + 255) / 256;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  quantize_nvfp4_kernel<<<static_cast<unsigned>(grid), 256, 0,
                          static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(x), reinterpret_cast<uint2*>(codes), scales, nullptr, n_blocks);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

/*
 * attn.h - C ABI of the exact tiled attention forward for NVIDIA B200
 * (sm_100a).  Library: exact_tiled_attention_39_b200/libattn.so.
 *
 * What is computed
 * ----------------
 * For every document D of a packed batch and every head h:
 *     S = scale * Q_D K_D^T            (rows: queries, columns: keys of D)
 *     S_ij = -inf  unless  (!causal || j <= i)    (indices relative to D)
 *     P = row-softmax(S),  O = P V_D,  lse_i = max_j S_ij + ln sum_j exp(S_ij - max_j S_ij)
 * "FlashAttention và IO" (aihero.vn), section "Ma trận trung gian là một
 * khoản chi phí", defines the dense computation (score matrix, softmax,
 * product with V).  Section "Tiling giữ công việc ở gần nơi tính" requires
 * that neither S nor P is ever written to device memory, and section
 * "Softmax qua nhiều khối cần thống kê chạy" gives the running statistics
 * (maximum m, normaliser l, weighted sum u, old part multiplied by
 * exp(m - m_new), result u / l) by which the kernel gets the exact result
 * tile by tile.  "FlashAttention, pelatihan multi-GPU, dan kuantisasi bobot"
 * (indonesian.itimpress.au), section 1, gives the loop order (outer loop
 * over query blocks, inner over key/value blocks), asynchronous tile copies
 * and producer / consumer warp roles.  The MXFP8 variant follows "FLAMIA:
 * Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin Flash
 * Mikro-Ölçeklemeli Dikkat Mekanizması" (blog.edumints.com), section
 * "FLAMIA Mimarisi ve Temel Tasarım İlkeleri": fused quantisation, packed
 * documents used in place, and scales that never let a future token
 * influence the past (here: one scale per token, head and 32 head-dim
 * elements).
 *
 * Layouts (all row-major, contiguous)
 * -----------------------------------
 *   q, k, v, out : bf16 [T, H, d]  (token, head, head-dim); token stride H*d.
 *   lse          : fp32 [H, T].
 *   cu_seqlens   : int32 [num_seqs + 1] in DEVICE memory: 0 = cu[0] <=
 *                  cu[1] <= ... <= cu[num_seqs] = T; document i is tokens
 *                  [cu[i], cu[i+1]).  NULL means dense: num_seqs documents
 *                  of max_seqlen tokens each, T = num_seqs * max_seqlen.
 *
 * Conventions
 * -----------
 *   - All tensor pointers are device pointers owned by the caller and must be
 *     16-byte aligned; they must stay valid until the stream work completes.
 *     The library allocates nothing and keeps no state between calls except
 *     a per-device cache of kernel attributes.
 *   - Supported: d in {64, 128}; H >= 1; T < 2^31; scale finite and > 0.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Host-checkable faults return a non-OK status
 *     before anything is launched.  Faults in the contents of cu_seqlens are
 *     found on the device: the call then records ATTN_ERR_BAD_SEQLENS in the
 *     workspace's error word and leaves out and lse untouched.  Every wait
 *     inside the kernels is bounded; if one runs out the kernel records
 *     ATTN_ERR_TIMEOUT and returns.  attn_get_device_error reads the word.
 *   - T == 0 is a no-op that returns ATTN_OK.  Empty documents are allowed.
 */
#ifndef EXACT_TILED_ATTENTION_ATTN_H
#define EXACT_TILED_ATTENTION_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_ABI_VERSION 4

typedef enum {
  ATTN_BF16 = 0,  /* bf16 operands, bf16 tensor-core products, fp32 softmax   */
  ATTN_MXFP8 = 1, /* bf16 inputs quantised in-call to E4M3 + E8M0 (per token,
                     head and 32 head-dim elements).  d = 128: Q K^T is a
                     block-scaled E4M3 product; P V runs in bf16 on the exact
                     dequantisation of V.  d = 64: every product runs in bf16
                     on the exactly dequantised Q, K and V (same values)     */
  ATTN_NVFP4 = 2  /* the mixed NVFP4 / FP8 path (forward only): bf16 inputs
                     quantised in-call, Q and K to NVFP4 (E2M1, one unsigned
                     E4M3 scale per token, head and 16 head-dim elements; see
                     attn_quantize_nvfp4), V to MXFP8.  d = 128: Q K^T is a
                     block-scaled E2M1 product; P V runs in bf16 on the
                     exact dequantisation of V.  d = 64: every product in
                     bf16 on the exactly dequantised operands             */
} attn_dtype_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* NULL pointer, negative size, bad scale, ...   */
  ATTN_ERR_UNSUPPORTED = 2,  /* head_dim or dtype not supported (also recorded
                                by a kernel that finds its shared memory
                                misaligned; never observed)                    */
  ATTN_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned              */
  ATTN_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than required       */
  ATTN_ERR_BAD_SEQLENS = 5,  /* device: cu_seqlens contents inconsistent      */
  ATTN_ERR_TIMEOUT = 6,      /* device: a bounded wait ran out                */
  ATTN_ERR_CUDA = 7          /* a CUDA runtime or driver call failed          */
} attn_status_t;

typedef struct {
  int32_t total_tokens; /* T                                                  */
  int32_t num_seqs;     /* number of documents                              */
  int32_t num_heads;    /* H                                                  */
  int32_t head_dim;     /* d                                                  */
  int32_t max_seqlen;   /* upper bound of every document length (dense: N)  */
} attn_shape_t;

/* Bytes of device workspace attn_fwd needs for this shape and dtype.  The
 * workspace holds the error word, the work list of the schedule-build step
 * and, for ATTN_MXFP8, the quantised operands.  Returns 0 for an invalid
 * shape.  Layout (for tests and tools): int32 error word at byte 0, int32
 * work-list length at byte 4, int32 unit counter at byte 8, int32 [n][4]
 * work list at byte 256, one entry (doc_start, doc_len, query_block, cost)
 * per 128-row query tile of a document, sorted by cost (key tiles needed),
 * largest first, ties in document then query-block order. */
size_t attn_workspace_size(const attn_shape_t* shape, attn_dtype_t dtype);

/* Exact attention forward.  q, k, v: bf16 [T, H, d]; out: bf16 [T, H, d];
 * lse: fp32 [H, T] (natural log, scaled-score units); causal: 0 or 1;
 * scale: the factor applied to q.k (1/sqrt(d) for standard attention).
 * Launches the schedule-build kernel, the MXFP8 quantisation kernel (dtype
 * ATTN_MXFP8 only) and the attention kernel on `stream`. */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                       void* out, float* lse, int causal, float scale, attn_dtype_t dtype,
                       void* stream, const attn_shape_t* shape, void* workspace,
                       size_t workspace_bytes);

/* The MXFP8 forward with incoherent processing ("FlashAttention, pelatihan
 * multi-GPU, dan kuantisasi bobot", section 1: FlashAttention-3 multiplies
 * Q and K by a random orthogonal matrix before FP8 quantisation, spreading
 * outlier channels over the head dimension; the scores are unchanged in
 * exact arithmetic).  Same arguments as attn_fwd with dtype ATTN_MXFP8,
 * plus signs: device fp32 [head_dim], each +1 or -1 (the caller's random
 * draw), 4-byte aligned, required when total_tokens > 0 (else
 * ATTN_ERR_INVALID_ARG).  Each row of q and k (one token of one head)
 * becomes (x * signs) H_d in fp32 (H_d the unnormalised Sylvester Hadamard
 * matrix, computed by the butterfly described at attn_quantize_mxfp8_rotated)
 * and is then quantised as by attn_quantize_mxfp8; v is quantised as it is;
 * the attention runs as for ATTN_MXFP8 with the softmax scale divided by
 * head_dim (the rotation multiplies every score by head_dim).  out and lse
 * are in the units of the unrotated problem.  Workspace: attn_workspace_size
 * of the shape with ATTN_MXFP8.  Launches the schedule-build kernel, one
 * rotating quantisation kernel for q, k and v, and the attention kernel. */
attn_status_t attn_fwd_incoherent(const void* q, const void* k, const void* v,
                                  const int32_t* cu_seqlens, void* out, float* lse, int causal,
                                  float scale, const float* signs, void* stream,
                                  const attn_shape_t* shape, void* workspace,
                                  size_t workspace_bytes);

/* attn_fwd for callers that cannot allocate device memory: a plugin or
 * custom operator that its host application hands only input and output
 * buffers, code running under a device-memory budget fixed up front by a
 * serving framework, or a latency-critical path that cannot afford the
 * implicit device synchronisation of cudaMalloc.  The pages have no
 * counterpart: this is an interface convenience, not part of the method.
 *
 * Same arguments and results as attn_fwd with dtype ATTN_BF16, minus the
 * workspace: its scratch (error word and work lists) is a 1 MiB array
 * inside the library's device image, which every GPU that loads the library
 * holds until the process exits.  Problems whose work lists need more
 * (total_tokens / 128 + num_seqs > 32751) are rejected with
 * ATTN_ERR_WORKSPACE before anything is launched.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls share the one array, and every call
 * rewrites what it reads (the error word is reset, the lists rebuilt), so
 * sequential calls are independent; calls that overlap on the GPU (other
 * streams, other host threads) race on the array and must be serialised by
 * the caller.  Device-side faults (bad cu_seqlens contents, a wait running
 * out) leave out and lse unwritten as with attn_fwd; their error word is in
 * the array and is not readable through this ABI. */
attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v,
                               const int32_t* cu_seqlens, void* out, float* lse, int causal,
                               float scale, void* stream, const attn_shape_t* shape);

/* The MXFP8 quantisation pre-pass on its own (FLAMIA section "FLAMIA
 * Mimarisi ve Temel Tasarım İlkeleri": quantisation fused into the
 * kernels).  x: bf16 [rows, cols] device, cols a multiple of 32 and of 8;
 * codes: uint8 [rows, cols] E4M3; scales: uint8 [rows, cols / 32] E8M0
 * (code c means 2^(c - 127)).  Scale rule: the smallest power of two that
 * maps the block's largest magnitude to at most 448; code clamped to
 * [0, 254]; an all-zero block gets 127.  Elements: x / 2^(c-127) rounded to
 * nearest E4M3 (ties to even, saturating at 448).  Asynchronous. */
attn_status_t attn_quantize_mxfp8(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows,
                                  int32_t cols, void* stream);

/* The NVFP4 quantisation pre-pass of the mixed NVFP4 / FP8 path on its own
 * (FLAMIA section "FLAMIA Mimarisi ve Temel Tasarım İlkeleri" names the
 * mixed path beside MXFP8).  x: bf16 [rows, cols] device, 16-byte aligned,
 * cols a multiple of 16; codes: uint8 [rows, cols / 2], 8-byte aligned, two
 * E2M1 codes per byte (element 2i in bits 0-3, 2i + 1 in bits 4-7; code =
 * sign << 3 | magnitude index of 0, 0.5, 1, 1.5, 2, 3, 4, 6); scales: uint8
 * [rows, cols / 16], unsigned E4M3 (one per 16 elements of a row).  Scale
 * rule: the smallest positive E4M3 value S with amax <= 6 S (448 past
 * 6 * 448; 1.0 for a block of zeros); no per-tensor scale.  Elements: the
 * fp32 quotient x / S (IEEE division) rounded to the nearest E2M1 value,
 * ties to even, saturating at 6, sign kept.  Asynchronous. */
attn_status_t attn_quantize_nvfp4(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows,
                                  int32_t cols, void* stream);

/* The MXFP8 pre-pass with incoherent processing ("FlashAttention, pelatihan
 * multi-GPU, dan kuantisasi bobot", section 1: Q and K multiplied by a random
 * orthogonal matrix before quantisation, to spread outlier channels).  Each
 * row r of x (bf16 [rows, cols], cols 64 or 128) becomes y = (x_r * s) H
 * with s = signs (device fp32 [cols], each +1 or -1) and H the unnormalised
 * Sylvester Hadamard matrix of order cols (H H^T = cols I), computed in fp32
 * by the fast Walsh-Hadamard butterfly (spans 1, 2, 4, ..., cols / 2; each
 * pair (a, b) -> (a + b, a - b), round to nearest); y is then quantised as by
 * attn_quantize_mxfp8.  Rotating both Q and K multiplies every score by
 * cols, so a caller divides its softmax scale by cols.  codes: uint8
 * [rows, cols] E4M3, 16-byte aligned; scales: uint8 [rows, cols / 32] E8M0,
 * 4-byte aligned.  ATTN_ERR_UNSUPPORTED for other cols.  Asynchronous. */
attn_status_t attn_quantize_mxfp8_rotated(const void* x, const float* signs, uint8_t* codes,
                                          uint8_t* scales, int64_t rows, int32_t cols,
                                          void* stream);

/* Synchronises `stream`, then reads the workspace's error word into
 * *device_status and clears it.  The word holds the outcome of the most
 * recent attn_fwd on this workspace (each call resets it when it starts):
 * ATTN_OK, ATTN_ERR_BAD_SEQLENS or ATTN_ERR_TIMEOUT.  Returns ATTN_ERR_CUDA
 * if the copy fails. */
attn_status_t attn_get_device_error(const void* workspace, void* stream,
                                    int32_t* device_status);

/* Kernel timing for benchmarks.  While enabled (process-wide), attn_fwd
 * records three CUDA events on its stream: at the start of the call, just
 * before the attention kernel and just after it.  attn_timing_read waits for
 * the events of the most recent timed call and returns, in milliseconds, the
 * attention kernel's duration and the duration of the work before it in the
 * same call (schedule build, MXFP8 pre-pass).  Recording the events ends the
 * overlap of the attention kernel's prologue with the schedule kernel, so a
 * timed call can be slightly slower than an untimed one; results are
 * unaffected.  Timed calls from several host threads at once give undefined
 * timings.  attn_timing_read returns ATTN_ERR_INVALID_ARG for null pointers
 * or when no call was timed since timing was enabled, ATTN_ERR_CUDA if the
 * events fail. */
attn_status_t attn_timing_enable(int32_t enable);
attn_status_t attn_timing_read(float* attention_ms, float* prepass_ms);

/* Bytes of device workspace attn_bwd needs for this shape and dtype (0 for
 * an invalid shape or dtype): the error word and work lists as for
 * attn_fwd, then D (fp32 [H, T]) and the fp32 dQ accumulator ([T, H, d]);
 * for ATTN_MXFP8 also the exactly dequantised q, k, v and dout (bf16
 * [T, H, d] each). */
size_t attn_bwd_workspace_size(const attn_shape_t* shape, attn_dtype_t dtype);

/* Exact attention backward: the gradients of attn_fwd's output with respect
 * to q, k and v, given the upstream gradient dout.  The pages print no
 * backward formulas (FLAMIA, section "Performans Sonuçları", measures forward
 * and backward together); these are the derivatives of the definition
 * above, per document and head, with P recomputed from the saved lse:
 *     P = exp(scale S - lse),  dV = P^T dO,  dP = dO V^T,
 *     D_i = dO_i . O_i,  dS = P * (dP - D),
 *     dQ = scale dS K,  dK = scale dS^T Q.
 * q, k, v, out, dout: bf16 [T, H, d] (out and lse as attn_fwd wrote them for
 * the same q, k, v, cu_seqlens, causal and scale); lse: fp32 [H, T];
 * dq, dk, dv: bf16 [T, H, d], written.  Same cu_seqlens, shape and causal
 * rules as attn_fwd; head dim 64 or 128.
 * dtype ATTN_MXFP8 is the backward of attn_fwd's MXFP8 path (FLAMIA,
 * section "FLAMIA Mimarisi ve Temel Tasarım İlkeleri": forward and
 * backward numerically consistent, quantised operands reused across matrix
 * orientations, no scale covering a future token): q, k, v and dout are
 * quantised per token, head and 32 head-dim elements exactly as the forward
 * quantises q, k, v, and the gradients are those of the attention on the
 * exactly dequantised operands (passed straight through the quantiser);
 * out and lse must come from the MXFP8 forward.  One quantisation of each
 * operand serves every product and orientation.
 * Launches the schedule-build kernel, for ATTN_MXFP8 one quantisation
 * kernel for q, k, v and dout, a kernel computing D and clearing the
 * accumulator, the backward kernel (one
 * 128-key tile of a document and head per work unit; dK and dV accumulate
 * on chip, dQ through fp32 vector reductions, so dq is not bit-reproducible
 * across calls) and the kernel that scales and rounds dQ.  Device faults
 * (bad cu_seqlens, a wait running out) are recorded in the workspace's error
 * word as for attn_fwd and leave dq unwritten. */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, const int32_t* cu_seqlens, void* dq,
                       void* dk, void* dv, int causal, float scale, attn_dtype_t dtype,
                       void* stream, const attn_shape_t* shape, void* workspace,
                       size_t workspace_bytes);

/* Static, human-readable name of a status code. */
const char* attn_status_string(attn_status_t status);

/* ATTN_ABI_VERSION of the built library. */
int32_t attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_TILED_ATTENTION_ATTN_H */

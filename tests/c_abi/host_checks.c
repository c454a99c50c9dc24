/* A plain C99 client of include/attn.h: the library links and loads from C
 * and its host-side paths answer as the header documents.  No call here
 * reaches a kernel (every case is rejected, or is a no-op, before anything
 * is launched), so it runs without a GPU.  Exit status 0 = all checks hold;
 * otherwise the number of the first failing check. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "attn.h"

static int failed = 0;
static int check_no = 0;

static void check(int cond, const char* what) {
  ++check_no;
  if (!cond && failed == 0) {
    failed = check_no;
    fprintf(stderr, "check %d failed: %s\n", check_no, what);
  }
}

static attn_shape_t shape(int32_t T, int32_t n, int32_t H, int32_t d, int32_t L) {
  attn_shape_t s;
  s.total_tokens = T;
  s.num_seqs = n;
  s.num_heads = H;
  s.head_dim = d;
  s.max_seqlen = L;
  return s;
}

int main(void) {
  /* any 16-byte aligned, non-null address: never dereferenced on these paths */
  void* const p16 = (void*)(uintptr_t)16;
  void* const p24 = (void*)(uintptr_t)24;
  const attn_shape_t ok = shape(256, 1, 2, 64, 256);
  const attn_shape_t bad_d = shape(256, 1, 2, 96, 256);
  const attn_shape_t dense_mismatch = shape(256, 2, 2, 64, 100);
  const attn_shape_t empty = shape(0, 0, 2, 64, 0);
  const attn_shape_t big = shape(16384, 7, 32, 128, 4096);

  check(attn_abi_version() == ATTN_ABI_VERSION, "abi version");
  check(strcmp(attn_status_string(ATTN_OK), "ATTN_OK") == 0, "status string OK");
  check(strcmp(attn_status_string(ATTN_ERR_TIMEOUT), "ATTN_ERR_TIMEOUT") == 0,
        "status string TIMEOUT");

  /* workspace sizes */
  check(attn_workspace_size(&big, ATTN_BF16) >= 256 + 2 * 16 * (16384 / 128 + 7 + 1),
        "forward workspace holds the work lists");
  check(attn_workspace_size(&big, ATTN_MXFP8) > attn_workspace_size(&big, ATTN_BF16),
        "MXFP8 workspace holds the quantised operands");
  check(attn_workspace_size(&bad_d, ATTN_BF16) == 0, "unsupported head dim: size 0");
  check(attn_bwd_workspace_size(&big, ATTN_BF16) >=
            (size_t)16384 * 32 * 4 + (size_t)16384 * 32 * 128 * 4,
        "backward workspace holds D and the dQ accumulator");
  check(attn_bwd_workspace_size(&big, ATTN_MXFP8) >=
            attn_bwd_workspace_size(&big, ATTN_BF16) + (size_t)4 * 2 * 16384 * 32 * 128,
        "MXFP8 backward workspace holds the dequantised operands");
  check(attn_bwd_workspace_size(&bad_d, ATTN_BF16) == 0,
        "backward: unsupported head dim: size 0");

  /* forward: rejected before launch */
  check(attn_fwd(p16, p16, p16, NULL, p16, (float*)p16, 1, 0.125f, ATTN_BF16, NULL, NULL, p16,
                 1 << 20) == ATTN_ERR_INVALID_ARG, "forward: NULL shape");
  check(attn_fwd(p16, p16, p16, NULL, p16, (float*)p16, 1, 0.125f, ATTN_BF16, NULL, &bad_d,
                 p16, 1 << 20) == ATTN_ERR_UNSUPPORTED, "forward: head dim 96");
  check(attn_fwd(p16, p16, p16, NULL, p16, (float*)p16, 1, -1.0f, ATTN_BF16, NULL, &ok, p16,
                 1 << 20) == ATTN_ERR_INVALID_ARG, "forward: negative scale");
  check(attn_fwd(p16, p16, p16, NULL, p16, (float*)p16, 1, 0.125f, ATTN_BF16, NULL,
                 &dense_mismatch, p16, 1 << 20) == ATTN_ERR_INVALID_ARG,
        "forward: dense T != B * N");
  check(attn_fwd(p16, p24, p16, NULL, p16, (float*)p16, 1, 0.125f, ATTN_BF16, NULL, &ok, p16,
                 1 << 20) == ATTN_ERR_ALIGNMENT, "forward: misaligned k");
  check(attn_fwd(p16, p16, p16, NULL, p16, (float*)p16, 1, 0.125f, ATTN_BF16, NULL, &ok, p16,
                 8) == ATTN_ERR_WORKSPACE, "forward: workspace too small");
  check(attn_fwd(NULL, NULL, NULL, NULL, NULL, NULL, 1, 0.125f, ATTN_BF16, NULL, &empty, NULL,
                 0) == ATTN_OK, "forward: T == 0 is a no-op");

  /* backward: rejected before launch */
  check(attn_bwd(p16, p16, p16, p16, p16, (const float*)p16, NULL, p16, p16, p16, 1, 0.125f,
                 (attn_dtype_t)7, NULL, &ok, p16, (size_t)1 << 30) == ATTN_ERR_UNSUPPORTED,
        "backward: unknown dtype");
  check(attn_bwd(p16, p16, p16, p16, p16, (const float*)p16, NULL, p16, p16, p16, 1, 0.125f,
                 ATTN_MXFP8, NULL, &ok, p16, attn_bwd_workspace_size(&ok, ATTN_BF16)) ==
            ATTN_ERR_WORKSPACE,
        "backward: MXFP8 workspace holds more than the bf16 one");
  check(attn_bwd(p16, p16, p16, p16, NULL, (const float*)p16, NULL, p16, p16, p16, 1, 0.125f,
                 ATTN_BF16, NULL, &ok, p16, (size_t)1 << 30) == ATTN_ERR_INVALID_ARG,
        "backward: NULL dout");
  check(attn_bwd(p16, p16, p16, p16, p16, (const float*)p16, NULL, p24, p16, p16, 1, 0.125f,
                 ATTN_BF16, NULL, &ok, p16, (size_t)1 << 30) == ATTN_ERR_ALIGNMENT,
        "backward: misaligned dq");
  check(attn_bwd(p16, p16, p16, p16, p16, (const float*)p16, NULL, p16, p16, p16, 1, 0.125f,
                 ATTN_BF16, NULL, &ok, p16, 64) == ATTN_ERR_WORKSPACE,
        "backward: workspace too small");
  check(attn_bwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 0.125f,
                 ATTN_BF16, NULL, &empty, NULL, 0) == ATTN_OK, "backward: T == 0 is a no-op");

  /* quantiser */
  check(attn_quantize_mxfp8(NULL, NULL, NULL, 4, 48, NULL) == ATTN_ERR_INVALID_ARG,
        "quantiser: cols not a multiple of 32");
  check(attn_quantize_mxfp8(NULL, NULL, NULL, 0, 64, NULL) == ATTN_OK, "quantiser: empty");
  check(attn_fwd_incoherent(p16, p16, p16, NULL, p16, (float*)p16, 1, 0.125f, NULL, NULL, &ok,
                            p16, (size_t)1 << 26) == ATTN_ERR_INVALID_ARG,
        "incoherent forward: signs required");
  check(attn_fwd_incoherent(NULL, NULL, NULL, NULL, NULL, NULL, 1, 0.125f, NULL, NULL, &empty,
                            NULL, 0) == ATTN_OK,
        "incoherent forward: empty problem is a no-op");

  if (failed == 0) printf("c abi host checks: %d ok\n", check_no);
  return failed;
}

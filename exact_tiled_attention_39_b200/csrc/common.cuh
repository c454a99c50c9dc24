// Constants shared by the host launcher and the device kernels.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/attn.h"

namespace attn {

constexpr int kBlockM = 128;        // query rows per tile (one TMEM lane per row)
constexpr int kBlockN = 128;        // keys per key/value tile
// Work units are 1 query tile (MXFP8 kernel) or 2 (bf16 kernel); the list
// is sized for the finer granularity.
constexpr int kRowsPerUnit = kBlockM;

// Workspace layout: a 256-byte header, then the work list.
constexpr size_t kWsErrorOffset = 0;     // int32 error word (attn_status_t)
constexpr size_t kWsCountOffset = 4;     // int32 number of work-list entries
constexpr size_t kWsUnitCounterOffset = 8;   // int32 dynamic unit counter (reset per call)
constexpr size_t kWsListOffset = 256;    // int4 entries
constexpr size_t kWsAlign = 256;

// Lazy rescaling threshold in log2 units: the output accumulator keeps a
// stale maximum until the row maximum has grown by more than this, so the
// unnormalised weights stay below 2^kRescaleTau.
constexpr float kRescaleTau = 8.0f;

// Unit order: heads are taken in groups whose K and V fit this much of the
// L2 (126 MB, split between the two dies), and all units of one group run
// before the next group's, heaviest first within the group.  Query tiles of
// one (document, head) then run at about the same time and each K/V tile is
// fetched from HBM about once instead of once per query tile.
constexpr double kL2HeadGroupBytes = 40.0 * 1024 * 1024;

// Number of head groups for a launch: heads per group from the budget above
// (K bytes + V bytes per head over all tokens), groups as equal as possible.
inline int head_group_count(int64_t total_tokens, int num_heads, int head_dim, int kv_elem_bytes) {
  const double per_head = static_cast<double>(total_tokens) * head_dim * kv_elem_bytes;
  int g_max = per_head > 0 ? static_cast<int>(kL2HeadGroupBytes / per_head) : num_heads;
  if (g_max < 1) g_max = 1;
  if (g_max > num_heads) g_max = num_heads;
  return (num_heads + g_max - 1) / g_max;
}

// Upper bound of the work-list length: every document contributes
// ceil(L / 128) <= L / 128 + 1 entries.
inline int64_t max_work_entries(int64_t total_tokens, int64_t num_seqs) {
  return total_tokens / kRowsPerUnit + num_seqs + 1;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace attn

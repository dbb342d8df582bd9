// Internal types shared by the host planner, the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <vector>

#include "../../include/mla.h"

namespace mla {

constexpr int kLatent = 576;   // ckv 512 | kpe 64
constexpr int kCkv = 512;
constexpr int kRope = 64;
constexpr int kTileM = 128;    // query rows per tile (tokens x heads)
constexpr int kTileN = MLA_KEY_TILE;  // keys per tile (64)
// Split-KV workspace per partial: the 128 x 512 output tile in bf16, then its 128 fp32
// log-sum-exps (all partials' tiles first, then all their lse rows).
constexpr size_t kPartialOBytes = size_t(kTileM) * kCkv * 2;
constexpr size_t kPartialBytes = kPartialOBytes + size_t(kTileM) * 4;

// One unit of attention work: a 128-row query tile against keys [key_begin, key_end)
// of one batch row.  Processed by one CTA pair; field order matches mla_plan_describe.
struct WorkItem {
  int32_t q_row0;     // first (token * H + head) row of the query tile
  int32_t n_rows;     // valid rows in the tile (tokens_in_tile * H)
  int32_t page_base;  // kv_indptr[b]: the row's first entry in kv_indices
  int32_t kv_len;     // k_b
  int32_t key_begin;  // multiple of kTileN
  int32_t key_end;    // exclusive
  int32_t diag_base;  // row r sees keys < clamp(diag_base + r / H + 1, 0, kv_len)
  int32_t partial;    // -1: final output; else workspace slot
};
static_assert(sizeof(WorkItem) == 4 * MLA_WORK_FIELDS, "WorkItem layout");

// A query tile whose keys were split: combine partials [first, first + n).
struct MergeItem {
  int32_t q_row0;
  int32_t n_rows;
  int32_t first_partial;
  int32_t n_partials;
};
static_assert(sizeof(MergeItem) == 4 * MLA_MERGE_FIELDS, "MergeItem layout");

struct PlanLayout {
  std::vector<int32_t> kv_len;
  std::vector<WorkItem> work;
  std::vector<MergeItem> merge;
  int32_t num_partials = 0;
  int32_t total_tokens = 0;
  int32_t chunk_tiles = 0;  // chosen split size in 64-key tiles (0: no split)
};

// Validate the step's tables and build the work and merge lists (host only).
mla_status build_layout(const mla_dims& d, int32_t batch, const int32_t* qo_indptr,
                        const int32_t* kv_indptr, const int32_t* kv_indices,
                        const int32_t* last_page_len, bool causal, int32_t split_keys,
                        int32_t num_sms, PlanLayout* out);

bool shape_supported(int kv_lora_rank, int rope_dim, int num_heads, int page_size);

}  // namespace mla

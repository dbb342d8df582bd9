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
// Split-KV workspace, addressed by row: each partial result occupies as many rows as
// its query tile.  All rows' bf16 outputs (512 wide) come first, then all their fp32
// log-sum-exps.
constexpr size_t kWsRowOBytes = size_t(kCkv) * 2;
constexpr size_t kWsRowBytes = kWsRowOBytes + 4;

// One unit of attention work: a query tile of up to 128 rows against keys
// [key_begin, key_end).  Processed by one CTA pair; field order matches
// mla_plan_describe.  n_rows == 0 marks an empty launch slot of a graph plan.
struct WorkItem {
  int32_t q_row0;     // first (token * H + head) row of the query tile
  int32_t n_rows;     // valid rows in the tile
  int32_t page_base;  // kv_indptr entry of the pages the item reads
  int32_t kv_len;     // keys addressable from page_base
  int32_t key_begin;  // multiple of kTileN
  int32_t key_end;    // exclusive
  int32_t diag_base;  // row r sees keys < clamp(diag_base + r / H + 1, 0, kv_len)
  int32_t partial;    // -1: final output; else first workspace row of the partial
};
static_assert(sizeof(WorkItem) == 4 * MLA_WORK_FIELDS, "WorkItem layout");

// Output rows [q_row0, q_row0 + n_rows) combine n_refs partial results; partial i
// holds the tile's row r in workspace row refs[first_ref + i] + r.
struct MergeItem {
  int32_t q_row0;
  int32_t n_rows;
  int32_t first_ref;
  int32_t n_refs;
};
static_assert(sizeof(MergeItem) == 4 * MLA_MERGE_FIELDS, "MergeItem layout");

// What the planner is asked to plan.
struct PlanRequest {
  mla_dims d{};
  int32_t batch = 0;
  const int32_t* qo_indptr = nullptr;
  const int32_t* kv_indptr = nullptr;
  const int32_t* kv_indices = nullptr;
  const int32_t* last_page_len = nullptr;
  bool causal = true;
  bool context_only = false;
  bool cascade = false;
  int32_t split_keys = 0;
  int32_t num_sms = 148;
  // Upper bounds for a graph plan (0: unbounded).  The planner keeps the split-KV
  // choice within them.
  int32_t max_work = 0;
  int32_t max_merge = 0;
  int32_t max_refs = 0;
  int32_t max_ws_rows = 0;
};

struct PlanLayout {
  std::vector<int32_t> kv_len;       // per row: keys attended (k_b, or c_b context-only)
  std::vector<WorkItem> work;
  std::vector<MergeItem> merge;
  std::vector<int32_t> refs;         // merge reference list
  std::vector<int32_t> append_rows;  // per token: destination cache row, -1 if none
  bool append_ok = true;             // every token has a slot
  int32_t num_partials = 0;
  int32_t ws_rows = 0;               // workspace rows in use
  int32_t num_cascade = 0;           // prefix items of cascaded row groups
  int32_t total_tokens = 0;
  int32_t chunk_tiles = 0;  // chosen split size in 64-key tiles (0: no split)
};

// Planner cost model, in units of one key tile step of a CTA pair: the fixed work of a
// work item (query load, pipeline fill and drain, epilogue), and the extra of an item
// whose result is a partial (its write and the merge pass that reads it back).
constexpr double kItemCost = 3.0;
constexpr double kSplitCost = 2.0;
// Split choice: the largest number of waves of SM pairs a split may fill.
constexpr int kMaxWaves = 6;
// When every item has an SM pair to itself, a split step lasts its longest item plus the
// merge launch that follows (about one key tile step).
constexpr double kMergeLatency = 1.0;

// Validate the step's tables and build the work and merge lists (host only).
mla_status build_layout(const PlanRequest& req, PlanLayout* out);

// Bounds of a graph plan for a bucket of `max_batch` rows and `max_tokens` tokens.
void graph_bounds(int32_t num_heads, int32_t max_batch, int32_t max_tokens, int32_t num_sms, PlanRequest* req);

bool shape_supported(int kv_lora_rank, int rope_dim, int num_heads, int page_size);

}  // namespace mla

// Host planner: validates one step's page tables and cuts the attention into work
// items (128-row query tiles x key chunks) balanced across the GPU's SM pairs.
//
// Page "mstar.engine.resources.attn.flashinfer_mla": FlashInferMLAWrapper.plan takes
// qo_indptr, paged_kv_indptr, paged_kv_indices and paged_kv_last_page_len, built on
// the host; FlashInferMLAManager.kv_len_buf exposes the planned per-row key counts.
// Long key ranges are split into chunks whose partial results are merged by their
// log-sum-exp (FlashInferMLAManager.run: the lse exists to merge key segments).
#include <algorithm>
#include <cmath>
#include <functional>
#include <limits>
#include <queue>

#include "mla_internal.h"

namespace mla {

bool shape_supported(int kv_lora_rank, int rope_dim, int num_heads, int page_size) {
  if (kv_lora_rank != kCkv || rope_dim != kRope) return false;
  if (num_heads != 16 && num_heads != 32 && num_heads != 64 && num_heads != 128) return false;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128) return false;
  return true;
}

namespace {

// A query tile before key splitting.
struct QTile {
  int32_t q_row0, n_rows, page_base, kv_len, diag_base, vis_hi, ntiles;
};

// Cost, in units of one key tile step, of the fixed work of one item: query load,
// pipeline fill/drain and epilogue.  Split items also write an fp32 partial that the
// merge kernel reads back.
constexpr double kItemCost = 3.0;
constexpr double kSplitCost = 2.0;

// Longest-processing-time-first makespan of `costs` over `units` identical units.
double lpt_makespan(std::vector<double> costs, int units) {
  std::sort(costs.begin(), costs.end(), std::greater<double>());
  std::priority_queue<double, std::vector<double>, std::greater<double>> load;
  for (int i = 0; i < units; ++i) load.push(0.0);
  double worst = 0.0;
  for (double c : costs) {
    double l = load.top();
    load.pop();
    l += c;
    worst = std::max(worst, l);
    load.push(l);
  }
  return worst;
}

// Split a tile of `ntiles` key tiles into pieces of at most `chunk` tiles, sizes
// differing by at most one.  Returns the number of pieces.
inline int32_t pieces_for(int32_t ntiles, int32_t chunk) {
  if (ntiles <= 0) return 1;
  if (chunk <= 0) return 1;
  return (ntiles + chunk - 1) / chunk;
}

double estimate(const std::vector<QTile>& tiles, int32_t chunk, int units) {
  std::vector<double> costs;
  costs.reserve(tiles.size() * 2);
  int64_t partials = 0;
  for (const QTile& t : tiles) {
    int32_t n = pieces_for(t.ntiles, chunk);
    if (n == 1) {
      costs.push_back(t.ntiles + kItemCost);
    } else {
      partials += n;
      for (int32_t p = 0; p < n; ++p) {
        int32_t lo = (int64_t)t.ntiles * p / n, hi = (int64_t)t.ntiles * (p + 1) / n;
        costs.push_back((hi - lo) + kItemCost + kSplitCost);
      }
    }
  }
  // The merge pass reads every partial once, spread over all units.
  return lpt_makespan(costs, units) + kSplitCost * double(partials) / units;
}

}  // namespace

mla_status build_layout(const mla_dims& d, int32_t batch, const int32_t* qo_indptr,
                        const int32_t* kv_indptr, const int32_t* kv_indices,
                        const int32_t* last_page_len, bool causal, int32_t split_keys,
                        int32_t num_sms, PlanLayout* out) {
  if (!out) return MLA_ERR_INVALID_ARGUMENT;
  if (!shape_supported(d.kv_lora_rank, d.rope_dim, d.num_heads, d.page_size))
    return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || d.num_pages < 1 || !std::isfinite(d.sm_scale) || !(d.sm_scale > 0.f))
    return MLA_ERR_INVALID_ARGUMENT;
  if (!qo_indptr || !kv_indptr || (batch > 0 && !last_page_len)) return MLA_ERR_INVALID_ARGUMENT;
  if (split_keys > 0 && split_keys % kTileN != 0) return MLA_ERR_INVALID_ARGUMENT;
  const int32_t H = d.num_heads, P = d.page_size;
  if ((int64_t)d.num_pages * P > std::numeric_limits<int32_t>::max())
    return MLA_ERR_INVALID_ARGUMENT;

  // --- indptr tables
  if (qo_indptr[0] != 0 || kv_indptr[0] != 0) return MLA_ERR_INVALID_ARGUMENT;
  for (int32_t b = 0; b < batch; ++b) {
    if (qo_indptr[b + 1] < qo_indptr[b] || kv_indptr[b + 1] < kv_indptr[b])
      return MLA_ERR_INVALID_ARGUMENT;
  }
  const int64_t T = qo_indptr[batch];
  const int64_t n_idx = kv_indptr[batch];
  if (T * H > std::numeric_limits<int32_t>::max() - kTileM) return MLA_ERR_INVALID_ARGUMENT;
  if (n_idx > 0 && !kv_indices) return MLA_ERR_INVALID_ARGUMENT;
  for (int64_t i = 0; i < n_idx; ++i)
    if (kv_indices[i] < 0 || kv_indices[i] >= d.num_pages) return MLA_ERR_INVALID_ARGUMENT;

  // --- per-row key counts
  out->kv_len.assign(batch, 0);
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = kv_indptr[b + 1] - kv_indptr[b];
    const int32_t last = last_page_len[b];
    if (n > 0) {
      if (last < 1 || last > P) return MLA_ERR_INVALID_ARGUMENT;
      const int64_t k = (n - 1) * P + last;
      if (k > std::numeric_limits<int32_t>::max() - kTileN) return MLA_ERR_INVALID_ARGUMENT;
      out->kv_len[b] = static_cast<int32_t>(k);
    } else {
      if (last < 0 || last > P) return MLA_ERR_INVALID_ARGUMENT;
    }
  }
  out->total_tokens = static_cast<int32_t>(T);

  // --- query tiles: 128 / H consecutive tokens of one row, all heads
  const int32_t tok_per_tile = kTileM / H;
  std::vector<QTile> tiles;
  int64_t total_key_tiles = 0;
  int32_t max_ntiles = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t q_b = qo_indptr[b + 1] - qo_indptr[b];
    const int32_t k_b = out->kv_len[b];
    for (int32_t tok0 = 0; tok0 < q_b; tok0 += tok_per_tile) {
      const int32_t ntok = std::min(tok_per_tile, q_b - tok0);
      QTile t;
      t.q_row0 = (qo_indptr[b] + tok0) * H;
      t.n_rows = ntok * H;
      t.page_base = kv_indptr[b];
      t.kv_len = k_b;
      // causal: token i sees keys < k_b - q_b + i + 1; non-causal: all k_b keys
      t.diag_base = causal ? (k_b - q_b + tok0) : k_b;
      const int64_t hi = causal ? (int64_t)t.diag_base + ntok : (int64_t)k_b;
      t.vis_hi = static_cast<int32_t>(std::max<int64_t>(0, std::min<int64_t>(hi, k_b)));
      t.ntiles = (t.vis_hi + kTileN - 1) / kTileN;
      total_key_tiles += t.ntiles;
      max_ntiles = std::max(max_ntiles, t.ntiles);
      tiles.push_back(t);
    }
  }

  // --- choose the split size
  const int units = std::max(1, num_sms / 2);
  int32_t chunk = 0;  // 0: no split
  if (split_keys > 0) {
    chunk = split_keys / kTileN;
  } else if (split_keys == 0 && !tiles.empty() && max_ntiles > 1) {
    double best = estimate(tiles, 0, units);
    const double avg = (double(total_key_tiles) + kItemCost * tiles.size()) / units;
    std::vector<int32_t> cands;
    for (int32_t dv = 2; dv <= 64; ++dv) cands.push_back((max_ntiles + dv - 1) / dv);
    for (double f : {1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 8.0}) cands.push_back((int32_t)std::ceil(avg / f));
    std::sort(cands.begin(), cands.end(), std::greater<int32_t>());
    cands.erase(std::unique(cands.begin(), cands.end()), cands.end());
    for (int32_t c : cands) {
      if (c < 2 || c >= max_ntiles) continue;
      const double e = estimate(tiles, c, units);
      if (e < best * 0.99) {  // prefer fewer splits unless clearly better
        best = e;
        chunk = c;
      }
    }
  }
  out->chunk_tiles = chunk;

  // --- emit items (longest first) and merge records
  out->work.clear();
  out->merge.clear();
  int32_t partial = 0;
  for (const QTile& t : tiles) {
    const int32_t n = chunk > 0 ? pieces_for(t.ntiles, chunk) : 1;
    if (n == 1) {
      out->work.push_back(
          WorkItem{t.q_row0, t.n_rows, t.page_base, t.kv_len, 0, t.vis_hi, t.diag_base, -1});
      continue;
    }
    out->merge.push_back(MergeItem{t.q_row0, t.n_rows, partial, n});
    for (int32_t p = 0; p < n; ++p) {
      const int32_t lo = (int64_t)t.ntiles * p / n, hi = (int64_t)t.ntiles * (p + 1) / n;
      WorkItem w{t.q_row0, t.n_rows, t.page_base, t.kv_len, lo * kTileN,
                 std::min(hi * kTileN, t.vis_hi), t.diag_base, partial + p};
      out->work.push_back(w);
    }
    partial += n;
  }
  out->num_partials = partial;
  std::stable_sort(out->work.begin(), out->work.end(), [](const WorkItem& a, const WorkItem& b) {
    return (a.key_end - a.key_begin) > (b.key_end - b.key_begin);
  });
  return MLA_OK;
}

}  // namespace mla

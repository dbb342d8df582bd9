// Host planner: validates one step's page tables and cuts the attention into work
// items (query tiles of up to 128 rows x key chunks) balanced across the GPU's SM pairs.
//
// Page "mstar.engine.resources.attn.flashinfer_mla": FlashInferMLAWrapper.plan takes
// qo_indptr, paged_kv_indptr, paged_kv_indices and paged_kv_last_page_len, built on
// the host; FlashInferMLAManager.kv_len_buf exposes the planned per-row key counts
// (the stored context for a context-only plan).  Long key ranges are split into chunks
// whose partial results are merged by their log-sum-exp (FlashInferMLAManager.run: the
// lse exists to merge key segments).  Page "mstar.engine.resources.attn.base",
// captured_page_capacity: rows that matched one cached prefix all name its pages, which
// the cascade option exploits by attending such a prefix once per group of rows.
#include <algorithm>
#include <cmath>
#include <limits>

#include "mla_internal.h"

namespace mla {

bool shape_supported(int kv_lora_rank, int rope_dim, int num_heads, int page_size) {
  // ckv 512 with kpe 64 or 0 (flashinfer_mla_supports: "ckv 512, kpe 0 or 64")
  if (kv_lora_rank != kCkv || (rope_dim != kRope && rope_dim != 0)) return false;
  if (num_heads != 16 && num_heads != 32 && num_heads != 64 && num_heads != 128) return false;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128) return false;
  return true;
}

void graph_bounds(int32_t num_heads, int32_t max_batch, int32_t max_tokens, int32_t num_sms, PlanRequest* req) {
  const int64_t H = std::max(1, num_heads);
  // a row's tiles hold 128 / H tokens; each row adds at most one partial tile
  const int64_t tiles =
      std::min<int64_t>(max_tokens, (int64_t(max_tokens) * H + kTileM - 1) / kTileM + max_batch);
  const int64_t units = std::max(1, num_sms / 2);
  // cascade prefix items at most double the tiles; splitting adds up to 4 items per unit
  const int64_t work = 2 * tiles + 4 * units;
  req->max_work = static_cast<int32_t>(std::min<int64_t>(work, 1 << 24));
  req->max_merge = static_cast<int32_t>(std::min<int64_t>(2 * tiles, 1 << 24));
  req->max_refs = static_cast<int32_t>(std::min<int64_t>(8 * work, 1 << 26));
  req->max_ws_rows = static_cast<int32_t>(std::min<int64_t>(int64_t(kTileM) * work, 1 << 28));
}

namespace {

// A query tile before key splitting.  Output tiles hold 128 / H consecutive tokens of
// one row; cascade tiles pack consecutive output tiles of a row group.
struct QTile {
  int32_t q_row0, n_rows, page_base, kv_len, diag_base;
  int32_t key0;    // first key (a multiple of kTileN)
  int32_t vis_hi;  // keys < vis_hi may be visible to some row
  int32_t ntiles;  // key tiles in [key0, vis_hi)
  bool must_merge; // its result is a partial even when unsplit
  bool cascade;    // a shared-prefix tile of a row group
  int32_t out_tile;  // output tile index (non-cascade tiles)
  int32_t first_out, n_out;  // output tiles covered (cascade tiles)
};

// Item costs are whole numbers of key-tile steps: a piece's key tiles plus the fixed
// cost of an item, plus the extra of a partial result.
constexpr int32_t kItemCostI = static_cast<int32_t>(kItemCost);
constexpr int32_t kSplitCostI = static_cast<int32_t>(kSplitCost);
static_assert(double(kItemCostI) == kItemCost && double(kSplitCostI) == kSplitCost, "integer item costs");

// Pieces of at most `chunk` key tiles (sizes differing by at most one).
inline int32_t pieces_for(int32_t ntiles, int32_t chunk) {
  if (ntiles <= 0) return 1;
  if (chunk <= 0) return 1;
  return (ntiles + chunk - 1) / chunk;
}

// ceil(ntiles / chunk) for 1 <= chunk, 0 <= ntiles < 2^24, from a float reciprocal
// (one multiply, corrected to the exact quotient) instead of an integer division.
struct PieceCounter {
  int32_t chunk;
  float inv;
  explicit PieceCounter(int32_t c) : chunk(c), inv(1.0f / float(c)) {}
  int32_t operator()(int32_t ntiles) const {
    if (ntiles <= 0) return 1;
    int32_t n = static_cast<int32_t>(float(ntiles) * inv);  // within one of ntiles / chunk
    while (n * chunk < ntiles) ++n;
    while (n > 1 && (n - 1) * chunk >= ntiles) --n;
    return n;
  }
};

// What a split size makes of the tiles, in one pass.
struct SplitStats {
  int64_t items = 0, partials = 0, ws_rows = 0;
  int64_t total_cost = 0;  // sum of item costs
  int32_t longest = 0;     // largest item cost
};

SplitStats stats_for(const std::vector<QTile>& tiles, int32_t chunk) {
  SplitStats st;
  if (chunk <= 0) {  // no split: one item per tile
    for (const QTile& t : tiles) {
      const int32_t fixed = kItemCostI + (t.must_merge ? kSplitCostI : 0);
      st.items += 1;
      st.total_cost += int64_t(t.ntiles) + fixed;
      st.longest = std::max(st.longest, t.ntiles + fixed);
      if (t.must_merge) {
        st.partials += 1;
        st.ws_rows += t.n_rows;
      }
    }
    return st;
  }
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    const bool part = n > 1 || t.must_merge;
    const int32_t fixed = kItemCostI + (part ? kSplitCostI : 0);
    st.items += n;
    st.total_cost += int64_t(t.ntiles) + int64_t(n) * fixed;
    st.longest = std::max(st.longest, (t.ntiles + n - 1) / n + fixed);
    if (part) {
      st.partials += n;
      st.ws_rows += int64_t(n) * t.n_rows;
    }
  }
  return st;
}

// The tiles counted by their number of key tiles, so that what a split size makes of
// them is evaluated in time proportional to (longest tile / chunk) rather than to the
// number of tiles.  Valid when no tile must merge (no cascade prefixes): then a tile's
// pieces are partials exactly when it is cut.
struct TileCounts {
  int32_t max_nt = 0;
  int64_t n = 0, sum_nt = 0;
  std::vector<int64_t> gt;     // gt[x]: tiles with more than x key tiles, x in [0, max_nt]
  std::vector<int32_t> le_max; // le_max[x]: the largest tile length <= x (-1 if none)

  void build(const std::vector<QTile>& tiles, int32_t max_ntiles) {
    max_nt = max_ntiles;
    n = static_cast<int64_t>(tiles.size());
    sum_nt = 0;
    gt.assign(static_cast<size_t>(max_nt) + 2, 0);
    le_max.assign(static_cast<size_t>(max_nt) + 1, -1);
    for (const QTile& t : tiles) {
      sum_nt += t.ntiles;
      ++gt[t.ntiles];  // first the count of each length
      le_max[t.ntiles] = t.ntiles;
    }
    int64_t above = 0;
    for (int32_t x = max_nt; x >= 0; --x) {  // then suffix sums: tiles longer than x
      const int64_t eq = gt[x];
      gt[x] = above;
      above += eq;
    }
    for (int32_t x = 1; x <= max_nt; ++x) le_max[x] = std::max(le_max[x], le_max[x - 1]);
  }
  // sum over j >= 1 of the tiles longer than j * c
  int64_t cut_sum(int32_t c) const {
    int64_t s = 0;
    for (int64_t x = c; x <= max_nt; x += c) s += gt[x];
    return s;
  }
  int64_t items(int32_t c) const { return n + cut_sum(c); }
  SplitStats stats(int32_t c) const {
    SplitStats st;
    const int64_t cuts = cut_sum(c);
    st.items = n + cuts;
    st.partials = gt[c] + cuts;  // the pieces of the tiles longer than c
    st.total_cost = sum_nt + kItemCostI * st.items + kSplitCostI * st.partials;
    // a lower bound on the longest item: the longest uncut tile, and a piece of the
    // longest tile if that one is cut
    int32_t longest = le_max[std::min(c, max_nt)] >= 0 ? le_max[std::min(c, max_nt)] + kItemCostI : 0;
    if (max_nt > c) {
      const int32_t pieces = (max_nt + c - 1) / c;
      longest = std::max(longest, (max_nt + pieces - 1) / pieces + kItemCostI + kSplitCostI);
    }
    st.longest = longest;
    return st;
  }
};

struct Counts {
  int64_t work = 0, merge = 0, refs = 0, ws_rows = 0, partials = 0;
};

// Items, merge records, references and workspace rows a split size produces.
Counts count_for(const std::vector<QTile>& tiles, int32_t n_out, int32_t chunk) {
  Counts c;
  std::vector<int64_t> refs_of(n_out, 0);
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    c.work += n;
    if (n == 1 && !t.must_merge) continue;
    c.partials += n;
    c.ws_rows += int64_t(n) * t.n_rows;
    if (t.cascade) {
      for (int32_t o = t.first_out; o < t.first_out + t.n_out; ++o) refs_of[o] += n;
    } else {
      refs_of[t.out_tile] += n;
    }
  }
  for (int32_t o = 0; o < n_out; ++o)
    if (refs_of[o] > 0) {
      ++c.merge;
      c.refs += refs_of[o];
    }
  return c;
}

bool bounded(const PlanRequest& r) { return r.max_work > 0 || r.max_merge > 0 || r.max_refs > 0 || r.max_ws_rows > 0; }

// Whether a split size stays within a graph plan's bounds and the int32 workspace rows.
bool fits(const std::vector<QTile>& tiles, int32_t n_out, int32_t chunk, const PlanRequest& r) {
  if (!bounded(r)) return stats_for(tiles, chunk).ws_rows <= std::numeric_limits<int32_t>::max() - kTileM;
  const Counts c = count_for(tiles, n_out, chunk);
  if (r.max_work > 0 && c.work > r.max_work) return false;
  if (r.max_merge > 0 && c.merge > r.max_merge) return false;
  if (r.max_refs > 0 && c.refs > r.max_refs) return false;
  if (r.max_ws_rows > 0 && c.ws_rows > r.max_ws_rows) return false;
  if (c.ws_rows > std::numeric_limits<int32_t>::max() - kTileM) return false;
  return true;
}

// Longest-processing-time-first makespan of the items a split size gives, over `units`
// identical SM pairs, plus the merge pass (which reads every partial once, spread over
// all units).  The costs are whole numbers no larger than `max_cost`, so the items are
// sorted by counting; and since the least loaded unit's load never decreases while items
// are placed, the units are kept as counts per load value with a pointer to the least
// load that only moves forward.  Stops early (returning a value >= `give_up`) once the
// makespan cannot end below `give_up`.
double estimate(const std::vector<QTile>& tiles, int32_t chunk, int units, int32_t max_cost,
                double give_up = std::numeric_limits<double>::infinity()) {
  static thread_local std::vector<int32_t> count;   // items per cost
  static thread_local std::vector<int32_t> at_load; // units per load value
  count.assign(static_cast<size_t>(max_cost) + 1, 0);
  int64_t partials = 0, total = 0;
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    const bool part = n > 1 || t.must_merge;
    const int32_t fixed = kItemCostI + (part ? kSplitCostI : 0);
    // n pieces: ntiles % n of them one tile longer than the rest
    const int32_t q = t.ntiles / n, r = t.ntiles % n;
    if (r > 0) count[q + 1 + fixed] += r;
    count[q + fixed] += n - r;
    total += int64_t(t.ntiles) + int64_t(n) * fixed;
    if (part) partials += n;
  }
  const double merge = kSplitCost * double(partials) / units;
  const double limit = give_up - merge;
  // every load stays below the makespan, which stays below min(total, limit) + max_cost
  int64_t top = total;
  if (limit < double(top)) top = std::max<int64_t>(0, static_cast<int64_t>(limit) + 1);
  at_load.assign(static_cast<size_t>(top + max_cost) + 2, 0);
  at_load[0] = units;
  int64_t least = 0, worst = 0;
  for (int32_t cost = max_cost; cost >= 0; --cost) {
    for (int32_t k = count[cost]; k > 0; --k) {
      while (at_load[least] == 0) ++least;
      const int64_t l = least + cost;
      --at_load[least];
      ++at_load[l];
      if (l > worst) {
        worst = l;
        if (double(worst) >= limit) return double(worst) + merge;
      }
    }
  }
  return double(worst) + merge;
}

}  // namespace

mla_status build_layout(const PlanRequest& req, PlanLayout* out) {
  if (!out) return MLA_ERR_INVALID_ARGUMENT;
  const mla_dims& d = req.d;
  const int32_t batch = req.batch;
  const int32_t* qo_indptr = req.qo_indptr;
  const int32_t* kv_indptr = req.kv_indptr;
  const int32_t* kv_indices = req.kv_indices;
  const int32_t* last_page_len = req.last_page_len;
  if (!shape_supported(d.kv_lora_rank, d.rope_dim, d.num_heads, d.page_size))
    return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || d.num_pages < 1 || !std::isfinite(d.sm_scale) || !(d.sm_scale > 0.f))
    return MLA_ERR_INVALID_ARGUMENT;
  if (!qo_indptr || !kv_indptr || (batch > 0 && !last_page_len)) return MLA_ERR_INVALID_ARGUMENT;
  if (req.split_keys > 0 && req.split_keys % kTileN != 0) return MLA_ERR_INVALID_ARGUMENT;
  const int32_t H = d.num_heads, P = d.page_size;
  int log2_P = 0;  // page sizes are powers of two (shape_supported)
  while ((1 << log2_P) < P) ++log2_P;
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
  {
    // every page id in [0, num_pages): one pass for the smallest and largest id
    int32_t lo = 0, hi = 0;
    if (n_idx > 0) lo = hi = kv_indices[0];
    for (int64_t i = 0; i < n_idx; ++i) {
      lo = std::min(lo, kv_indices[i]);
      hi = std::max(hi, kv_indices[i]);
    }
    if (lo < 0 || hi >= d.num_pages) return MLA_ERR_INVALID_ARGUMENT;
  }

  // --- per-row key counts (k_b from the tables; c_b = k_b - q_b attended if context-only)
  // Working arrays live in per-thread scratch that keeps its capacity from call to call,
  // so planning a step of a size seen before allocates nothing but the plan's own lists.
  static thread_local std::vector<int32_t> k_full, row_first_tile, suffix_from, ref_count, ref_next;
  static thread_local std::vector<uint8_t> out_cascaded;
  static thread_local std::vector<QTile> outs, tiles;
  static thread_local std::vector<uint64_t> order;
  static thread_local std::vector<WorkItem> sorted;
  k_full.assign(batch, 0);
  out->kv_len.assign(batch, 0);
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = kv_indptr[b + 1] - kv_indptr[b];
    const int32_t last = last_page_len[b];
    if (n > 0) {
      if (last < 1 || last > P) return MLA_ERR_INVALID_ARGUMENT;
      const int64_t k = (n - 1) * P + last;
      if (k > std::numeric_limits<int32_t>::max() - kTileN) return MLA_ERR_INVALID_ARGUMENT;
      k_full[b] = static_cast<int32_t>(k);
    } else {
      if (last < 0 || last > P) return MLA_ERR_INVALID_ARGUMENT;
    }
    const int32_t q_b = qo_indptr[b + 1] - qo_indptr[b];
    if (req.context_only) {
      if (k_full[b] < q_b) return MLA_ERR_INVALID_ARGUMENT;  // the tables lack the step's slots
      out->kv_len[b] = k_full[b] - q_b;
    } else {
      out->kv_len[b] = k_full[b];
    }
  }
  out->total_tokens = static_cast<int32_t>(T);

  // --- append slots: token i of row b is key k_b - q_b + i of its row
  out->append_rows.assign(static_cast<size_t>(T), -1);
  out->append_ok = true;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t q_b = qo_indptr[b + 1] - qo_indptr[b];
    for (int32_t i = 0; i < q_b; ++i) {
      const int64_t pos = int64_t(k_full[b]) - q_b + i;
      if (pos < 0) {
        out->append_ok = false;
        continue;
      }
      const int32_t page = kv_indices[kv_indptr[b] + (pos >> log2_P)];
      out->append_rows[qo_indptr[b] + i] = page * P + static_cast<int32_t>(pos & (P - 1));
    }
  }
  // A page listed twice can give two tokens one slot.  The later token's row is the one
  // kept: earlier tokens naming a slot that a later token also names get no destination,
  // so no two threads of the append ever store to one slot (their 16-byte pieces could
  // otherwise interleave).  Tokens are visited last to first against a hash set of the
  // slots already claimed.
  if (T > 1) {
    static thread_local std::vector<int32_t> seen;
    size_t cap = 16;
    while (cap < 2 * static_cast<size_t>(T)) cap <<= 1;
    if (seen.size() < cap) seen.resize(cap);
    std::fill(seen.begin(), seen.begin() + cap, -1);
    const size_t mask = cap - 1;
    for (int64_t t = T - 1; t >= 0; --t) {
      const int32_t row = out->append_rows[t];
      if (row < 0) continue;
      size_t h = (static_cast<uint32_t>(row) * 2654435761u) & mask;
      while (seen[h] >= 0 && seen[h] != row) h = (h + 1) & mask;
      if (seen[h] == row)
        out->append_rows[t] = -1;  // a later token writes this slot
      else
        seen[h] = row;
    }
  }

  // --- output tiles: 128 / H consecutive tokens of one row, all heads
  const int32_t tok_per_tile = kTileM / H;
  outs.clear();  // one per output tile, keys from 0
  row_first_tile.assign(batch + 1, 0);
  for (int32_t b = 0; b < batch; ++b) {
    row_first_tile[b] = static_cast<int32_t>(outs.size());
    const int32_t q_b = qo_indptr[b + 1] - qo_indptr[b];
    const int32_t k_b = out->kv_len[b];
    const bool causal = req.causal && !req.context_only;
    for (int32_t tok0 = 0; tok0 < q_b; tok0 += tok_per_tile) {
      const int32_t ntok = std::min(tok_per_tile, q_b - tok0);
      QTile t{};
      t.q_row0 = (qo_indptr[b] + tok0) * H;
      t.n_rows = ntok * H;
      t.page_base = kv_indptr[b];
      t.kv_len = k_b;
      // causal: token i sees keys < k_b - q_b + i + 1; otherwise all k_b keys
      t.diag_base = causal ? (k_b - q_b + tok0) : k_b;
      const int64_t hi = causal ? (int64_t)t.diag_base + ntok : (int64_t)k_b;
      t.vis_hi = static_cast<int32_t>(std::max<int64_t>(0, std::min<int64_t>(hi, k_b)));
      t.key0 = 0;
      t.out_tile = static_cast<int32_t>(outs.size());
      outs.push_back(t);
    }
  }
  row_first_tile[batch] = static_cast<int32_t>(outs.size());
  const int32_t n_out = static_cast<int32_t>(outs.size());

  // --- cascade: groups of consecutive rows sharing leading page ids
  tiles.clear();  // what gets split: cascade tiles and per-row (suffix) tiles
  suffix_from.assign(n_out, 0);  // first key of each output tile's own item
  out_cascaded.assign(n_out, 0);
  int32_t num_cascade_tiles = 0;
  if (req.cascade) {
    int32_t g = 0;
    while (g < batch) {
      // the longest run g..e-1 whose common page prefix still covers >= one key tile
      const int32_t n_g = kv_indptr[g + 1] - kv_indptr[g];
      int32_t lcp = n_g;  // pages common to rows g..e-1
      int32_t e = g + 1;
      while (e < batch) {
        const int32_t n_e = kv_indptr[e + 1] - kv_indptr[e];
        int32_t l = 0;
        const int32_t lim = std::min(lcp, n_e);
        while (l < lim && kv_indices[kv_indptr[g] + l] == kv_indices[kv_indptr[e] + l]) ++l;
        if (int64_t(l) * P < kTileN) break;
        lcp = l;
        ++e;
      }
      if (e - g >= 2) {
        // keys of the shared prefix every query of the group sees in full
        int64_t s = int64_t(lcp) * P;
        bool any_query = false;
        for (int32_t b = g; b < e; ++b) {
          const int32_t q_b = qo_indptr[b + 1] - qo_indptr[b];
          if (q_b == 0) continue;
          any_query = true;
          const int64_t k_b = out->kv_len[b];
          const bool causal = req.causal && !req.context_only;
          s = std::min<int64_t>(s, causal ? k_b - q_b + 1 : k_b);
        }
        s = s / kTileN * kTileN;
        if (any_query && s >= kTileN) {
          // pack the group's output tiles into cascade tiles of at most 128 rows
          const int32_t o0 = row_first_tile[g], o1 = row_first_tile[e];
          int32_t o = o0;
          while (o < o1) {
            QTile c{};
            c.q_row0 = outs[o].q_row0;
            c.n_rows = 0;
            c.first_out = o;
            c.n_out = 0;
            while (o < o1 && c.n_rows + outs[o].n_rows <= kTileM) {
              c.n_rows += outs[o].n_rows;
              ++c.n_out;
              ++o;
            }
            // A prefix tile that serves a single output tile reads the same keys for the
            // same queries as that tile would, and only adds a merge: leave it out.
            if (c.n_out < 2) continue;
            for (int32_t oo = c.first_out; oo < c.first_out + c.n_out; ++oo) {
              out_cascaded[oo] = 1;
              suffix_from[oo] = static_cast<int32_t>(s);
            }
            c.page_base = kv_indptr[g];
            c.kv_len = static_cast<int32_t>(s);
            c.diag_base = static_cast<int32_t>(s);  // every row sees all s keys
            c.key0 = 0;
            c.vis_hi = static_cast<int32_t>(s);
            c.ntiles = static_cast<int32_t>(s / kTileN);
            c.must_merge = true;
            c.cascade = true;
            c.out_tile = -1;
            tiles.push_back(c);
            ++num_cascade_tiles;
          }
        }
      }
      g = e;
    }
  }
  for (int32_t o = 0; o < n_out; ++o) {
    QTile t = outs[o];
    t.key0 = suffix_from[o];
    t.ntiles = t.vis_hi > t.key0 ? (t.vis_hi - t.key0 + kTileN - 1) / kTileN : 0;
    t.must_merge = out_cascaded[o];
    t.cascade = false;
    if (out_cascaded[o] && t.ntiles == 0) continue;  // the prefix covers every visible key
    tiles.push_back(t);
  }
  int64_t total_key_tiles = 0;
  int32_t max_ntiles = 0;
  for (const QTile& t : tiles) {
    total_key_tiles += t.ntiles;
    max_ntiles = std::max(max_ntiles, t.ntiles);
  }

  // --- choose the split size (within a graph plan's bounds)
  const int units = std::max(1, req.num_sms / 2);
  const int32_t max_cost = max_ntiles + kItemCostI + kSplitCostI;
  int32_t chunk = 0;  // 0: no split
  if (req.split_keys > 0) {
    chunk = req.split_keys / kTileN;
    if (!fits(tiles, n_out, chunk, req)) return MLA_ERR_INVALID_ARGUMENT;
  } else {
    if (!fits(tiles, n_out, 0, req)) return MLA_ERR_INVALID_ARGUMENT;
    const double avg = (double(total_key_tiles) + kItemCost * tiles.size()) / units;
    // No split can help when the longest tile already fits in the average load of a pair.
    if (req.split_keys == 0 && !tiles.empty() && max_ntiles > 1 && max_ntiles + kItemCost > avg) {
      // Items are dispatched to the SM pairs longest first, and a split pays when its
      // items fill whole waves of pairs.  The candidates are therefore, for each number
      // of waves k, the finest split whose items still fit in k waves (the number of
      // items does not grow with the chunk size, so a bisection finds it).  Each is
      // scored by the list-scheduling model, in order of a lower bound on its makespan
      // (the longest item and the average load per pair, plus the merge pass), and a
      // split is kept only if it is 1% better than the best so far.
      struct Cand {
        double bound;
        int32_t chunk;
      };
      Cand cands[kMaxWaves + 3];
      int n_cands = 0;
      bool any_must = false;
      for (const QTile& t : tiles) any_must |= t.must_merge;
      static thread_local TileCounts hist;
      if (!any_must) hist.build(tiles, max_ntiles);
      auto stats = [&](int32_t c) { return any_must ? stats_for(tiles, c) : hist.stats(c); };
      auto add = [&](int32_t c) {
        if (c < 2 || c >= max_ntiles) return;
        for (int i = 0; i < n_cands; ++i)
          if (cands[i].chunk == c) return;
        const SplitStats st = stats(c);
        const double bound = std::max(double(st.longest), double(st.total_cost) / units) +
                             kSplitCost * double(st.partials) / units;
        cands[n_cands++] = Cand{bound, c};
      };
      int32_t prev = -1;
      for (int64_t k = 1; k <= kMaxWaves; ++k) {
        int32_t lo = 2, hi = (prev > 0 ? prev : max_ntiles) - 1, found = -1;
        while (lo <= hi) {
          const int32_t mid = lo + (hi - lo) / 2;
          int64_t items = 0;
          if (any_must) {
            const PieceCounter pieces(mid);
            for (const QTile& t : tiles) items += pieces(t.ntiles);
          } else {
            items = hist.items(mid);
          }
          if (items <= k * units) {
            found = mid;
            hi = mid - 1;
          } else {
            lo = mid + 1;
          }
        }
        if (found < 0 || found == prev) continue;
        prev = found;
        add(found);
      }
      // ... and the balance point, where the longest item stops being shorter than the
      // average load of a pair (the chunk that minimises the lower bound), with its
      // neighbours: between whole waves the model can still prefer a split there.
      {
        int32_t lo = 2, hi = max_ntiles - 1, found = -1;
        while (lo <= hi) {
          const int32_t mid = lo + (hi - lo) / 2;
          const SplitStats st = stats(mid);
          if (double(st.longest) >= double(st.total_cost) / units) {
            found = mid;
            hi = mid - 1;
          } else {
            lo = mid + 1;
          }
        }
        if (found > 0) {
          add(found - 1);
          add(found);
          add(found + 1);
        }
      }
      std::sort(cands, cands + n_cands, [](const Cand& x, const Cand& y) { return x.bound < y.bound; });
      double best = estimate(tiles, 0, units, max_cost);
      for (int i = 0; i < n_cands; ++i) {
        if (cands[i].bound >= best * 0.99) break;  // neither this nor any later one can win
        if (!fits(tiles, n_out, cands[i].chunk, req)) continue;
        const double e = estimate(tiles, cands[i].chunk, units, max_cost, best * 0.99);
        if (e < best * 0.99) {
          best = e;
          chunk = cands[i].chunk;
        }
      }
    }
  }
  // Latency regime: when the items fit in one wave, every item runs on its own pair and
  // the step lasts as long as its longest item (plus a merge launch if anything is
  // split), so split the longest tiles further, down to single key tiles, while the
  // items still fit one wave (a tiny decode step: 14.8 us instead of 16.8 us).
  if (req.split_keys == 0 && !tiles.empty() && max_ntiles > 1) {
    auto latency = [&](int32_t c, int64_t* items) {
      double longest = 0.0;
      int64_t it = 0, partials = 0;
      for (const QTile& t : tiles) {
        const int32_t n = c > 0 ? pieces_for(t.ntiles, c) : 1;
        it += n;
        if (n > 1 || t.must_merge) partials += n;
        longest = std::max(longest, double((t.ntiles + n - 1) / n) + kItemCost);
      }
      *items = it;
      return longest + (partials > 0 ? kMergeLatency : 0.0);
    };
    int64_t items = 0;
    double best_lat = latency(chunk, &items);
    if (items <= units) {
      for (int32_t c = std::max<int32_t>(1, chunk > 0 ? chunk - 1 : max_ntiles - 1); c >= 1; --c) {
        int64_t it = 0;
        const double l = latency(c, &it);
        if (it > units) break;  // finer splits only add items
        if (l < best_lat * 0.99 && fits(tiles, n_out, c, req)) {
          best_lat = l;
          chunk = c;
        }
      }
    }
  }
  out->chunk_tiles = chunk;

  // --- emit items and the merge references of every output tile.  Each output tile's
  // references are its partials in emission order; they are counted first, so that the
  // merge list and the reference list are written in place.
  ref_count.assign(n_out, 0);
  int64_t n_items = 0;
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    n_items += n;
    if (n == 1 && !t.must_merge) continue;
    if (t.cascade) {
      for (int32_t o = t.first_out; o < t.first_out + t.n_out; ++o) ref_count[o] += n;
    } else {
      ref_count[t.out_tile] += n;
    }
  }
  out->merge.clear();
  ref_next.resize(n_out);
  int32_t n_refs = 0;
  for (int32_t o = 0; o < n_out; ++o) {
    ref_next[o] = n_refs;
    if (ref_count[o] == 0) continue;
    out->merge.push_back(MergeItem{outs[o].q_row0, outs[o].n_rows, n_refs, ref_count[o]});
    n_refs += ref_count[o];
  }
  out->refs.resize(n_refs);
  sorted.resize(static_cast<size_t>(n_items));
  int32_t ws_row = 0, partials = 0, cascade_items = 0;
  size_t wi = 0;
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    const bool part = n > 1 || t.must_merge;
    // piece p covers key tiles [floor(ntiles * p / n), floor(ntiles * (p + 1) / n)),
    // stepped exactly without a division per piece: ntiles = q * n + r
    const int32_t q = t.ntiles / n, r = t.ntiles % n;
    int32_t hi = 0, rem = 0;
    for (int32_t p = 0; p < n; ++p) {
      const int32_t lo = hi;
      hi = lo + q;
      rem += r;
      if (rem >= n) {
        rem -= n;
        ++hi;
      }
      WorkItem w{t.q_row0, t.n_rows, t.page_base, t.kv_len, t.key0 + lo * kTileN,
                 std::min(t.key0 + hi * kTileN, t.vis_hi), t.diag_base, -1};
      if (t.ntiles == 0) w.key_begin = w.key_end = t.key0;
      if (part) {
        w.partial = ws_row;
        if (t.cascade) {
          for (int32_t o = t.first_out; o < t.first_out + t.n_out; ++o)
            out->refs[ref_next[o]++] = ws_row + (outs[o].q_row0 - t.q_row0);
        } else {
          out->refs[ref_next[t.out_tile]++] = ws_row;
        }
        ws_row += t.n_rows;
        ++partials;
      }
      if (t.cascade) ++cascade_items;
      sorted[wi++] = w;
    }
  }
  out->num_partials = partials;
  out->ws_rows = ws_row;
  out->num_cascade = cascade_items;
  // Longest first; equal lengths keep their order, so a group's prefix items stay
  // adjacent.  Sorted as (length descending, emission index) keys: a total order, so the
  // result is the stable order without a stable sort's buffer.
  order.resize(sorted.size());
  for (size_t i = 0; i < sorted.size(); ++i) {
    const uint32_t len = static_cast<uint32_t>(sorted[i].key_end - sorted[i].key_begin);
    order[i] = (uint64_t(~len) << 32) | uint64_t(i);
  }
  if (order.size() <= 512) {
    std::sort(order.begin(), order.end());
  } else {
    // Many items (prefill steps): a least-significant-digit radix sort on the 32-bit
    // length key, 11 bits a pass; each pass is stable, and the keys are built in
    // emission order, so equal lengths keep that order.
    static thread_local std::vector<uint64_t> tmp;
    tmp.resize(order.size());
    for (int shift = 32; shift < 64; shift += 11) {
      size_t count[2049] = {0};
      for (uint64_t k : order) ++count[((k >> shift) & 2047) + 1];
      if (count[((order[0] >> shift) & 2047) + 1] == order.size()) continue;  // one digit: no-op
      for (int i = 0; i < 2048; ++i) count[i + 1] += count[i];
      for (uint64_t k : order) tmp[count[(k >> shift) & 2047]++] = k;
      order.swap(tmp);
    }
  }
  out->work.resize(sorted.size());
  for (size_t i = 0; i < order.size(); ++i) out->work[i] = sorted[static_cast<uint32_t>(order[i])];
  return MLA_OK;
}

}  // namespace mla

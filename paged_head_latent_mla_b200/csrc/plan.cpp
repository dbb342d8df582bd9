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
#include <functional>
#include <limits>
#include <queue>

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

// Longest-processing-time-first makespan of `costs` over `units` identical units.  Stops
// early (returning a value >= `give_up`) once the makespan cannot end below `give_up`.
double lpt_makespan(std::vector<double>& costs, int units, double give_up) {
  std::sort(costs.begin(), costs.end(), std::greater<double>());
  std::priority_queue<double, std::vector<double>, std::greater<double>> load;
  for (int i = 0; i < units; ++i) load.push(0.0);
  double worst = 0.0;
  for (double c : costs) {
    double l = load.top();
    load.pop();
    l += c;
    worst = std::max(worst, l);
    if (worst >= give_up) return worst;
    load.push(l);
  }
  return worst;
}

// Pieces of at most `chunk` key tiles (sizes differing by at most one).
inline int32_t pieces_for(int32_t ntiles, int32_t chunk) {
  if (ntiles <= 0) return 1;
  if (chunk <= 0) return 1;
  return (ntiles + chunk - 1) / chunk;
}

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

bool fits(const Counts& c, const PlanRequest& r) {
  if (r.max_work > 0 && c.work > r.max_work) return false;
  if (r.max_merge > 0 && c.merge > r.max_merge) return false;
  if (r.max_refs > 0 && c.refs > r.max_refs) return false;
  if (r.max_ws_rows > 0 && c.ws_rows > r.max_ws_rows) return false;
  if (c.ws_rows > std::numeric_limits<int32_t>::max() - kTileM) return false;
  return true;
}

double estimate(const std::vector<QTile>& tiles, int32_t chunk, int units,
                double give_up = std::numeric_limits<double>::infinity()) {
  std::vector<double> costs;
  costs.reserve(tiles.size() * 2);
  int64_t partials = 0;
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    if (n == 1 && !t.must_merge) {
      costs.push_back(t.ntiles + kItemCost);
    } else {
      partials += n;
      for (int32_t p = 0; p < n; ++p) {
        const int32_t lo = (int64_t)t.ntiles * p / n, hi = (int64_t)t.ntiles * (p + 1) / n;
        costs.push_back((hi - lo) + kItemCost + kSplitCost);
      }
    }
  }
  // The merge pass reads every partial once, spread over all units.
  const double merge = kSplitCost * double(partials) / units;
  return lpt_makespan(costs, units, give_up - merge) + merge;
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

  // --- per-row key counts (k_b from the tables; c_b = k_b - q_b attended if context-only)
  std::vector<int32_t> k_full(batch, 0);
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
      const int32_t page = kv_indices[kv_indptr[b] + pos / P];
      out->append_rows[qo_indptr[b] + i] = page * P + static_cast<int32_t>(pos % P);
    }
  }

  // --- output tiles: 128 / H consecutive tokens of one row, all heads
  const int32_t tok_per_tile = kTileM / H;
  std::vector<QTile> outs;  // one per output tile, keys from 0
  std::vector<int32_t> row_first_tile(batch + 1, 0);
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
  std::vector<QTile> tiles;  // what gets split: cascade tiles and per-row (suffix) tiles
  std::vector<int32_t> suffix_from(n_out, 0);  // first key of each output tile's own item
  std::vector<bool> out_cascaded(n_out, false);
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
              out_cascaded[oo] = true;
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
  int32_t chunk = 0;  // 0: no split
  if (req.split_keys > 0) {
    chunk = req.split_keys / kTileN;
    if (!fits(count_for(tiles, n_out, chunk), req)) return MLA_ERR_INVALID_ARGUMENT;
  } else {
    if (!fits(count_for(tiles, n_out, 0), req)) return MLA_ERR_INVALID_ARGUMENT;
    const double avg = (double(total_key_tiles) + kItemCost * tiles.size()) / units;
    // No split can help when the longest tile already fits in the average load of a pair.
    if (req.split_keys == 0 && !tiles.empty() && max_ntiles > 1 && max_ntiles + kItemCost > avg) {
      // Every chunk size is a candidate (at most ~1000 of them, evenly spaced).
      std::vector<int32_t> cands;
      const int32_t stride = std::max<int32_t>(1, (max_ntiles - 2) / 1024);
      for (int32_t c = 2; c < max_ntiles; c += stride) cands.push_back(c);
      // Finalists for the full LPT estimate: for each number of waves k (items in k x
      // pairs), the smallest chunk whose items still fit in k waves (the finest split
      // with no straggling last wave), and the two candidates with the lowest bound on
      // the makespan (the largest of: the longest item, the average load per pair, and
      // the items some pair must take times the shortest item; plus the merge pass).
      struct Scored {
        double bound;
        int32_t chunk;
        int64_t items;
      };
      std::vector<Scored> scored;
      for (int32_t c : cands) {
        double longest = 0.0, shortest = std::numeric_limits<double>::infinity(), sum = 0.0, partials = 0.0;
        int64_t items = 0;
        for (const QTile& t : tiles) {
          const int32_t n = pieces_for(t.ntiles, c);
          const bool part = n > 1 || t.must_merge;
          const double fixed = kItemCost + (part ? kSplitCost : 0.0);
          longest = std::max(longest, double((t.ntiles + n - 1) / n) + fixed);
          shortest = std::min(shortest, double(t.ntiles / n) + fixed);
          sum += t.ntiles + n * fixed;
          items += n;
          if (part) partials += n;
        }
        const double per_unit = double((items + units - 1) / units) * shortest;
        scored.push_back(Scored{std::max({longest, sum / units, per_unit}) + kSplitCost * partials / units, c, items});
      }
      std::vector<int32_t> finalists;
      for (int64_t k = 1; k <= kMaxWaves; ++k) {
        // cands ascend, items descend: the first candidate within k waves
        for (const Scored& x : scored)
          if (x.items <= k * units) {
            if (finalists.empty() || finalists.back() != x.chunk) finalists.push_back(x.chunk);
            break;
          }
      }
      std::sort(scored.begin(), scored.end(), [](const Scored& x, const Scored& y) { return x.bound < y.bound; });
      for (size_t i = 0; i < scored.size() && i < 2; ++i) finalists.push_back(scored[i].chunk);
      std::sort(finalists.begin(), finalists.end(), std::greater<int32_t>());
      finalists.erase(std::unique(finalists.begin(), finalists.end()), finalists.end());
      double best = estimate(tiles, 0, units);
      for (int32_t c : finalists) {
        if (!fits(count_for(tiles, n_out, c), req)) continue;
        // (an estimate that cannot beat best * 0.99 stops early: prefer fewer splits
        // unless clearly better)
        const double e = estimate(tiles, c, units, best * 0.99);
        if (e < best * 0.99) {
          best = e;
          chunk = c;
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
        if (l < best_lat * 0.99 && fits(count_for(tiles, n_out, c), req)) {
          best_lat = l;
          chunk = c;
        }
      }
    }
  }
  out->chunk_tiles = chunk;

  // --- emit items and the merge references of every output tile
  out->work.clear();
  out->merge.clear();
  out->refs.clear();
  std::vector<std::vector<int32_t>> refs_of(n_out);
  int32_t ws_row = 0, partials = 0, cascade_items = 0;
  for (const QTile& t : tiles) {
    const int32_t n = pieces_for(t.ntiles, chunk);
    const bool part = n > 1 || t.must_merge;
    for (int32_t p = 0; p < n; ++p) {
      const int32_t lo = (int64_t)t.ntiles * p / n, hi = (int64_t)t.ntiles * (p + 1) / n;
      WorkItem w{t.q_row0, t.n_rows, t.page_base, t.kv_len, t.key0 + lo * kTileN,
                 std::min(t.key0 + hi * kTileN, t.vis_hi), t.diag_base, -1};
      if (t.ntiles == 0) w.key_begin = w.key_end = t.key0;
      if (part) {
        w.partial = ws_row;
        if (t.cascade) {
          for (int32_t o = t.first_out; o < t.first_out + t.n_out; ++o)
            refs_of[o].push_back(ws_row + (outs[o].q_row0 - t.q_row0));
        } else {
          refs_of[t.out_tile].push_back(ws_row);
        }
        ws_row += t.n_rows;
        ++partials;
      }
      if (t.cascade) ++cascade_items;
      out->work.push_back(w);
    }
  }
  for (int32_t o = 0; o < n_out; ++o) {
    if (refs_of[o].empty()) continue;
    out->merge.push_back(MergeItem{outs[o].q_row0, outs[o].n_rows, static_cast<int32_t>(out->refs.size()),
                                   static_cast<int32_t>(refs_of[o].size())});
    out->refs.insert(out->refs.end(), refs_of[o].begin(), refs_of[o].end());
  }
  out->num_partials = partials;
  out->ws_rows = ws_row;
  out->num_cascade = cascade_items;
  // longest first; equal lengths keep their order, so a group's prefix items stay adjacent
  std::stable_sort(out->work.begin(), out->work.end(), [](const WorkItem& a, const WorkItem& b) {
    return (a.key_end - a.key_begin) > (b.key_end - b.key_begin);
  });
  return MLA_OK;
}

}  // namespace mla

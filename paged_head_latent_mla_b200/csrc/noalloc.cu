// mla_run_noalloc: the attention call for callers that must not allocate memory.
//
// Some callers cannot call cudaMalloc at the point where they run attention: serving
// processes whose memory manager has already handed all of HBM to its own pools (a KV
// page pool, an activation arena) and forbids any other allocation; plug-in hosts that
// own device memory and give a library no allocator; latency-critical loops where a
// cudaMalloc or cudaFree could synchronise the device.  mla_plan allocates (work lists,
// page-table copy, split-KV workspace, pinned staging), so those callers use this entry
// point instead: it plans on the host without touching the heap, and every piece of
// device scratch it needs (status word, work list, merge list, page-table copy and the
// split-KV partial results) lives in one array compiled into the library.
//
// The array is a file-scope __device__ variable: every GPU that loads the library
// holds kScratchBytes of it until the process exits.  Host code may not use the
// array's name as a device address (it is a host-side stand-in), so the device address
// is looked up once per device with cudaGetSymbolAddress, with that device current.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <mutex>

#include "mla_internal.h"
#include "mla_launch.h"

namespace {

using namespace mla;

// Fixed scratch budget and its layout.
constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kMaxWork = 16384;                     // work items
constexpr int kMaxMerge = 4096;                     // split query tiles
constexpr int kMaxPageIds = 1 << 19;                // kv_indptr[batch]
constexpr size_t kOffStatus = 0;
constexpr size_t kOffWork = 256;
constexpr size_t kOffMerge = kOffWork + sizeof(WorkItem) * kMaxWork;
constexpr size_t kOffRefs = kOffMerge + sizeof(MergeItem) * kMaxMerge;
constexpr size_t kOffPages = kOffRefs + sizeof(int32_t) * kMaxWork;
constexpr size_t kOffPartials = (kOffPages + sizeof(int32_t) * kMaxPageIds + 255) / 256 * 256;
// workspace rows of split partial results (each partial takes its tile's rows)
constexpr int kMaxWsRows = static_cast<int>((kScratchBytes - kOffPartials) / kWsRowBytes);
static_assert(kMaxWsRows >= 32 * kTileM, "scratch too small for useful splitting");

// Host-side planning buffers: static, so planning never touches the heap.  Calls that
// overlap on the host would race on these, like they race on the device array.
WorkItem g_work[kMaxWork];
MergeItem g_merge[kMaxMerge];
int32_t g_refs[kMaxWork];
int32_t g_tile_nt[kMaxWork];    // key tiles of each query tile
int32_t g_tile_rows[kMaxWork];  // rows of each query tile
double g_costs[kMaxWork];       // item costs of one split candidate
constexpr int kMaxUnits = 1024;
double g_loads[kMaxUnits];

inline int32_t pieces_of(int32_t nt, int32_t chunk) { return (chunk > 0 && nt > chunk) ? (nt + chunk - 1) / chunk : 1; }

// Items, merge records and workspace rows of a split size; false if beyond the scratch.
bool split_fits(int n_tiles, int32_t chunk, int64_t* items) {
  int64_t it = 0, merges = 0, rows = 0;
  for (int i = 0; i < n_tiles; ++i) {
    const int32_t n = pieces_of(g_tile_nt[i], chunk);
    it += n;
    if (n > 1) {
      ++merges;
      rows += int64_t(n) * g_tile_rows[i];
    }
  }
  *items = it;
  return it <= kMaxWork && merges <= kMaxMerge && rows <= kMaxWsRows;
}

// Longest-first list-scheduling makespan of a split size over `units` SM pairs, the same
// model as mla_plan's (static buffers only).
double split_makespan(int n_tiles, int32_t chunk, int units) {
  int m = 0;
  int64_t partials = 0;
  for (int i = 0; i < n_tiles; ++i) {
    const int32_t nt = g_tile_nt[i], n = pieces_of(nt, chunk);
    for (int32_t p = 0; p < n; ++p) {
      const int32_t lo = int32_t(int64_t(nt) * p / n), hi = int32_t(int64_t(nt) * (p + 1) / n);
      g_costs[m++] = (hi - lo) + kItemCost + (n > 1 ? kSplitCost : 0.0);
    }
    if (n > 1) partials += n;
  }
  std::sort(g_costs, g_costs + m, [](double a, double b) { return a > b; });
  for (int u = 0; u < units; ++u) g_loads[u] = 0.0;
  double worst = 0.0;
  for (int i = 0; i < m; ++i) {
    int best = 0;
    for (int u = 1; u < units; ++u)
      if (g_loads[u] < g_loads[best]) best = u;
    g_loads[best] += g_costs[i];
    worst = std::max(worst, g_loads[best]);
  }
  return worst + kSplitCost * double(partials) / units;
}

// The split size: no split when no query tile exceeds the average load of a pair;
// otherwise, for each wave count k, the finest split whose items fit in k waves of the
// pairs, scored by the makespan model (a split must be 1% better than the one before).
int32_t choose_chunk(int n_tiles, int64_t total_tiles, int units) {
  int32_t max_nt = 0;
  for (int i = 0; i < n_tiles; ++i) max_nt = std::max(max_nt, g_tile_nt[i]);
  const double avg = (double(total_tiles) + kItemCost * n_tiles) / units;
  if (n_tiles == 0 || max_nt <= 1 || max_nt + kItemCost <= avg) return 0;
  int32_t chunk = 0;
  double best = split_makespan(n_tiles, 0, units);
  int32_t last_tried = -1;
  for (int k = 1; k <= kMaxWaves; ++k) {
    // items(c) does not increase with c: bisect for the smallest c within k waves
    int32_t lo = 2, hi = max_nt - 1, found = -1;
    while (lo <= hi) {
      const int32_t mid = lo + (hi - lo) / 2;
      int64_t items = 0;
      const bool ok = split_fits(n_tiles, mid, &items);
      if (items <= int64_t(k) * units) {
        if (ok) found = mid;
        hi = mid - 1;
      } else {
        lo = mid + 1;
      }
    }
    if (found < 0 || found == last_tried) continue;
    last_tried = found;
    const double e = split_makespan(n_tiles, found, units);
    if (e < best * 0.99) {
      best = e;
      chunk = found;
    }
  }
  return chunk;
}

struct DeviceScratch {
  unsigned char* ptr = nullptr;
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceScratch g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Validate the tables and cut the work into g_work / g_merge without allocating.  The
// split size follows mla_plan's rule (whole waves of SM pairs, the same cost model), kept
// within the scratch array; a tile whose pieces would not fit the rest runs unsplit.
mla_status plan_fixed(const mla_dims& d, int32_t batch, const int32_t* qo, const int32_t* kvp,
                      const int32_t* kvi, const int32_t* last, bool causal, int num_sms, int* n_work,
                      int* n_merge, int* n_refs, int* n_ws_rows, int32_t* total_tokens) {
  if (!shape_supported(d.kv_lora_rank, d.rope_dim, d.num_heads, d.page_size)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || d.num_pages < 1 || !std::isfinite(d.sm_scale) || !(d.sm_scale > 0.f))
    return MLA_ERR_INVALID_ARGUMENT;
  if (!qo || !kvp || (batch > 0 && !last)) return MLA_ERR_INVALID_ARGUMENT;
  const int32_t H = d.num_heads, P = d.page_size;
  if (int64_t(d.num_pages) * P > std::numeric_limits<int32_t>::max()) return MLA_ERR_INVALID_ARGUMENT;
  if (qo[0] != 0 || kvp[0] != 0) return MLA_ERR_INVALID_ARGUMENT;
  for (int32_t b = 0; b < batch; ++b)
    if (qo[b + 1] < qo[b] || kvp[b + 1] < kvp[b]) return MLA_ERR_INVALID_ARGUMENT;
  const int64_t T = qo[batch], n_idx = kvp[batch];
  if (T * H > std::numeric_limits<int32_t>::max() - kTileM) return MLA_ERR_INVALID_ARGUMENT;
  if (n_idx > kMaxPageIds) return MLA_ERR_INVALID_ARGUMENT;  // beyond the fixed scratch
  if (n_idx > 0 && !kvi) return MLA_ERR_INVALID_ARGUMENT;
  for (int64_t i = 0; i < n_idx; ++i)
    if (kvi[i] < 0 || kvi[i] >= d.num_pages) return MLA_ERR_INVALID_ARGUMENT;
  // pass 1: validate rows, count tiles
  int64_t total_tiles = 0, n_tiles = 0;
  const int32_t tok_per_tile = kTileM / H;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = kvp[b + 1] - kvp[b];
    if (n > 0 ? (last[b] < 1 || last[b] > P) : (last[b] < 0 || last[b] > P)) return MLA_ERR_INVALID_ARGUMENT;
    const int64_t k = n > 0 ? (n - 1) * P + last[b] : 0;
    if (k > std::numeric_limits<int32_t>::max() - kTileN) return MLA_ERR_INVALID_ARGUMENT;
    const int32_t q_b = qo[b + 1] - qo[b];
    for (int32_t tok0 = 0; tok0 < q_b; tok0 += tok_per_tile) {
      const int32_t ntok = std::min(tok_per_tile, q_b - tok0);
      const int64_t diag = causal ? k - q_b + tok0 : k;
      const int64_t hi = std::max<int64_t>(0, std::min<int64_t>(causal ? diag + ntok : k, k));
      if (n_tiles >= kMaxWork) return MLA_ERR_INVALID_ARGUMENT;  // beyond the fixed scratch
      g_tile_nt[n_tiles] = static_cast<int32_t>((hi + kTileN - 1) / kTileN);
      g_tile_rows[n_tiles] = ntok * H;
      total_tiles += g_tile_nt[n_tiles];
      ++n_tiles;
    }
  }
  const int units = std::min(kMaxUnits, std::max(1, num_sms / 2));
  const int32_t chunk = choose_chunk(static_cast<int>(n_tiles), total_tiles, units);
  // pass 2: emit (every tile still to come keeps at least one work slot)
  int nw = 0, nm = 0, nr = 0, rows_used = 0;
  int64_t tiles_left = n_tiles;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = kvp[b + 1] - kvp[b];
    const int32_t k = n > 0 ? static_cast<int32_t>((n - 1) * P + last[b]) : 0;
    const int32_t q_b = qo[b + 1] - qo[b];
    for (int32_t tok0 = 0; tok0 < q_b; tok0 += tok_per_tile) {
      const int32_t ntok = std::min(tok_per_tile, q_b - tok0);
      const int32_t diag = causal ? k - q_b + tok0 : k;
      const int64_t hi64 = std::max<int64_t>(0, std::min<int64_t>(causal ? int64_t(diag) + ntok : k, k));
      const int32_t vis_hi = static_cast<int32_t>(hi64);
      const int32_t nt = (vis_hi + kTileN - 1) / kTileN;
      const int32_t q_row0 = (qo[b] + tok0) * H;
      int32_t pieces = pieces_of(nt, chunk);
      --tiles_left;
      if (pieces > 1 && (rows_used + pieces * ntok * H > kMaxWsRows || nm >= kMaxMerge ||
                         nw + pieces + tiles_left > kMaxWork))
        pieces = 1;  // no scratch left for partials: run this tile unsplit
      if (nw + pieces > kMaxWork) return MLA_ERR_INVALID_ARGUMENT;
      if (pieces == 1) {
        g_work[nw++] = WorkItem{q_row0, ntok * H, kvp[b], k, 0, vis_hi, diag, -1};
        continue;
      }
      g_merge[nm++] = MergeItem{q_row0, ntok * H, nr, pieces};
      for (int32_t i = 0; i < pieces; ++i) {
        const int32_t lo = int32_t(int64_t(nt) * i / pieces), hi = int32_t(int64_t(nt) * (i + 1) / pieces);
        g_refs[nr++] = rows_used;
        g_work[nw++] =
            WorkItem{q_row0, ntok * H, kvp[b], k, lo * kTileN, std::min(hi * kTileN, vis_hi), diag, rows_used};
        rows_used += ntok * H;
      }
    }
  }
  std::sort(g_work, g_work + nw, [](const WorkItem& a, const WorkItem& c) {
    return (a.key_end - a.key_begin) > (c.key_end - c.key_begin);
  });
  *n_work = nw;
  *n_merge = nm;
  *n_refs = nr;
  *n_ws_rows = rows_used;
  *total_tokens = static_cast<int32_t>(T);
  return MLA_OK;
}

}  // namespace

// The scratch array itself.  Device code could name it directly; host code only ever
// uses the address returned by cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_mla_noalloc_scratch[kScratchBytes];

extern "C" mla_status mla_run_noalloc(const mla_dims* dims, int32_t batch, const int32_t* qo_indptr,
                                      const int32_t* kv_indptr, const int32_t* kv_indices,
                                      const int32_t* last_page_len, int32_t causal, const void* q_nope,
                                      const void* q_pe, const void* cache, void* out, float* lse, void* stream,
                                      int32_t* status_out) {
  if (!dims || (causal != 0 && causal != 1)) return MLA_ERR_INVALID_ARGUMENT;
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u)) return MLA_ERR_INVALID_ARGUMENT;
  // The copies below read the static host buffers at enqueue time; a graph captured
  // here would keep pointing at them (and at the caller's page table) while its launch
  // shapes stayed those of this step, so a replay could run another step's work list.
  {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cs) != cudaSuccess) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    if (cs != cudaStreamCaptureStatusNone) return MLA_ERR_UNSUPPORTED;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;

  // One-time set-up on this device (with it current): the scratch array's device
  // address and the SM count.
  {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_dev[dev].ptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_mla_noalloc_scratch) != cudaSuccess || !ptr) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
      }
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MLA_ERR_CUDA;
      g_dev[dev].ptr = static_cast<unsigned char*>(ptr);
      g_dev[dev].num_sms = sms;
    }
  }
  unsigned char* scratch = g_dev[dev].ptr;

  int n_work = 0, n_merge = 0, n_refs = 0, n_ws_rows = 0;
  int32_t T = 0;
  mla_status st = plan_fixed(*dims, batch, qo_indptr, kv_indptr, kv_indices, last_page_len, causal != 0,
                             g_dev[dev].num_sms, &n_work, &n_merge, &n_refs, &n_ws_rows, &T);
  if (st != MLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_work == 0) {
    if (status_out && cudaMemsetAsync(status_out, 0, sizeof(int32_t), s) != cudaSuccess) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    return MLA_OK;
  }
  const bool rope = dims->rope_dim > 0;  // without kpe, q_pe is not read (may be NULL)
  if (!q_nope || (rope && !q_pe) || !cache || !out) return MLA_ERR_INVALID_ARGUMENT;
  auto misaligned = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) != 0; };
  if (misaligned(q_nope) || (rope && misaligned(q_pe)) || misaligned(cache) || misaligned(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return MLA_ERR_INVALID_ARGUMENT;

  // Fill the scratch: status word cleared, work and merge lists, page-table copy.  The
  // copies read host memory that is pageable, so each returns once its source has been
  // read and the static host buffers may be reused by the next call.
  const size_t n_idx = static_cast<size_t>(kv_indptr[batch]);
  if (cudaMemsetAsync(scratch + kOffStatus, 0, 256, s) != cudaSuccess ||
      cudaMemcpyAsync(scratch + kOffWork, g_work, sizeof(WorkItem) * n_work, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      (n_merge > 0 && cudaMemcpyAsync(scratch + kOffMerge, g_merge, sizeof(MergeItem) * n_merge,
                                      cudaMemcpyHostToDevice, s) != cudaSuccess) ||
      (n_merge > 0 && cudaMemcpyAsync(scratch + kOffRefs, g_refs, sizeof(int32_t) * n_refs,
                                      cudaMemcpyHostToDevice, s) != cudaSuccess) ||
      (n_idx > 0 && cudaMemcpyAsync(scratch + kOffPages, kv_indices, sizeof(int32_t) * n_idx,
                                    cudaMemcpyHostToDevice, s) != cudaSuccess)) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }

  unsigned char* partials = scratch + kOffPartials;
  AttnLaunch a;
  AttnParams& ap = a.p;
  ap.work = reinterpret_cast<const WorkItem*>(scratch + kOffWork);
  ap.kv_indices = reinterpret_cast<const int32_t*>(scratch + kOffPages);
  ap.out = out;
  ap.lse = lse;
  ap.ws_o = partials;
  ap.ws_lse = reinterpret_cast<float*>(partials + size_t(n_ws_rows) * kWsRowOBytes);
  ap.status = reinterpret_cast<int32_t*>(scratch + kOffStatus);
  ap.status_mirror = nullptr;  // read back by a device-to-device copy below
  ap.scale_log2 = dims->sm_scale * 1.4426950408889634f;
  ap.num_heads = dims->num_heads;
  ap.page_size = dims->page_size;
  ap.rope_dim = dims->rope_dim;
  ap.timeout_ns = 4000000000ull;
  ap.debug_flags = 0;
  a.q_nope = q_nope;
  a.q_pe = q_pe;
  a.cache = cache;
  a.rows = uint64_t(T) * dims->num_heads;
  a.cache_rows = uint64_t(dims->num_pages) * dims->page_size;
  a.num_work = n_work;
  a.wait_prior_grid = false;
  if (launch_attention(a, s) != cudaSuccess) return MLA_ERR_CUDA;
  if (n_merge > 0) {
    MergeParams mp{reinterpret_cast<const MergeItem*>(scratch + kOffMerge),
                   reinterpret_cast<const int32_t*>(scratch + kOffRefs), ap.ws_o, ap.ws_lse, out, lse};
    if (launch_merge(mp, n_merge, s) != cudaSuccess) return MLA_ERR_CUDA;
  }
  // The status word the kernels wrote (0, or MLA_ERR_DEVICE_TIMEOUT in its low byte),
  // handed to the caller's own word once the stream has passed the launches.
  if (status_out && cudaMemcpyAsync(status_out, scratch + kOffStatus, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                                    s) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

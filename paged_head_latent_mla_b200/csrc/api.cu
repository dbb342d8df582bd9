// C ABI of the paged latent-attention library: plan ownership, launches and the device
// status word.  See include/mla.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "mla_internal.h"

#include "mla_launch.h"

using namespace mla;

struct mla_plan_s {
  mla_dims dims{};
  int32_t batch = 0;
  bool causal = true;
  mla_plan_options opts{};
  PlanLayout layout;
  PlanLayout spare;  // the previous step's layout, kept so a re-plan reuses its capacity
  int device = -1;
  bool host_only = false;
  bool graph = false;     // fixed buffers and launch shapes (opts.graph_max_*)
  bool captured = false;  // mla_run was called on a capturing stream
  // the step's tables, to recognise an unchanged step in mla_plan_update
  std::vector<int32_t> fp_qo, fp_kvp, fp_kvi, fp_last;
  // capacities of the device lists (exact sizes unless a graph plan) and the layout of
  // the device blob: [status (256 B)] [work] [merge] [refs] [append rows] [kv_indices]
  struct Sizes {
    int64_t cap_work = 0, cap_merge = 0, cap_refs = 0, cap_tokens = 0, cap_idx = 0, cap_ws_rows = 0;
    size_t off_work = 0, off_merge = 0, off_refs = 0, off_append = 0, off_idx = 0, blob_bytes = 0;
  } sz;
  void* d_blob = nullptr;
  bool blob_fresh = false;  // the blob's status word has not been cleared yet
  uint8_t* d_ws = nullptr;  // [ws rows][512] bf16 o, then [ws rows] fp32 lse
  // pinned staging, double-buffered so an update need not wait for the latest upload
  void* h_staging[2] = {nullptr, nullptr};
  size_t staging_cap[2] = {0, 0};
  cudaEvent_t ev_upload[2] = {nullptr, nullptr};
  bool upload_pending[2] = {false, false};
  int64_t uploads = 0;
  size_t blob_cap = 0, ws_cap = 0;  // capacities of the pooled device buffers
  cudaEvent_t ev_last = nullptr;
  int32_t* h_status = nullptr;  // host-mapped mirror of the status word (see status_slot_take)
  // kernel timing ring (MLA_DEBUG_KERNEL_TIMING): 3 events per run
  static constexpr int kRing = 256;
  cudaEvent_t* ring = nullptr;
  int64_t runs = 0;

  int32_t* d_status() const { return static_cast<int32_t*>(d_blob); }
  const WorkItem* d_work() const { return reinterpret_cast<const WorkItem*>(static_cast<uint8_t*>(d_blob) + sz.off_work); }
  const MergeItem* d_merge() const {
    return reinterpret_cast<const MergeItem*>(static_cast<uint8_t*>(d_blob) + sz.off_merge);
  }
  const int32_t* d_refs() const { return reinterpret_cast<const int32_t*>(static_cast<uint8_t*>(d_blob) + sz.off_refs); }
  const int32_t* d_append() const {
    return reinterpret_cast<const int32_t*>(static_cast<uint8_t*>(d_blob) + sz.off_append);
  }
  const int32_t* d_kv_indices() const {
    return reinterpret_cast<const int32_t*>(static_cast<uint8_t*>(d_blob) + sz.off_idx);
  }
};

namespace {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Buffers of destroyed plans are kept for reuse, so that a caller that plans every step
// (a serving loop whose batch changes each step) allocates nothing once the pool is
// warm: cudaMalloc, cudaMallocHost and their frees synchronise and cost milliseconds.
// Device buffers are keyed by device, pinned host buffers are not; capacities are powers
// of two from 64 KB up, and at most kPoolKeep buffers of each kind and device are kept.
enum PoolKind { kPoolDevice = 0, kPoolPinned = 1 };
struct PoolEntry {
  void* ptr;
  size_t cap;
  int device;
  int kind;
};
std::mutex g_pool_mutex;
std::vector<PoolEntry>* g_pool = new std::vector<PoolEntry>();  // never destroyed: usable during exit
constexpr int kPoolKeep = 8;

void* pool_take(int kind, int device, size_t bytes, size_t* cap) {
  {
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    int best = -1;
    for (int i = 0; i < static_cast<int>(g_pool->size()); ++i) {
      const PoolEntry& e = (*g_pool)[i];
      if (e.kind == kind && (kind == kPoolPinned || e.device == device) && e.cap >= bytes &&
          (best < 0 || e.cap < (*g_pool)[best].cap))
        best = i;
    }
    if (best >= 0) {
      void* ptr = (*g_pool)[best].ptr;
      *cap = (*g_pool)[best].cap;
      g_pool->erase(g_pool->begin() + best);
      return ptr;
    }
  }
  size_t c = size_t(64) << 10;
  while (c < bytes) c <<= 1;
  void* ptr = nullptr;
  const cudaError_t e = kind == kPoolDevice ? cudaMalloc(&ptr, c) : cudaMallocHost(&ptr, c);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  *cap = c;
  return ptr;
}

void pool_give(int kind, int device, void* ptr, size_t cap) {
  if (!ptr) return;
  PoolEntry evict{nullptr, 0, device, kind};
  {
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    g_pool->push_back(PoolEntry{ptr, cap, device, kind});
    int n = 0, smallest = -1;
    for (int i = 0; i < static_cast<int>(g_pool->size()); ++i) {
      const PoolEntry& e = (*g_pool)[i];
      if (e.kind != kind || (kind == kPoolDevice && e.device != device)) continue;
      ++n;
      if (smallest < 0 || e.cap < (*g_pool)[smallest].cap) smallest = i;
    }
    if (n > kPoolKeep) {
      evict = (*g_pool)[smallest];
      g_pool->erase(g_pool->begin() + smallest);
    }
  }
  if (evict.ptr) {
    if (evict.kind == kPoolDevice) {
      int cur = -1;
      cudaGetDevice(&cur);
      cudaSetDevice(evict.device);
      cudaFree(evict.ptr);
      cudaSetDevice(cur);
    } else {
      cudaFreeHost(evict.ptr);
    }
  }
}

// The plan's events (last run, uploads) come from a per-device list as well: creating
// and destroying them costs microseconds of host time on every plan.  At most
// kEventKeep events per device are kept.
struct PooledEvent {
  cudaEvent_t ev;
  int device;
};
std::vector<PooledEvent>* g_events = new std::vector<PooledEvent>();  // never destroyed
constexpr int kEventKeep = 32;

cudaEvent_t event_take(int device) {
  {
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    for (size_t i = g_events->size(); i-- > 0;)
      if ((*g_events)[i].device == device) {
        const cudaEvent_t e = (*g_events)[i].ev;
        g_events->erase(g_events->begin() + static_cast<std::ptrdiff_t>(i));
        return e;
      }
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

// The event must have completed (the plan was quiesced).
void event_give(int device, cudaEvent_t e) {
  if (!e) return;
  {
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    int n = 0;
    for (const PooledEvent& x : *g_events) n += x.device == device;
    if (n < kEventKeep) {
      g_events->push_back(PooledEvent{e, device});
      return;
    }
  }
  cudaEventDestroy(e);
}

// Host-visible mirrors of the plans' status words.  The attention kernel that records a
// plan's first error also stores it here (mapped pinned memory), so mla_plan_check reads
// it once the launch has finished, with no copy: a synchronous device-to-host copy of the
// device word would queue behind the device-to-host copies other streams have pending
// (a serving loop's result downloads) and wait for them.  Slots lie 64 bytes apart in
// 4 KB slabs that are never freed; the slab's device address must equal its host
// address (unified addressing).
std::vector<int32_t*>* g_status_free = new std::vector<int32_t*>();  // never destroyed
constexpr size_t kStatusSlab = 4096, kStatusStride = 64;

int32_t* status_slot_take() {
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  if (g_status_free->empty()) {
    void* slab = nullptr;
    void* dev = nullptr;
    if (cudaHostAlloc(&slab, kStatusSlab, cudaHostAllocPortable | cudaHostAllocMapped) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if (cudaHostGetDevicePointer(&dev, slab, 0) != cudaSuccess || dev != slab) {
      cudaGetLastError();
      cudaFreeHost(slab);
      return nullptr;
    }
    for (size_t off = kStatusSlab; off >= kStatusStride; off -= kStatusStride)
      g_status_free->push_back(reinterpret_cast<int32_t*>(static_cast<uint8_t*>(slab) + off - kStatusStride));
  }
  int32_t* slot = g_status_free->back();
  g_status_free->pop_back();
  *reinterpret_cast<volatile int32_t*>(slot) = 0;
  return slot;
}

void status_slot_give(int32_t* slot) {
  if (!slot) return;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  g_status_free->push_back(slot);
}

// Wait until no launch or upload of the plan can still be reading its buffers.
void quiesce(mla_plan_s* p) {
  if (p->captured) {
    // graphs captured from the plan may have replayed on any stream
    cudaDeviceSynchronize();
    cudaGetLastError();
  } else if (p->ev_last) {
    cudaEventSynchronize(p->ev_last);
  }
  for (int i = 0; i < 2; ++i)
    if (p->ev_upload[i] && p->upload_pending[i]) cudaEventSynchronize(p->ev_upload[i]);
}

void free_plan(mla_plan_s* p) {
  if (!p) return;
  if (!p->host_only) {
    quiesce(p);
    event_give(p->device, p->ev_last);
    for (int i = 0; i < 2; ++i) event_give(p->device, p->ev_upload[i]);
    if (p->ring) {
      for (int i = 0; i < 3 * mla_plan_s::kRing; ++i)
        if (p->ring[i]) cudaEventDestroy(p->ring[i]);
      delete[] p->ring;
    }
    pool_give(kPoolDevice, p->device, p->d_blob, p->blob_cap);
    pool_give(kPoolDevice, p->device, p->d_ws, p->ws_cap);
    for (int i = 0; i < 2; ++i) pool_give(kPoolPinned, -1, p->h_staging[i], p->staging_cap[i]);
    status_slot_give(p->h_status);
  }
  delete p;
}

// The request a plan's options describe, for its current tables.
PlanRequest request_of(const mla_plan_s* p, int32_t batch, const int32_t* qo, const int32_t* kvp, const int32_t* kvi,
                       const int32_t* last) {
  PlanRequest r;
  r.d = p->dims;
  r.batch = batch;
  r.qo_indptr = qo;
  r.kv_indptr = kvp;
  r.kv_indices = kvi;
  r.last_page_len = last;
  r.causal = p->causal;
  r.context_only = p->opts.context_only != 0;
  r.cascade = p->opts.cascade != 0;
  r.split_keys = p->opts.split_keys;
  r.num_sms = p->opts.num_sms;
  if (p->graph)
    graph_bounds(p->dims.num_heads, p->opts.graph_max_batch, p->opts.graph_max_tokens, p->opts.num_sms, &r);
  return r;
}

// Bucket bounds of a graph plan: the step must fit them.
bool fits_bucket(const mla_plan_s* p, int32_t batch, const int32_t* qo, const int32_t* kvp) {
  if (!p->graph) return true;
  if (batch < 0 || batch > p->opts.graph_max_batch || !qo || !kvp) return false;
  return qo[batch] <= p->opts.graph_max_tokens && kvp[batch] <= p->opts.graph_max_page_ids;
}

// Device list capacities and blob offsets: exact sizes, or the bucket's bounds.
void size_lists(mla_plan_s* p, const PlanLayout& L, int64_t n_idx) {
  if (p->graph) {
    PlanRequest r;
    graph_bounds(p->dims.num_heads, p->opts.graph_max_batch, p->opts.graph_max_tokens, p->opts.num_sms, &r);
    p->sz.cap_work = r.max_work;
    p->sz.cap_merge = r.max_merge;
    p->sz.cap_refs = r.max_refs;
    p->sz.cap_ws_rows = r.max_ws_rows;
    p->sz.cap_tokens = p->opts.graph_max_tokens;
    p->sz.cap_idx = p->opts.graph_max_page_ids;
  } else {
    p->sz.cap_work = static_cast<int64_t>(L.work.size());
    p->sz.cap_merge = static_cast<int64_t>(L.merge.size());
    p->sz.cap_refs = static_cast<int64_t>(L.refs.size());
    p->sz.cap_ws_rows = L.ws_rows;
    p->sz.cap_tokens = L.total_tokens;
    p->sz.cap_idx = n_idx;
  }
  p->sz.off_work = 256;
  p->sz.off_merge = align_up(p->sz.off_work + sizeof(WorkItem) * p->sz.cap_work, 256);
  p->sz.off_refs = align_up(p->sz.off_merge + sizeof(MergeItem) * p->sz.cap_merge, 256);
  p->sz.off_append = align_up(p->sz.off_refs + sizeof(int32_t) * p->sz.cap_refs, 256);
  p->sz.off_idx = align_up(p->sz.off_append + sizeof(int32_t) * p->sz.cap_tokens, 256);
  p->sz.blob_bytes = align_up(p->sz.off_idx + sizeof(int32_t) * p->sz.cap_idx, 256);
}

// Make sure the pooled device buffers hold the current capacities.  Growing a buffer
// waits for the plan's last run first (its kernels may still read the old one).
mla_status reserve_device(mla_plan_s* p) {
  const size_t ws = static_cast<size_t>(p->sz.cap_ws_rows) * kWsRowBytes;
  const bool grow_blob = p->sz.blob_bytes > p->blob_cap, grow_ws = ws > p->ws_cap;
  if (!grow_blob && !grow_ws) return MLA_OK;
  if (p->d_blob || p->d_ws) quiesce(p);
  // the workspace first: if the blob cannot grow afterwards, the plan still holds its
  // previous step intact (a larger workspace is harmless)
  if (grow_ws) {
    size_t cap = 0;
    void* nw = pool_take(kPoolDevice, p->device, ws, &cap);
    if (!nw) return MLA_ERR_OUT_OF_MEMORY;
    pool_give(kPoolDevice, p->device, p->d_ws, p->ws_cap);
    p->d_ws = static_cast<uint8_t*>(nw);
    p->ws_cap = cap;
  }
  if (grow_blob) {
    size_t cap = 0;
    void* nb = pool_take(kPoolDevice, p->device, p->sz.blob_bytes, &cap);
    if (!nb) return MLA_ERR_OUT_OF_MEMORY;
    pool_give(kPoolDevice, p->device, p->d_blob, p->blob_cap);
    p->d_blob = nb;
    p->blob_cap = cap;
    p->blob_fresh = true;  // the next upload clears its status word
  }
  return MLA_OK;
}

// Stage the current layout and page table in pinned memory and enqueue their upload
// (everything after the status word).  Unused capacity of a graph plan is filled with
// empty work and merge items and append rows of -1.
mla_status upload(mla_plan_s* p, const int32_t* kv_indices, int64_t n_idx, cudaStream_t s) {
  const int k = static_cast<int>(p->uploads & 1);
  if (p->upload_pending[k]) {
    if (cudaEventSynchronize(p->ev_upload[k]) != cudaSuccess) return MLA_ERR_CUDA;
    p->upload_pending[k] = false;
  }
  if (p->staging_cap[k] < p->sz.blob_bytes) {
    pool_give(kPoolPinned, -1, p->h_staging[k], p->staging_cap[k]);
    p->h_staging[k] = pool_take(kPoolPinned, -1, p->sz.blob_bytes, &p->staging_cap[k]);
    if (!p->h_staging[k]) {
      p->staging_cap[k] = 0;
      return MLA_ERR_OUT_OF_MEMORY;
    }
  }
  if (!p->ev_upload[k] && !(p->ev_upload[k] = event_take(p->device))) return MLA_ERR_CUDA;
  const PlanLayout& L = p->layout;
  uint8_t* h = static_cast<uint8_t*>(p->h_staging[k]);
  std::memset(h + p->sz.off_work, 0, p->sz.off_refs - p->sz.off_work);  // empty work and merge slots
  if (!L.work.empty()) std::memcpy(h + p->sz.off_work, L.work.data(), sizeof(WorkItem) * L.work.size());
  if (!L.merge.empty()) std::memcpy(h + p->sz.off_merge, L.merge.data(), sizeof(MergeItem) * L.merge.size());
  if (!L.refs.empty()) std::memcpy(h + p->sz.off_refs, L.refs.data(), sizeof(int32_t) * L.refs.size());
  int32_t* app = reinterpret_cast<int32_t*>(h + p->sz.off_append);
  for (int64_t t = 0; t < p->sz.cap_tokens; ++t)
    app[t] = t < static_cast<int64_t>(L.append_rows.size()) ? L.append_rows[t] : -1;
  if (n_idx > 0) std::memcpy(h + p->sz.off_idx, kv_indices, sizeof(int32_t) * n_idx);
  // a fresh blob's status word is cleared by the same copy; later uploads leave it alone
  // (a run still in flight may be reporting a timeout there)
  const size_t from = p->blob_fresh ? 0 : p->sz.off_work;
  if (p->blob_fresh) std::memset(h, 0, p->sz.off_work);
  uint8_t* d = static_cast<uint8_t*>(p->d_blob);
  if (cudaMemcpyAsync(d + from, h + from, p->sz.blob_bytes - from, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaEventRecord(p->ev_upload[k], s) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  p->upload_pending[k] = true;
  p->blob_fresh = false;
  ++p->uploads;
  return MLA_OK;
}

void remember_tables(mla_plan_s* p, int32_t batch, const int32_t* qo, const int32_t* kvp, const int32_t* kvi,
                     const int32_t* last) {
  p->batch = batch;
  p->fp_qo.assign(qo, qo + batch + 1);
  p->fp_kvp.assign(kvp, kvp + batch + 1);
  const int32_t n_idx = batch > 0 ? kvp[batch] : 0;
  if (n_idx > 0)
    p->fp_kvi.assign(kvi, kvi + n_idx);
  else
    p->fp_kvi.clear();
  if (batch > 0)
    p->fp_last.assign(last, last + batch);
  else
    p->fp_last.clear();
}

bool same_tables(const mla_plan_s* p, int32_t batch, const int32_t* qo, const int32_t* kvp, const int32_t* kvi,
                 const int32_t* last) {
  if (batch != p->batch || batch < 0 || !qo || !kvp) return false;
  if (std::memcmp(qo, p->fp_qo.data(), sizeof(int32_t) * (batch + 1)) != 0) return false;
  if (std::memcmp(kvp, p->fp_kvp.data(), sizeof(int32_t) * (batch + 1)) != 0) return false;
  if (batch > 0 && (!last || std::memcmp(last, p->fp_last.data(), sizeof(int32_t) * batch) != 0)) return false;
  const int32_t n_idx = batch > 0 ? kvp[batch] : 0;
  if (n_idx != static_cast<int32_t>(p->fp_kvi.size())) return false;
  if (n_idx > 0 && (!kvi || std::memcmp(kvi, p->fp_kvi.data(), sizeof(int32_t) * n_idx) != 0)) return false;
  return true;
}

bool stream_capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return cs == cudaStreamCaptureStatusActive;
}

inline bool misaligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) != 0; }

// Shared checks and parameter set-up of the attention launch.
mla_status attention_launch_of(mla_plan_t p, const void* q_nope, const void* q_pe, const void* cache, void* out,
                               float* lse, AttnLaunch* a) {
  const bool rope = p->dims.rope_dim > 0;  // without kpe, q_pe is not read (may be NULL)
  if (!q_nope || (rope && !q_pe) || !cache || !out) return MLA_ERR_INVALID_ARGUMENT;
  if (misaligned16(q_nope) || (rope && misaligned16(q_pe)) || misaligned16(cache) || misaligned16(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return MLA_ERR_INVALID_ARGUMENT;
  AttnParams& ap = a->p;
  ap.work = p->d_work();
  ap.kv_indices = p->d_kv_indices();
  ap.out = out;
  ap.lse = lse;
  ap.ws_o = p->d_ws;
  ap.ws_lse = p->d_ws ? reinterpret_cast<float*>(p->d_ws + static_cast<size_t>(p->sz.cap_ws_rows) * kWsRowOBytes)
                      : nullptr;
  ap.status = p->d_status();
  ap.status_mirror = p->h_status;
  ap.scale_log2 = p->dims.sm_scale * 1.4426950408889634f;
  ap.num_heads = p->dims.num_heads;
  ap.page_size = p->dims.page_size;
  ap.rope_dim = p->dims.rope_dim;
  ap.timeout_ns = p->opts.wait_timeout_ns ? p->opts.wait_timeout_ns : 4000000000ull;
  ap.debug_flags = p->opts.debug_flags;
  a->q_nope = q_nope;
  a->q_pe = q_pe;
  a->cache = cache;
  a->rows = static_cast<uint64_t>(p->sz.cap_tokens) * p->dims.num_heads;
  a->cache_rows = static_cast<uint64_t>(p->dims.num_pages) * p->dims.page_size;
  a->num_work = static_cast<int>(p->sz.cap_work);
  a->wait_prior_grid = false;
  return MLA_OK;
}

mla_status check_device(mla_plan_t p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) return MLA_ERR_INVALID_ARGUMENT;
  return MLA_OK;
}

mla_status append_launch_of(mla_plan_t p, const void* kv_new, void* cache, AppendParams* ap, int* n_tokens) {
  if (!kv_new || !cache || misaligned16(kv_new) || misaligned16(cache)) return MLA_ERR_INVALID_ARGUMENT;
  if (!p->layout.append_ok) return MLA_ERR_INVALID_ARGUMENT;
  ap->rows = p->d_append();
  ap->src = kv_new;
  ap->cache = cache;
  ap->width = kCkv + p->dims.rope_dim;
  *n_tokens = static_cast<int>(p->sz.cap_tokens);
  return MLA_OK;
}

// Attention (and the merge of split tiles), with the plan's event bookkeeping.
mla_status enqueue_attention(mla_plan_t p, AttnLaunch& a, cudaStream_t s) {
  const bool capturing = stream_capturing(s);
  if (capturing) p->captured = true;
  cudaEvent_t* ev = (p->ring && !capturing) ? p->ring + 3 * (p->runs % mla_plan_s::kRing) : nullptr;
  if (ev && cudaEventRecord(ev[0], s) != cudaSuccess) return MLA_ERR_CUDA;
  if (launch_attention(a, s) != cudaSuccess) return MLA_ERR_CUDA;
  if (ev && cudaEventRecord(ev[1], s) != cudaSuccess) return MLA_ERR_CUDA;
  // a graph plan always launches the merge: a later step of the bucket may split
  if (p->sz.cap_merge > 0 && (p->graph || !p->layout.merge.empty())) {
    MergeParams mp{p->d_merge(), p->d_refs(), a.p.ws_o, a.p.ws_lse, a.p.out, a.p.lse};
    if (launch_merge(mp, static_cast<int>(p->sz.cap_merge), s) != cudaSuccess) return MLA_ERR_CUDA;
  }
  if (ev) {
    if (cudaEventRecord(ev[2], s) != cudaSuccess) return MLA_ERR_CUDA;
    ++p->runs;
  }
  if (!capturing && cudaEventRecord(p->ev_last, s) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_supports(int kv_lora_rank, int rope_dim, int num_heads, int page_size) {
  return shape_supported(kv_lora_rank, rope_dim, num_heads, page_size) ? 1 : 0;
}

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_OUT_OF_MEMORY: return "out of memory";
    case MLA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

mla_status mla_plan(const mla_dims* dims, int32_t batch, const int32_t* qo_indptr, const int32_t* kv_indptr,
                    const int32_t* kv_indices, const int32_t* last_page_len, int32_t causal, void* stream,
                    const mla_plan_options* opts, mla_plan_t* out_plan) {
  if (!out_plan) return MLA_ERR_INVALID_ARGUMENT;
  *out_plan = nullptr;
  if (!dims || (causal != 0 && causal != 1)) return MLA_ERR_INVALID_ARGUMENT;
  mla_plan_s* p = new (std::nothrow) mla_plan_s();
  if (!p) return MLA_ERR_OUT_OF_MEMORY;
  p->dims = *dims;
  p->causal = causal != 0;
  if (opts) p->opts = *opts;
  p->host_only = p->opts.host_only != 0;
  const mla_plan_options& o = p->opts;
  const int graph_fields = (o.graph_max_batch > 0) + (o.graph_max_tokens > 0) + (o.graph_max_page_ids > 0);
  if ((graph_fields != 0 && graph_fields != 3) || o.graph_max_batch < 0 || o.graph_max_tokens < 0 ||
      o.graph_max_page_ids < 0 || (o.context_only != 0 && o.context_only != 1) ||
      (o.cascade != 0 && o.cascade != 1)) {
    free_plan(p);
    return MLA_ERR_INVALID_ARGUMENT;
  }
  p->graph = graph_fields == 3;

  int num_sms = p->opts.num_sms;
  if (!p->host_only) {
    if (cudaGetDevice(&p->device) != cudaSuccess) { free_plan(p); return MLA_ERR_CUDA; }
    if (num_sms <= 0) {
      if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess) {
        free_plan(p);
        return MLA_ERR_CUDA;
      }
    }
  } else if (num_sms <= 0) {
    num_sms = 148;
  }
  p->opts.num_sms = num_sms;

  if (!fits_bucket(p, batch, qo_indptr, kv_indptr)) { free_plan(p); return MLA_ERR_INVALID_ARGUMENT; }
  mla_status st = build_layout(request_of(p, batch, qo_indptr, kv_indptr, kv_indices, last_page_len), &p->layout);
  if (st != MLA_OK) { free_plan(p); return st; }
  remember_tables(p, batch, qo_indptr, kv_indptr, kv_indices, last_page_len);
  if (p->host_only) { *out_plan = p; return MLA_OK; }

  // ---- device buffers owned by the plan, uploaded through plan-owned pinned staging
  const int64_t n_idx = batch > 0 ? kv_indptr[batch] : 0;
  size_lists(p, p->layout, n_idx);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = reserve_device(p);
  if (st != MLA_OK) { free_plan(p); return st; }
  if (p->opts.debug_flags & MLA_DEBUG_KERNEL_TIMING) {
    p->ring = new (std::nothrow) cudaEvent_t[3 * mla_plan_s::kRing]();
    if (!p->ring) { free_plan(p); return MLA_ERR_OUT_OF_MEMORY; }
    for (int i = 0; i < 3 * mla_plan_s::kRing; ++i)
      if (cudaEventCreate(&p->ring[i]) != cudaSuccess) { cudaGetLastError(); free_plan(p); return MLA_ERR_CUDA; }
  }
  if (!(p->ev_last = event_take(p->device)) || !(p->h_status = status_slot_take())) {
    free_plan(p);
    return MLA_ERR_CUDA;
  }
  st = upload(p, kv_indices, n_idx, s);
  if (st != MLA_OK || cudaEventRecord(p->ev_last, s) != cudaSuccess) {
    cudaGetLastError();
    free_plan(p);
    return st != MLA_OK ? st : MLA_ERR_CUDA;
  }
  *out_plan = p;
  return MLA_OK;
}

mla_status mla_plan_update(mla_plan_t p, int32_t batch, const int32_t* qo_indptr, const int32_t* kv_indptr,
                           const int32_t* kv_indices, const int32_t* last_page_len, void* stream,
                           int32_t* reused) {
  if (reused) *reused = 0;
  if (!p) return MLA_ERR_INVALID_ARGUMENT;
  if (same_tables(p, batch, qo_indptr, kv_indptr, kv_indices, last_page_len)) {
    if (reused) *reused = 1;
    return MLA_OK;
  }
  if (!fits_bucket(p, batch, qo_indptr, kv_indptr)) return MLA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!p->host_only) {
    if (check_device(p) != MLA_OK || stream_capturing(s)) return MLA_ERR_INVALID_ARGUMENT;
  }
  // The new layout is built in the spare one (whose vectors keep their capacity from
  // earlier steps), then the two are swapped.
  PlanLayout& L = p->spare;
  mla_status st = build_layout(request_of(p, batch, qo_indptr, kv_indptr, kv_indices, last_page_len), &L);
  if (st != MLA_OK) return st;
  const int64_t n_idx = batch > 0 ? kv_indptr[batch] : 0;
  if (p->host_only) {
    std::swap(p->layout, p->spare);
    remember_tables(p, batch, qo_indptr, kv_indptr, kv_indices, last_page_len);
    return MLA_OK;
  }
  // Size the lists for the new step; a graph plan's sizes are its bucket's and fixed.
  const mla_plan_s::Sizes saved = p->sz;
  size_lists(p, L, n_idx);
  st = reserve_device(p);
  if (st != MLA_OK) {
    p->sz = saved;
    return st;
  }
  std::swap(p->layout, p->spare);
  st = upload(p, kv_indices, n_idx, s);
  if (st != MLA_OK) {
    std::swap(p->layout, p->spare);  // the plan keeps describing its previous step
    return st;
  }
  remember_tables(p, batch, qo_indptr, kv_indptr, kv_indices, last_page_len);
  if (cudaEventRecord(p->ev_last, s) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status mla_run(mla_plan_t p, const void* q_nope, const void* q_pe, const void* cache, void* out, float* lse,
                   void* stream) {
  if (!p || p->host_only) return MLA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->layout.work.empty() && !p->graph) return MLA_OK;
  if (check_device(p) != MLA_OK) return MLA_ERR_INVALID_ARGUMENT;
  AttnLaunch a;
  mla_status st = attention_launch_of(p, q_nope, q_pe, cache, out, lse, &a);
  if (st != MLA_OK) return st;
  return enqueue_attention(p, a, s);
}

mla_status mla_append_kv(mla_plan_t p, const void* kv_new, void* cache, void* stream) {
  if (!p || p->host_only) return MLA_ERR_INVALID_ARGUMENT;
  if (check_device(p) != MLA_OK) return MLA_ERR_INVALID_ARGUMENT;
  AppendParams ap;
  int n = 0;
  mla_status st = append_launch_of(p, kv_new, cache, &ap, &n);
  if (st != MLA_OK) return st;
  if (n == 0) return MLA_OK;
  return launch_append(ap, n, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_run_append(mla_plan_t p, const void* q_nope, const void* q_pe, const void* kv_new, void* cache,
                          void* out, float* lse, void* stream) {
  if (!p || p->host_only) return MLA_ERR_INVALID_ARGUMENT;
  if (check_device(p) != MLA_OK) return MLA_ERR_INVALID_ARGUMENT;
  AppendParams app;
  int n = 0;
  mla_status st = append_launch_of(p, kv_new, cache, &app, &n);
  if (st != MLA_OK) return st;
  const bool attend = !p->layout.work.empty() || p->graph;
  AttnLaunch a;
  if (attend) {
    st = attention_launch_of(p, q_nope, q_pe, cache, out, lse, &a);
    if (st != MLA_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n > 0) {
    if (launch_append(app, n, s) != cudaSuccess) return MLA_ERR_CUDA;
    a.wait_prior_grid = true;  // only the key loads wait for the append's writes
  }
  if (!attend) return MLA_OK;
  return enqueue_attention(p, a, s);
}

mla_status mla_merge_state(const void* out_a, const float* lse_a, const void* out_b, const float* lse_b, void* out,
                           float* lse, int64_t rows, void* stream) {
  if (rows < 0) return MLA_ERR_INVALID_ARGUMENT;
  if (rows == 0) return MLA_OK;
  if (!out_a || !lse_a || !out_b || !lse_b || !out || misaligned16(out_a) || misaligned16(out_b) ||
      misaligned16(out) || (reinterpret_cast<uintptr_t>(lse_a) & 3u) || (reinterpret_cast<uintptr_t>(lse_b) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return MLA_ERR_INVALID_ARGUMENT;
  if (rows > (int64_t(1) << 40)) return MLA_ERR_INVALID_ARGUMENT;
  MergeStateParams mp{out_a, lse_a, out_b, lse_b, out, lse, rows};
  return launch_merge_state(mp, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_plan_check(mla_plan_t p) {
  if (!p) return MLA_ERR_INVALID_ARGUMENT;
  if (p->host_only) return MLA_OK;
  if (p->captured) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
  } else if (cudaEventSynchronize(p->ev_last) != cudaSuccess) {
    return MLA_ERR_CUDA;
  }
  // the launches have finished: the mirror holds the first error they recorded
  const int32_t st = *reinterpret_cast<volatile int32_t*>(p->h_status);
  if (st != 0) {
    // The bits above the low byte name the wait that gave up (diagnostics only).
    if (std::getenv("MLA_DEBUG_STATUS")) std::fprintf(stderr, "mla: device status word 0x%x\n", st);
    if (cudaMemset(p->d_status(), 0, sizeof(st)) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
    *reinterpret_cast<volatile int32_t*>(p->h_status) = 0;
    return static_cast<mla_status>(st & 0xff);
  }
  return MLA_OK;
}

mla_status mla_plan_get_info(mla_plan_t p, mla_plan_info* info) {
  if (!p || !info) return MLA_ERR_INVALID_ARGUMENT;
  info->batch = p->batch;
  info->total_tokens = p->layout.total_tokens;
  info->num_work = static_cast<int32_t>(p->layout.work.size());
  info->num_merge = static_cast<int32_t>(p->layout.merge.size());
  info->num_partials = p->layout.num_partials;
  info->num_sms = p->opts.num_sms;
  info->workspace_bytes = static_cast<int64_t>(p->layout.ws_rows) * static_cast<int64_t>(kWsRowBytes);
  info->num_merge_refs = static_cast<int32_t>(p->layout.refs.size());
  info->num_cascade = p->layout.num_cascade;
  info->graph = p->graph ? 1 : 0;
  if (p->graph) {
    PlanRequest r;
    graph_bounds(p->dims.num_heads, p->opts.graph_max_batch, p->opts.graph_max_tokens, p->opts.num_sms, &r);
    info->work_capacity = r.max_work;
  } else {
    info->work_capacity = info->num_work;
  }
  return MLA_OK;
}

mla_status mla_plan_describe(mla_plan_t p, int32_t* kv_len, int32_t* work, int32_t* merge, int32_t* refs) {
  if (!p) return MLA_ERR_INVALID_ARGUMENT;
  if (kv_len && p->batch > 0) std::memcpy(kv_len, p->layout.kv_len.data(), sizeof(int32_t) * p->batch);
  if (work && !p->layout.work.empty())
    std::memcpy(work, p->layout.work.data(), sizeof(WorkItem) * p->layout.work.size());
  if (merge && !p->layout.merge.empty())
    std::memcpy(merge, p->layout.merge.data(), sizeof(MergeItem) * p->layout.merge.size());
  if (refs && !p->layout.refs.empty()) std::memcpy(refs, p->layout.refs.data(), sizeof(int32_t) * p->layout.refs.size());
  return MLA_OK;
}

mla_status mla_plan_kernel_times(mla_plan_t p, int32_t capacity, float* attn_ms, float* merge_ms,
                                 int32_t* count) {
  if (!p || !p->ring || capacity < 0 || !count || (capacity > 0 && (!attn_ms || !merge_ms)))
    return MLA_ERR_INVALID_ARGUMENT;
  *count = 0;
  const int64_t have = p->runs < mla_plan_s::kRing ? p->runs : mla_plan_s::kRing;
  const int64_t n = have < capacity ? have : capacity;
  if (n == 0) return MLA_OK;
  if (cudaEventSynchronize(p->ring[3 * ((p->runs - 1) % mla_plan_s::kRing) + 2]) != cudaSuccess)
    return MLA_ERR_CUDA;
  for (int64_t i = 0; i < n; ++i) {
    const cudaEvent_t* ev = p->ring + 3 * ((p->runs - n + i) % mla_plan_s::kRing);
    if (cudaEventElapsedTime(&attn_ms[i], ev[0], ev[1]) != cudaSuccess ||
        cudaEventElapsedTime(&merge_ms[i], ev[1], ev[2]) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  *count = static_cast<int32_t>(n);
  return MLA_OK;
}

void mla_plan_destroy(mla_plan_t p) { free_plan(p); }

}  // extern "C"

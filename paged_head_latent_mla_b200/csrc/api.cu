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
  int device = -1;
  bool host_only = false;
  // one device blob: [status (256 B)] [work] [merge] [kv_indices]
  void* d_blob = nullptr;
  int32_t* d_status = nullptr;
  WorkItem* d_work = nullptr;
  MergeItem* d_merge = nullptr;
  int32_t* d_kv_indices = nullptr;
  uint8_t* d_ws = nullptr;  // [partials][128][512] bf16 o, then [partials][128] fp32 lse
  void* h_staging = nullptr;
  size_t blob_cap = 0, ws_cap = 0, staging_cap = 0;  // capacities of the pooled buffers
  cudaEvent_t ev_last = nullptr;
  // kernel timing ring (MLA_DEBUG_KERNEL_TIMING): 3 events per run
  static constexpr int kRing = 256;
  cudaEvent_t* ring = nullptr;
  int64_t runs = 0;
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

void free_plan(mla_plan_s* p) {
  if (!p) return;
  if (!p->host_only) {
    // the buffers may still be in use by this plan's last launches
    if (p->ev_last) {
      cudaEventSynchronize(p->ev_last);
      cudaEventDestroy(p->ev_last);
    }
    if (p->ring) {
      for (int i = 0; i < 3 * mla_plan_s::kRing; ++i)
        if (p->ring[i]) cudaEventDestroy(p->ring[i]);
      delete[] p->ring;
    }
    pool_give(kPoolDevice, p->device, p->d_blob, p->blob_cap);
    pool_give(kPoolDevice, p->device, p->d_ws, p->ws_cap);
    pool_give(kPoolPinned, -1, p->h_staging, p->staging_cap);
  }
  delete p;
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
  p->batch = batch;
  p->causal = causal != 0;
  if (opts) p->opts = *opts;
  p->host_only = p->opts.host_only != 0;

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

  mla_status st = build_layout(*dims, batch, qo_indptr, kv_indptr, kv_indices, last_page_len, p->causal,
                               p->opts.split_keys, num_sms, &p->layout);
  if (st != MLA_OK) { free_plan(p); return st; }
  if (p->host_only) { *out_plan = p; return MLA_OK; }

  // ---- device buffers owned by the plan, uploaded through plan-owned pinned staging
  const size_t n_idx = batch > 0 ? static_cast<size_t>(kv_indptr[batch]) : 0;
  const size_t off_work = 256;
  const size_t off_merge = align_up(off_work + sizeof(WorkItem) * p->layout.work.size(), 256);
  const size_t off_idx = align_up(off_merge + sizeof(MergeItem) * p->layout.merge.size(), 256);
  const size_t blob = align_up(off_idx + sizeof(int32_t) * n_idx, 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  p->d_blob = pool_take(kPoolDevice, p->device, blob, &p->blob_cap);
  if (!p->d_blob) { free_plan(p); return MLA_ERR_OUT_OF_MEMORY; }
  p->h_staging = pool_take(kPoolPinned, -1, blob, &p->staging_cap);
  if (!p->h_staging) { free_plan(p); return MLA_ERR_OUT_OF_MEMORY; }
  uint8_t* h = static_cast<uint8_t*>(p->h_staging);
  std::memset(h, 0, off_work);
  if (!p->layout.work.empty()) std::memcpy(h + off_work, p->layout.work.data(), sizeof(WorkItem) * p->layout.work.size());
  if (!p->layout.merge.empty())
    std::memcpy(h + off_merge, p->layout.merge.data(), sizeof(MergeItem) * p->layout.merge.size());
  if (n_idx) std::memcpy(h + off_idx, kv_indices, sizeof(int32_t) * n_idx);
  uint8_t* d = static_cast<uint8_t*>(p->d_blob);
  p->d_status = reinterpret_cast<int32_t*>(d);
  p->d_work = reinterpret_cast<WorkItem*>(d + off_work);
  p->d_merge = reinterpret_cast<MergeItem*>(d + off_merge);
  p->d_kv_indices = reinterpret_cast<int32_t*>(d + off_idx);
  if (p->layout.num_partials > 0) {
    const size_t ws = static_cast<size_t>(p->layout.num_partials) * kPartialBytes;
    p->d_ws = static_cast<uint8_t*>(pool_take(kPoolDevice, p->device, ws, &p->ws_cap));
    if (!p->d_ws) { free_plan(p); return MLA_ERR_OUT_OF_MEMORY; }
  }
  if (p->opts.debug_flags & MLA_DEBUG_KERNEL_TIMING) {
    p->ring = new (std::nothrow) cudaEvent_t[3 * mla_plan_s::kRing]();
    if (!p->ring) { free_plan(p); return MLA_ERR_OUT_OF_MEMORY; }
    for (int i = 0; i < 3 * mla_plan_s::kRing; ++i)
      if (cudaEventCreate(&p->ring[i]) != cudaSuccess) { cudaGetLastError(); free_plan(p); return MLA_ERR_CUDA; }
  }
  if (cudaEventCreateWithFlags(&p->ev_last, cudaEventDisableTiming) != cudaSuccess ||
      cudaMemcpyAsync(p->d_blob, p->h_staging, blob, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaEventRecord(p->ev_last, s) != cudaSuccess) {
    cudaGetLastError();
    free_plan(p);
    return MLA_ERR_CUDA;
  }
  *out_plan = p;
  return MLA_OK;
}

mla_status mla_run(mla_plan_t p, const void* q_nope, const void* q_pe, const void* cache, void* out, float* lse,
                   void* stream) {
  if (!p || p->host_only) return MLA_ERR_INVALID_ARGUMENT;
  const int64_t rows = static_cast<int64_t>(p->layout.total_tokens) * p->dims.num_heads;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->layout.work.empty()) return MLA_OK;
  if (!q_nope || !q_pe || !cache || !out) return MLA_ERR_INVALID_ARGUMENT;
  auto misaligned = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) != 0; };
  if (misaligned(q_nope) || misaligned(q_pe) || misaligned(cache) || misaligned(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return MLA_ERR_INVALID_ARGUMENT;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) return MLA_ERR_INVALID_ARGUMENT;

  AttnLaunch a;
  AttnParams& ap = a.p;
  ap.work = p->d_work;
  ap.kv_indices = p->d_kv_indices;
  ap.out = out;
  ap.lse = lse;
  ap.ws_o = p->d_ws;
  ap.ws_lse = p->d_ws ? reinterpret_cast<float*>(p->d_ws + static_cast<size_t>(p->layout.num_partials) * kPartialOBytes)
                      : nullptr;
  ap.status = p->d_status;
  ap.scale_log2 = p->dims.sm_scale * 1.4426950408889634f;
  ap.num_heads = p->dims.num_heads;
  ap.page_size = p->dims.page_size;
  ap.timeout_ns = p->opts.wait_timeout_ns ? p->opts.wait_timeout_ns : 4000000000ull;
  ap.debug_flags = p->opts.debug_flags;
  a.q_nope = q_nope;
  a.q_pe = q_pe;
  a.cache = cache;
  a.rows = static_cast<uint64_t>(rows);
  a.cache_rows = static_cast<uint64_t>(p->dims.num_pages) * p->dims.page_size;
  a.num_work = static_cast<int>(p->layout.work.size());
  cudaEvent_t* ev = p->ring ? p->ring + 3 * (p->runs % mla_plan_s::kRing) : nullptr;
  if (ev && cudaEventRecord(ev[0], s) != cudaSuccess) return MLA_ERR_CUDA;
  cudaError_t e = launch_attention(a, s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  if (ev && cudaEventRecord(ev[1], s) != cudaSuccess) return MLA_ERR_CUDA;
  if (!p->layout.merge.empty()) {
    MergeParams mp{p->d_merge, ap.ws_o, ap.ws_lse, ap.out, lse};
    e = launch_merge(mp, static_cast<int>(p->layout.merge.size()), s);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
  }
  if (ev) {
    if (cudaEventRecord(ev[2], s) != cudaSuccess) return MLA_ERR_CUDA;
    ++p->runs;
  }
  if (cudaEventRecord(p->ev_last, s) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status mla_plan_check(mla_plan_t p) {
  if (!p) return MLA_ERR_INVALID_ARGUMENT;
  if (p->host_only) return MLA_OK;
  if (cudaEventSynchronize(p->ev_last) != cudaSuccess) return MLA_ERR_CUDA;
  int32_t st = 0;
  if (cudaMemcpy(&st, p->d_status, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (st != 0) {
    // The bits above the low byte name the wait that gave up (diagnostics only).
    if (std::getenv("MLA_DEBUG_STATUS")) std::fprintf(stderr, "mla: device status word 0x%x\n", st);
    if (cudaMemset(p->d_status, 0, sizeof(st)) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
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
  info->workspace_bytes = static_cast<int64_t>(p->layout.num_partials) * static_cast<int64_t>(kPartialBytes);
  return MLA_OK;
}

mla_status mla_plan_describe(mla_plan_t p, int32_t* kv_len, int32_t* work, int32_t* merge) {
  if (!p) return MLA_ERR_INVALID_ARGUMENT;
  if (kv_len && p->batch > 0) std::memcpy(kv_len, p->layout.kv_len.data(), sizeof(int32_t) * p->batch);
  if (work && !p->layout.work.empty())
    std::memcpy(work, p->layout.work.data(), sizeof(WorkItem) * p->layout.work.size());
  if (merge && !p->layout.merge.empty())
    std::memcpy(merge, p->layout.merge.data(), sizeof(MergeItem) * p->layout.merge.size());
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

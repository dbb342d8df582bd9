// Launch interface between the C-ABI layer and the sm_100a kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>

#include <cstdint>

#include "mla_internal.h"

namespace mla {

// Kernel parameters of the attention kernel (the tensor maps travel beside them).
struct AttnParams {
  const WorkItem* work;
  const int32_t* kv_indices;
  const void* q_nope;  // bf16 [T*H, 512] (the kernel reads part of Q directly)
  const void* q_pe;    // bf16 [T*H, 64]; unused when rope_dim == 0
  void* out;         // bf16 [T*H, 512]
  float* lse;        // fp32 [T*H] or nullptr
  void* ws_o;        // bf16 [partials, 128, 512]
  float* ws_lse;     // fp32 [partials, 128]
  int32_t* status;   // device status word
  int32_t* status_mirror;  // host-mapped pinned copy of the first error recorded, or null
  float scale_log2;  // sm_scale * log2(e)
  float nan_guard;   // always NaN: `x != nan_guard` is true for every x, yet the compiler
                     // cannot fold it, so a vote on it waits for x to be computed
  int32_t num_heads;
  int32_t page_size;
  int32_t box_rows;  // rows per KV box: min(page_size, 64)
  int32_t rope_dim;  // kpe width: 64, or 0 (cache rows are then 512 wide)
  uint64_t timeout_ns;
  int32_t debug_flags;
};

// Everything one attention launch needs; the launcher encodes the TMA tensor maps from
// the raw pointers, because their box shapes belong to the kernel's tiling.
struct AttnLaunch {
  AttnParams p;
  const void* q_nope;   // bf16 [rows, 512]
  const void* q_pe;     // bf16 [rows, 64] (null when rope_dim == 0)
  const void* cache;    // bf16 [cache_rows, 512 + rope_dim]
  uint64_t rows;        // T * H
  uint64_t cache_rows;  // num_pages * page_size
  int num_work;         // launch slots (CTA pairs)
  bool wait_prior_grid; // launched as a programmatic dependent of the previous kernel
                        // (an append): the key loads wait for that grid's writes
};

struct MergeParams {
  const MergeItem* merge;
  const int32_t* refs;
  const void* ws_o;
  const float* ws_lse;
  void* out;
  float* lse;
};

// Latent-cache append: token t's row of src goes to cache row rows[t] (skipped if < 0).
struct AppendParams {
  const int32_t* rows;  // [tokens]
  const void* src;      // bf16 [tokens, width]
  void* cache;          // bf16 [cache_rows, width]
  int32_t width;        // 512 + rope_dim
};

// Merge of two attention states by their log-sum-exps.
struct MergeStateParams {
  const void* out_a;
  const float* lse_a;
  const void* out_b;
  const float* lse_b;
  void* out;
  float* lse;  // may be null
  int64_t rows;
};

// cudaErrorInvalidValue when a tensor map cannot be encoded.
cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, int num_merge, cudaStream_t stream);
cudaError_t launch_append(const AppendParams& p, int num_tokens, cudaStream_t stream);
cudaError_t launch_merge_state(const MergeStateParams& p, cudaStream_t stream);

}  // namespace mla

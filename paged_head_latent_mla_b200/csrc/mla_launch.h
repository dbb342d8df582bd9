// Launch interface between the C-ABI layer and the sm_100a kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>

#include <cstdint>

#include "mla_internal.h"

namespace mla {

struct AttnParams {
  const WorkItem* work;
  const int32_t* kv_indices;
  const void* q_nope;  // bf16 [T*H, 512]
  const void* q_pe;    // bf16 [T*H, 64]
  int32_t total_rows;  // T*H
  void* out;       // bf16 [T*H, 512]
  float* lse;      // fp32 [T*H] or nullptr
  float* ws_o;     // fp32 [partials, 128, 512]
  float* ws_lse;   // fp32 [partials, 128]
  int32_t* status; // device status word
  float scale_log2;  // sm_scale * log2(e)
  float nan_guard;   // always NaN: `x != nan_guard` is true for every x, yet the compiler
                     // cannot fold it, so a vote on it waits for x to be computed
  int32_t num_heads;
  int32_t page_size;
  int32_t box_rows;  // min(page_size, 64)
  uint64_t timeout_ns;
  int32_t debug_flags;
};

struct MergeParams {
  const MergeItem* merge;
  const float* ws_o;
  const float* ws_lse;
  void* out;
  float* lse;
};

cudaError_t launch_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_qpe, const CUtensorMap& tm_kv,
                             const CUtensorMap& tm_kpe, const AttnParams& p, int num_work,
                             cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, int num_merge, cudaStream_t stream);

}  // namespace mla

// The two small kernels around the attention: the latent-cache append that precedes it
// and the merge of two attention states that may follow it.
//
// Append (page "mstar.engine.resources.attn.base", AttentionManager.requires_kv_write:
// a layer writes the step's K/V through the KV resource before calling run): every
// token's [ckv | kpe] row (576 wide, or 512 without kpe) is copied to the cache row the
// plan assigned it.  The copy is HBM-bound: 1152 B (1024 B) read and written per token,
// moved as 16-byte vectors, one thread per vector and consecutive threads along a row,
// so that each token row is one contiguous access on both sides.
//
// Merge (page "mstar.engine.resources.attn.flashinfer_mla", FlashInferMLAManager.run:
// the log-sum-exp is returned for merging with another key segment): two states over
// disjoint key sets combine as out = (e^{lse_a-M} out_a + e^{lse_b-M} out_b) / Z,
// lse = M + ln Z with M = max(lse_a, lse_b) and Z the sum of the two weights.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mla_launch.h"
#include "sm100_ptx.cuh"

namespace mla {

namespace {

constexpr int kMaxRowChunks = kLatent * 2 / 16;  // 16-byte pieces per cache row (72, or 64)
constexpr int kAppendTokens = 4;                 // tokens per block

__global__ void __launch_bounds__(kAppendTokens * kMaxRowChunks) mla_append_kernel(const AppendParams p,
                                                                                    int num_tokens) {
  // The attention launched after this grid as its programmatic dependent may start its
  // set-up now; its key loads wait for this grid to finish.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int chunks = p.width / 8;  // blockDim.x == kAppendTokens * chunks
  const int t = blockIdx.x * kAppendTokens + threadIdx.x / chunks;
  const int c = threadIdx.x % chunks;
  if (t >= num_tokens) return;
  const int32_t row = p.rows[t];
  if (row < 0) return;  // an empty slot of a graph plan
  const size_t row_bytes = static_cast<size_t>(p.width) * 2;
  const uint4 v = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.src) + t * row_bytes)[c];
  reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.cache) + static_cast<size_t>(row) * row_bytes)[c] = v;
}

// One warp per row; lane l owns columns [16l, 16l + 16).
__global__ void __launch_bounds__(256) mla_merge_state_kernel(const MergeStateParams p) {
  const int lane = threadIdx.x & 31;
  const float neg_inf = -__int_as_float(0x7f800000);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); r < p.rows; r += stride) {
    const float la = p.lse_a[r], lb = p.lse_b[r];
    const float M = fmaxf(la, lb);
    const size_t off = (static_cast<size_t>(r) * kCkv + 16 * lane) * 2;
    const uint4* a = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.out_a) + off);
    const uint4* b = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.out_b) + off);
    uint4 va[2] = {a[0], a[1]}, vb[2] = {b[0], b[1]};
    uint4 o[2];
    uint32_t* ov = reinterpret_cast<uint32_t*>(o);
    float lse;
    if (M == neg_inf) {  // neither state saw a key
      o[0] = o[1] = make_uint4(0u, 0u, 0u, 0u);
      lse = neg_inf;
    } else {
      const float wa = expf(la - M), wb = expf(lb - M);  // e^{-inf} = 0 drops an empty state
      const float z = wa + wb, inv = 1.f / z;
      const uint32_t* xa = reinterpret_cast<const uint32_t*>(va);
      const uint32_t* xb = reinterpret_cast<const uint32_t*>(vb);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float lo = (wa * __uint_as_float(xa[k] << 16) + wb * __uint_as_float(xb[k] << 16)) * inv;
        const float hi =
            (wa * __uint_as_float(xa[k] & 0xffff0000u) + wb * __uint_as_float(xb[k] & 0xffff0000u)) * inv;
        ov[k] = ptx::pack_bf16x2(lo, hi);
      }
      lse = M + logf(z);
    }
    // every lane has read its columns of both inputs: out may alias either
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + off);
    dst[0] = o[0];
    dst[1] = o[1];
    if (p.lse != nullptr && lane == 0) p.lse[r] = lse;
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, int num_tokens, cudaStream_t stream) {
  if (num_tokens <= 0) return cudaSuccess;
  if (p.width != kCkv && p.width != kLatent) return cudaErrorInvalidValue;
  const int threads = kAppendTokens * (p.width / 8);
  mla_append_kernel<<<(num_tokens + kAppendTokens - 1) / kAppendTokens, threads, 0, stream>>>(p, num_tokens);
  return cudaGetLastError();
}

cudaError_t launch_merge_state(const MergeStateParams& p, cudaStream_t stream) {
  if (p.rows <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (p.rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  mla_merge_state_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla

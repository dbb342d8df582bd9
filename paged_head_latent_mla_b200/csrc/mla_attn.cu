// sm_100a kernels for paged latent attention (absorbed MLA) and the split-KV merge.
//
// What is computed (page "mstar.engine.resources.attn.flashinfer_mla": module
// description, FlashInferMLAWrapper.run, FlashInferMLAManager.run): for each query
// row (token t, head h) of batch row b,
//     s_j = sm_scale * (q_nope[t,h] . ckv_j + q_pe[t,h] . kpe_j),  j < vis(t)
//     out = softmax(s) . ckv           (bf16, [T, H, 512])
//     lse = ln sum_j exp(s_j)          (fp32, [T, H], natural log)
// with the cache rows [ckv | kpe] gathered page by page and causal visibility aligned
// to the end of the row's keys (page "mstar.engine.resources.attn.ragged.wrappers",
// PrefixedPrefillWrapper).
//
// Design (B200):
//  * One work item = a 128-row query tile (128 / H tokens x H heads of one batch row)
//    against a chunk of that row's keys, processed by a cluster of two CTAs on two SMs.
//  * The fp32 output accumulator of 128 rows x 512 columns would fill all 512 TMEM
//    columns of an SM, leaving none for scores.  So the pair splits the latent width:
//    CTA r owns ckv columns [256r, 256r + 256) and kpe columns [32r, 32r + 32), i.e.
//    288 of the 576 contraction columns.  Each CTA TMA-gathers only its columns of
//    every key, so every cache byte crosses HBM once.
//  * Per 64-key tile: each CTA computes a partial S = Q_half . K_half^T (tcgen05,
//    M=128, N=64, K=288) into TMEM; the softmax warps push their partial to the peer
//    over DSMEM, add the peer's partial (fp32 addition commutes, so both CTAs hold
//    bit-identical S), apply mask and online softmax (log2 domain, lazy rescale), and
//    store P as bf16 into TMEM.  Then O_half += P . V_half (tcgen05, A = P from TMEM,
//    B = the ckv columns of the same shared-memory tile read MN-major, N = 256).
//  * Roles: warp 0 issues TMA, warp 1 issues MMAs (one thread) and zeroes key rows
//    past the row's end, warps 2..5 run softmax, exchange and epilogue.
//  * Every wait is bounded; on timeout the kernel records MLA_ERR_DEVICE_TIMEOUT in
//    the plan's status word and every role unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mla_internal.h"
#include "mla_launch.h"
#include "sm100_ptx.cuh"

namespace mla {

using namespace ptx;

namespace attn {

constexpr int kStages = 3;
constexpr int kThreads = 192;

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t kQCkv = 0;              // 4 chunks x [128 rows x 128 B], 128B swizzle
constexpr uint32_t kQKpe = 65536;          // [128 rows x 64 B], 64B swizzle
constexpr uint32_t kKV = 73728;            // kStages stages
constexpr uint32_t kStageBytes = 36864;    //   4 chunks x [64 keys x 128 B] + [64 x 64 B]
constexpr uint32_t kStageKpe = 32768;
constexpr uint32_t kX = kKV + kStages * kStageBytes;  // peer partial scores
constexpr uint32_t kXRowBytes = 272;                  // 64 fp32 + 16 B pad (no bank conflicts)
constexpr uint32_t kXBytes = 128 * kXRowBytes;
constexpr uint32_t kBar = kX + kXBytes;
constexpr uint32_t kMisc = kBar + 256;
constexpr uint32_t kSmemUsed = kMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// Barrier indices (8 bytes each from kBar).
constexpr int bQFull = 0;
constexpr int bKVFull = 1;                 // + stage
constexpr int bKVEmpty = bKVFull + kStages;
constexpr int bSFull = bKVEmpty + kStages;  // + buffer (2)
constexpr int bSEmpty = bSFull + 2;
constexpr int bPFull = bSEmpty + 2;
constexpr int bPVDone = bPFull + 2;
constexpr int bXFull = bPVDone + 1;         // + quarter (4)
constexpr int bXEmpty = bXFull + 4;
constexpr int bFin = bXEmpty + 4;
constexpr int kNumBars = bFin + 1;
static_assert(kNumBars * 8 <= 256, "barrier area");

// TMEM columns.
constexpr uint32_t kColO = 0;     // 256 fp32 columns: this CTA's half of O
constexpr uint32_t kColS = 256;   // 2 x 64 fp32 columns
constexpr uint32_t kColP = 384;   // 2 x 32 columns of packed bf16 pairs
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kQBytes = 65536 + 8192;
constexpr float kNegInf = -__builtin_huge_valf();

// Error sites (bits 8.. of the status word) for diagnosis.
enum : int32_t {
  kSiteProducer = 1,
  kSiteMmaQ = 2,
  kSiteMmaKV = 3,
  kSiteMmaS = 4,
  kSiteMmaP = 5,
  kSiteSoftS = 6,
  kSiteSoftX = 7,
  kSiteSoftPV = 8,
  kSiteEpilogue = 9,
  kSiteTeardown = 10,
};

__device__ __forceinline__ void record_error(int32_t* status, int32_t site) {
  atomicCAS(status, 0, MLA_ERR_DEVICE_TIMEOUT | (site << 8));
}

}  // namespace attn

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(attn::kThreads, 1)
    mla_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qpe,
                    const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_kpe,
                    const AttnParams p) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const WorkItem w = p.work[blockIdx.x >> 1];
  const int ntiles = w.key_end > w.key_begin ? (w.key_end - w.key_begin + kTileN - 1) / kTileN : 0;

  auto bar = [&](int i) -> uint32_t { return sb + kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMisc + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMisc);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(bQFull), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(bKVFull + s), 1);
      mbar_init(bar(bKVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(bSFull + b), 1);
      mbar_init(bar(bSEmpty + b), 4);
      mbar_init(bar(bPFull + b), 4);
    }
    mbar_init(bar(bPVDone), 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(bar(bXFull + q), 32);
      mbar_init(bar(bXEmpty + q), 32);
    }
    mbar_init(bar(bFin), 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_qpe);
    tma_prefetch_desc(&tm_kv);
    tma_prefetch_desc(&tm_kpe);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The peer's barriers must be initialised before any remote arrive or DSMEM store.
  cluster_arrive();
  cluster_wait();
  const uint32_t tmem = *tmem_slot;
  const uint64_t TO = p.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (ntiles > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(bQFull), kQBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_2d(sb + kQCkv + c * 16384, &tm_q, bar(bQFull), 256 * rank + 64 * c, w.q_row0);
        tma_load_2d(sb + kQKpe, &tm_qpe, bar(bQFull), 32 * rank, w.q_row0);
      }
      const int P = p.page_size, BR = p.box_rows, nbox = kTileN / BR;
      const int last_page = (w.kv_len + P - 1) / P - 1;
      // physical start row of box `lane` of tile j (lanes >= nbox unused)
      auto box_row = [&](int j) -> int {
        int rs = 0;
        if (lane < nbox) {
          const int key0 = w.key_begin + kTileN * j + lane * BR;
          const int lp = min(key0 / P, last_page);
          rs = __ldg(p.kv_indices + w.page_base + lp) * P + (key0 % P);
        }
        return rs;
      };
      int last_issued[kStages] = {-1, -1, -1};
      int rs_next = box_row(0);
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        const int rs = rs_next;
        if (j + 1 < ntiles) rs_next = box_row(j + 1);
        if (j >= kStages) {
          bool ok = mbar_wait(bar(bKVEmpty + st), ((j / kStages) - 1) & 1, TO, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            if (lane == 0) { record_error(p.status, kSiteProducer); *abort_flag = 1; }
            break;
          }
        }
        if ((p.debug_flags & MLA_DEBUG_DROP_FIRST_KV_LOAD) && j == 0) continue;
        const uint32_t dst = sb + kKV + st * kStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(bar(bKVFull + st), kStageBytes);
        for (int b = 0; b < nbox; ++b) {
          const int row = __shfl_sync(0xffffffffu, rs, b);
          if (lane == 0) {
            for (int c = 0; c < 4; ++c)
              tma_load_2d(dst + c * 8192 + b * BR * 128, &tm_kv, bar(bKVFull + st), 256 * rank + 64 * c, row);
            tma_load_2d(dst + kStageKpe + b * BR * 64, &tm_kpe, bar(bKVFull + st), kCkv + 32 * rank, row);
          }
        }
        last_issued[st] = j;
      }
      // Do not leave while our own copies may still be landing.
      if (lane == 0) {
        if (!mbar_wait(bar(bQFull), 0, TO, abort_flag)) record_error(p.status, kSiteTeardown);
        for (int s = 0; s < kStages; ++s)
          if (last_issued[s] >= 0 &&
              !mbar_wait(bar(bKVFull + s), (last_issued[s] / kStages) & 1, TO, abort_flag))
            record_error(p.status, kSiteTeardown);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (ntiles > 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, 64, false, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 256, false, true);
      bool ok = mbar_wait(bar(bQFull), 0, TO, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) { record_error(p.status, kSiteMmaQ); *abort_flag = 1; }
      tc_fence_after();
      auto issue_pv = [&](int j) {
        const uint32_t kv = sb + kKV + (j % kStages) * kStageBytes;
        const uint32_t pcol = tmem + kColP + 32 * (j & 1);
        for (int s = 0; s < 4; ++s) {
          const uint64_t bd = smem_desc(kv + s * 2048, 8192, 1024, 2);
          mma_ts(tmem + kColO, pcol + 8 * s, bd, id_pv, (j > 0 || s > 0) ? 1u : 0u);
        }
        mma_commit(bar(bKVEmpty + (j % kStages)));
        mma_commit(bar(bPVDone));
      };
      int j = 0;
      for (; ok && j < ntiles; ++j) {
        const int st = j % kStages, b2 = j & 1;
        ok = mbar_wait(bar(bKVFull + st), (j / kStages) & 1, TO, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) { if (lane == 0) { record_error(p.status, kSiteMmaKV); *abort_flag = 1; } break; }
        if (j >= 2) {
          ok = mbar_wait(bar(bSEmpty + b2), ((j >> 1) - 1) & 1, TO, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) { if (lane == 0) { record_error(p.status, kSiteMmaS); *abort_flag = 1; } break; }
        }
        tc_fence_after();
        const uint32_t kv = sb + kKV + st * kStageBytes;
        // Keys at or past the row's end hold whatever the page's unused slots contain;
        // zero their ckv rows so that P = 0 never meets a non-finite V.
        const int key0 = w.key_begin + kTileN * j;
        if (key0 + kTileN > w.kv_len) {
          const int first_bad = max(0, w.kv_len - key0);
          const int n16 = (kTileN - first_bad) * 8;  // 16-byte pieces per chunk
          const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int i = lane; i < 4 * n16; i += 32) {
            const int c = i / n16, k = i % n16;
            float4* dst = reinterpret_cast<float4*>(smem + kKV + st * kStageBytes + c * 8192 +
                                                    first_bad * 128 + k * 16);
            *dst = z;
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t scol = tmem + kColS + 64 * b2;
          for (int c = 0; c < 4; ++c)
            for (int s = 0; s < 4; ++s) {
              const uint64_t ad = smem_desc(sb + kQCkv + c * 16384 + s * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(kv + c * 8192 + s * 32, 16, 1024, 2);
              mma_ss(scol, ad, bd, id_qk, (c | s) ? 1u : 0u);
            }
          for (int s = 0; s < 2; ++s) {
            const uint64_t ad = smem_desc(sb + kQKpe + s * 32, 16, 512, 4);
            const uint64_t bd = smem_desc(kv + kStageKpe + s * 32, 16, 512, 4);
            mma_ss(scol, ad, bd, id_qk, 1u);
          }
          mma_commit(bar(bSFull + b2));
        }
        __syncwarp();
        if (j >= 1) {
          ok = mbar_wait(bar(bPFull + ((j - 1) & 1)), ((j - 1) >> 1) & 1, TO, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) { if (lane == 0) { record_error(p.status, kSiteMmaP); *abort_flag = 1; } break; }
          tc_fence_after();
          if (lane == 0) issue_pv(j - 1);
          __syncwarp();
        }
      }
      if (ok) {
        const int jl = ntiles - 1;
        ok = mbar_wait(bar(bPFull + (jl & 1)), (jl >> 1) & 1, TO, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          if (lane == 0) { record_error(p.status, kSiteMmaP); *abort_flag = 1; }
        } else {
          tc_fence_after();
          if (lane == 0) issue_pv(jl);
          __syncwarp();
        }
      }
      // Every MMA this thread issued must retire before TMEM is released.
      if (lane == 0) {
        mma_commit(bar(bFin));
        if (!mbar_wait(bar(bFin), 0, TO, abort_flag)) record_error(p.status, kSiteTeardown);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    const int r = 32 * q + lane;          // tile row owned by this thread
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    int vis = w.diag_base + r / p.num_heads + 1;
    vis = max(0, min(vis, w.kv_len));
    if (r >= w.n_rows) vis = 0;
    const int lim = min(vis, w.key_end);  // keys < lim are visible in this chunk
    const uint32_t xrow = sb + kX + r * kXRowBytes;
    const uint32_t xrow_peer = map_to_cta(xrow, peer);
    const float* xrow_ptr = reinterpret_cast<const float*>(smem + kX + r * kXRowBytes);
    float m_run = kNegInf, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int b2 = j & 1;
      ok = mbar_wait(bar(bSFull + b2), (j >> 1) & 1, TO, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { if (lane == 0) { record_error(p.status, kSiteSoftS); *abort_flag = 1; } break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(trow + kColS + 64 * b2, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(trow + kColS + 64 * b2 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bSEmpty + b2));

      // --- exchange partial scores with the peer CTA
      if (j >= 1) {
        ok = mbar_wait<true>(bar(bXEmpty + q), (j - 1) & 1, TO, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) { if (lane == 0) { record_error(p.status, kSiteSoftX); *abort_flag = 1; } break; }
      }
#pragma unroll
      for (int c = 0; c < 16; ++c)
        st_cluster_v4(xrow_peer + 16 * c, __uint_as_float(sr[4 * c]), __uint_as_float(sr[4 * c + 1]),
                      __uint_as_float(sr[4 * c + 2]), __uint_as_float(sr[4 * c + 3]));
      mbar_arrive_remote(bar(bXFull + q), peer);
      ok = mbar_wait<true>(bar(bXFull + q), j & 1, TO, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { if (lane == 0) { record_error(p.status, kSiteSoftX); *abort_flag = 1; } break; }
      float t[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(xrow_ptr + 4 * c);
        t[4 * c + 0] = __uint_as_float(sr[4 * c + 0]) + x.x;
        t[4 * c + 1] = __uint_as_float(sr[4 * c + 1]) + x.y;
        t[4 * c + 2] = __uint_as_float(sr[4 * c + 2]) + x.z;
        t[4 * c + 3] = __uint_as_float(sr[4 * c + 3]) + x.w;
      }
      mbar_arrive_remote(bar(bXEmpty + q), peer);

      // --- mask, running max (log2 domain), lazy rescale
      const int nvalid = lim - (w.key_begin + kTileN * j);
      float mt = kNegInf;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        t[c] = (c < nvalid) ? t[c] * p.scale_log2 : kNegInf;
        mt = fmaxf(mt, t[c]);
      }
      // Keep the old reference max unless the new one exceeds it by more than 8 (a
      // factor of 256 in the weights); then rescale the running sum and output row.
      const bool bump = mt > m_run + 8.f;
      const float m_old = m_run;
      float alpha = 1.f;
      if (bump) {
        alpha = ex2_approx(m_old - mt);  // 0 when m_old is -inf
        l_run *= alpha;
        m_run = mt;
      }
      const bool resc = bump && j > 0 && m_old != kNegInf;
      if (__any_sync(0xffffffffu, resc)) {
        ok = mbar_wait(bar(bPVDone), (j - 1) & 1, TO, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) { if (lane == 0) { record_error(p.status, kSiteSoftPV); *abort_flag = 1; } break; }
        tc_fence_after();
        const float a = resc ? alpha : 1.f;
        for (int cc = 0; cc < 256; cc += 32) {
          uint32_t o[32];
          tmem_ld32(trow + kColO + cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
          tmem_st16(trow + kColO + cc, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
          tmem_st16(trow + kColO + cc + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
        }
        tmem_wait_st();
      }

      // --- P = exp2(t - m) into TMEM as bf16; the running sum takes the fp32 values
      const float msub = (m_run == kNegInf) ? 0.f : m_run;
      uint32_t pk[32];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = ex2_approx(t[2 * c] - msub);
        const float p1 = ex2_approx(t[2 * c + 1] - msub);
        pk[c] = pack_bf16x2(p0, p1);
        lsum += p0 + p1;
      }
      l_run += lsum;
      tmem_st16(trow + kColP + 32 * b2, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(trow + kColP + 32 * b2 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bPFull + b2));
    }

    // --- epilogue
    if (ok) {
      const bool has = l_run > 0.f;
      const float inv_l = has ? 1.f / l_run : 0.f;
      const float lse_nat = has ? (m_run + __log2f(l_run)) * 0.69314718055994531f : kNegInf;
      const bool row_ok = r < w.n_rows;
      if (ntiles > 0) {
        ok = mbar_wait(bar(bPVDone), (ntiles - 1) & 1, TO, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) { record_error(p.status, kSiteEpilogue); *abort_flag = 1; }
        tc_fence_after();
      }
      if (ok) {
        if (w.partial < 0) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(w.q_row0 + r) * kCkv + 256 * rank;
          for (int cc = 0; cc < 256; cc += 32) {
            uint32_t o[32];
            if (ntiles > 0) {
              tmem_ld32(trow + kColO + cc, o);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
            if (row_ok) {
              uint4 v[4];
              uint32_t* vp = reinterpret_cast<uint32_t*>(v);
#pragma unroll
              for (int i = 0; i < 16; ++i)
                vp[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
              uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
              for (int i = 0; i < 4; ++i) d4[i] = v[i];
            }
          }
          if (rank == 0 && p.lse != nullptr && row_ok) p.lse[w.q_row0 + r] = lse_nat;
        } else {
          float* dst = p.ws_o + (static_cast<size_t>(w.partial) * kTileM + r) * kCkv + 256 * rank;
          for (int cc = 0; cc < 256; cc += 32) {
            uint32_t o[32];
            if (ntiles > 0) {
              tmem_ld32(trow + kColO + cc, o);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
            if (row_ok) {
              float4* d4 = reinterpret_cast<float4*>(dst + cc);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                d4[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                    __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
            }
          }
          if (rank == 0 && row_ok) p.ws_lse[static_cast<size_t>(w.partial) * kTileM + r] = lse_nat;
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // The peer may still store into our shared memory or arrive on our barriers.
  cluster_arrive();
  cluster_wait();
}

// Combine the fp32 partials of split query tiles by their log-sum-exp:
// M = max_i lse_i, out = sum_i e^{lse_i - M} o_i / sum_i e^{lse_i - M},
// lse = M + ln sum_i e^{lse_i - M} (FlashInferMLAManager.run: merging key segments).
__global__ void __launch_bounds__(256) mla_merge_kernel(const MergeParams p) {
  const MergeItem m = p.merge[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < m.n_rows; r += 8) {
    float M = -__int_as_float(0x7f800000);
    for (int i = 0; i < m.n_partials; ++i)
      M = fmaxf(M, p.ws_lse[static_cast<size_t>(m.first_partial + i) * kTileM + r]);
    float4 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    float z = 0.f;
    if (M != -__int_as_float(0x7f800000)) {
      for (int i = 0; i < m.n_partials; ++i) {
        const size_t slot = static_cast<size_t>(m.first_partial + i) * kTileM + r;
        const float wgt = __expf(p.ws_lse[slot] - M);
        z += wgt;
        const float4* src = reinterpret_cast<const float4*>(p.ws_o + slot * kCkv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 v = src[lane + 32 * k];
          acc[k].x += wgt * v.x;
          acc[k].y += wgt * v.y;
          acc[k].z += wgt * v.z;
          acc[k].w += wgt * v.w;
        }
      }
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(m.q_row0 + r) * kCkv;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint2 v;
      v.x = ptx::pack_bf16x2(acc[k].x * inv, acc[k].y * inv);
      v.y = ptx::pack_bf16x2(acc[k].z * inv, acc[k].w * inv);
      *reinterpret_cast<uint2*>(dst + 4 * (lane + 32 * k)) = v;
    }
    if (p.lse != nullptr && lane == 0)
      p.lse[m.q_row0 + r] = z > 0.f ? M + __logf(z) : -__int_as_float(0x7f800000);
  }
}

// ---------------------------------------------------------------------- launchers
cudaError_t launch_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_qpe, const CUtensorMap& tm_kv,
                             const CUtensorMap& tm_kpe, const AttnParams& p, int num_work, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(mla_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(attn::kSmemAlloc));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  mla_attn_kernel<<<2 * num_work, attn::kThreads, attn::kSmemAlloc, stream>>>(tm_q, tm_qpe, tm_kv, tm_kpe, p);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeParams& p, int num_merge, cudaStream_t stream) {
  mla_merge_kernel<<<num_merge, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla

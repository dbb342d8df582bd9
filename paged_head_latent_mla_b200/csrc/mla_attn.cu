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
//    M=128, N=64, K=288) into TMEM; the exchange warps push it to the peer over DSMEM
//    (st.async completing on the peer's mbarrier); the softmax warps add the peer's
//    partial (fp32 addition commutes, so both CTAs hold bit-identical S), apply mask
//    and online softmax (log2 domain, lazy rescale), and store P as bf16 into TMEM.
//    Then O_half += P . V_half (tcgen05, A = P from TMEM, B = the ckv columns of the
//    same shared-memory tile read MN-major, N = 256).
//  * Roles (11 warps): warps 0..3 softmax and epilogue, 4..7 exchange (one per TMEM
//    lane quarter in each group), 8 TMA producer, 9 QK issuer (one thread; also TMEM
//    allocation and zeroing of key rows past the row's end), 10 PV issuer.
//  * An empty work item (an unused launch slot of a graph plan) returns at once; the
//    producer waits for a preceding cache append (programmatic dependent launch)
//    before its first key load; the kpe width is a run-time parameter (64 or 0).
//  * Every wait is bounded; on timeout the kernel records MLA_ERR_DEVICE_TIMEOUT in
//    the plan's status word and every role unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "mla_internal.h"
#include "mla_launch.h"
#include "sm100_ptx.cuh"

namespace mla {

using namespace ptx;

namespace attn {

#ifndef MLA_KV_STAGES
#define MLA_KV_STAGES 4
#endif
#ifndef MLA_X_SLOTS
#define MLA_X_SLOTS 1
#endif
constexpr int kStages = MLA_KV_STAGES;  // KV ring depth
constexpr int kXSlots = MLA_X_SLOTS;    // exchange buffers (1 or 2)
constexpr int kThreads = 352;  // 11 warps, roles below

// Warp roles.  Warps 0..3 and 4..7 each cover the four TMEM lane quarters (a warp may
// only touch lanes 32 * (warp % 4) .. + 31).
constexpr int kWarpSoftmax0 = 0;   // 0..3: softmax, lazy rescale, P, epilogue
constexpr int kWarpExchange0 = 4;  // 4..7: push our partial scores to the peer CTA
constexpr int kWarpProducer = 8;   // TMA page gather
constexpr int kWarpMma = 9;        // QK^T issue, TMEM allocation, zeroing past-the-end keys
constexpr int kWarpPv = 10;        // P.V issue
static_assert(kWarpSoftmax0 == 0 && kWarpExchange0 == 4, "quarter = warp % 4 in both groups");

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t kQCkv = 0;              // 3 chunks x [128 rows x 128 B], 128B swizzle
constexpr int kQSmemChunks = 3;            // the 4th ckv chunk and the kpe part live in TMEM
constexpr uint32_t kKV = 49152;            // kStages stages
constexpr uint32_t kStageBytes = 36864;    //   4 chunks x [64 keys x 128 B] + [64 x 64 B]
constexpr uint32_t kStageKpe = 32768;
constexpr uint32_t kX = kKV + kStages * kStageBytes;  // the peer's partial scores
constexpr uint32_t kXSlotBytes = 128 * 64 * 4;       // 4 quarters x 16 chunks x 32 lanes x 16 B
constexpr uint32_t kBar = kX + kXSlots * kXSlotBytes;
constexpr uint32_t kMisc = kBar + 512;
constexpr uint32_t kSmemUsed = kMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// Barrier indices (8 bytes each from kBar).
constexpr int bQFull = 0;                   // TMA part of Q landed
constexpr int bQTmem = 1;                   // TMEM part of Q stored (4 softmax warps)
constexpr int bKVFull = 2;                  // + stage
constexpr int bKVEmpty = bKVFull + kStages;
constexpr int bSFull = bKVEmpty + kStages;  // + buffer (2)
constexpr int bSEmpty = bSFull + 2;
constexpr int bPFull = bSEmpty + 2;
constexpr int bPVDone = bPFull + 2;         // + P buffer (2): PV(j) done, j % 2
constexpr int bXFull = bPVDone + 2;         // + slot * 4 + quarter
constexpr int bXEmpty = bXFull + 4 * kXSlots;
constexpr int bFin = bXEmpty + 4 * kXSlots;  // + issuer (2)
constexpr int kNumBars = bFin + 2;
static_assert(kNumBars * 8 <= 512, "barrier area");

// TMEM columns.
constexpr uint32_t kColO = 0;     // 256 fp32 columns: this CTA's half of O
constexpr uint32_t kColS = 256;   // 2 x 64 fp32 columns
constexpr uint32_t kColP = 384;   // 2 x 32 columns of packed bf16 pairs
constexpr uint32_t kColQ = 448;   // 32 columns: ckv chunk 3 of Q (64 bf16), packed pairs
constexpr uint32_t kColQpe = 480; // 16 columns: this CTA's 32 kpe columns of Q
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kQBytes = kQSmemChunks * 16384;
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
  kSiteExchange = 11,
};

// The first error wins the device word; its recorder also copies it to the host-mapped
// mirror (a plain store: only the winner writes it), which the host reads once the
// launch has finished without going through a copy engine.
__device__ __forceinline__ void record_error(int32_t* status, int32_t* mirror, int32_t site) {
  const int32_t v = MLA_ERR_DEVICE_TIMEOUT | (site << 8);
  if (atomicCAS(status, 0, v) == 0 && mirror != nullptr) {
    *reinterpret_cast<volatile int32_t*>(mirror) = v;
    __threadfence_system();
  }
}

}  // namespace attn

// Pipeline per 64-key tile j (phases of every two-buffer barrier are j >> 1):
//   producer : KV(j) -> stage j % 3                        (after PV(j - 3) freed it)
//   QK warp  : QK(j) -> S[j % 2], as soon as KV(j) landed and S(j - 2) was read
//   exchange : S(j) partial -> peer over DSMEM (st.async, completes the peer's x_full)
//   softmax  : S(j) = ours + peer's; mask, online softmax, P(j) -> P[j % 2]
//   PV warp  : PV(j): O += P[j % 2] . V(stage j % 3), as soon as P(j) is written
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(attn::kThreads, 1)
    mla_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                    const __grid_constant__ CUtensorMap tm_kpe, const AttnParams p) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  // A merge grid launched after this one may be scheduled as SMs free up; it waits for
  // this grid to finish before reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const WorkItem w = p.work[blockIdx.x >> 1];
  // An empty launch slot (graph plans launch a fixed grid): both CTAs of the pair read
  // the same item and leave before touching any shared state.
  if (w.n_rows <= 0) return;
  const int ntiles = w.key_end > w.key_begin ? (w.key_end - w.key_begin + kTileN - 1) / kTileN : 0;

  auto bar = [&](int i) -> uint32_t { return sb + kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMisc + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMisc);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(bQFull), 1);
    mbar_init(bar(bQTmem), 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(bKVFull + s), 1);
      mbar_init(bar(bKVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(bSFull + b), 1);
      mbar_init(bar(bSEmpty + b), 8);  // softmax and exchange warps both read S
      mbar_init(bar(bPFull + b), 4);
      mbar_init(bar(bPVDone + b), 1);
    }
    for (int i = 0; i < 4 * kXSlots; ++i) {
      mbar_init(bar(bXFull + i), 1);   // our expect_tx + the peer's 8 KB of st.async
      mbar_init(bar(bXEmpty + i), 1);  // the peer drained the 8 KB we pushed
    }
    mbar_init(bar(bFin), 1);
    mbar_init(bar(bFin + 1), 1);
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kv);
    if (p.rope_dim > 0) tma_prefetch_desc(&tm_kpe);
  }
  if (warp == kWarpMma) {
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

  // Bounded wait shared by every role: all lanes poll, the warp agrees, lane 0 records.
  auto wait_warp = [&](uint32_t b, uint32_t parity, int32_t site, bool cluster_scope) -> bool {
    bool good = cluster_scope ? mbar_wait<true>(b, parity, TO, abort_flag) : mbar_wait(b, parity, TO, abort_flag);
    good = __all_sync(0xffffffffu, good);
    if (!good && lane == 0) {
      record_error(p.status, p.status_mirror, site);
      *abort_flag = 1;
    }
    return good;
  };

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ TMA producer
    if (ntiles > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(bQFull), kQBytes);
        for (int c = 0; c < kQSmemChunks; ++c)
          tma_load_2d(sb + kQCkv + c * 16384, &tm_q, bar(bQFull), 256 * rank + 64 * c, w.q_row0);
      }
      const int P = p.page_size, BR = p.box_rows, nbox = kTileN / BR;
      const int last_page = (w.kv_len + P - 1) / P - 1;
      // Page ids are read 32 at a time (lane i holds logical page win + i) so that no
      // dependent global load sits between a free stage and its TMA issue.
      int win = -64, win_id = 0;
      auto page_of = [&](int lp) -> int {
        lp = min(lp, last_page);
        if (lp - win < 0 || lp - win >= 32) {  // warp-uniform
          win = lp;
          win_id = (win + lane <= last_page) ? __ldg(p.kv_indices + w.page_base + win + lane) : 0;
        }
        return __shfl_sync(0xffffffffu, win_id, lp - win);
      };
      int last_issued[kStages];
#pragma unroll
      for (int s2 = 0; s2 < kStages; ++s2) last_issued[s2] = -1;
      // Launched as a programmatic dependent of a cache append, the key loads must see
      // its writes: wait for that grid (a no-op for an ordinary launch).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !wait_warp(bar(bKVEmpty + st), ((j / kStages) - 1) & 1, kSiteProducer, false)) break;
        if ((p.debug_flags & MLA_DEBUG_DROP_FIRST_KV_LOAD) && j == 0) continue;
        const uint32_t dst = sb + kKV + st * kStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(bar(bKVFull + st), p.rope_dim > 0 ? kStageBytes : kStageKpe);
        for (int b = 0; b < nbox; ++b) {
          const int key0 = w.key_begin + kTileN * j + b * BR;
          const int row = page_of(key0 / P) * P + (key0 % P);
          if (lane == 0) {
            for (int c = 0; c < 4; ++c)
              tma_load_2d(dst + c * 8192 + b * BR * 128, &tm_kv, bar(bKVFull + st), 256 * rank + 64 * c, row);
            if (p.rope_dim > 0)
              tma_load_2d(dst + kStageKpe + b * BR * 64, &tm_kpe, bar(bKVFull + st), kCkv + 32 * rank, row);
          }
        }
        last_issued[st] = j;
      }
      // Do not leave while our own copies may still be landing.
      if (lane == 0) {
        if (!mbar_wait(bar(bQFull), 0, TO, abort_flag)) record_error(p.status, p.status_mirror, kSiteTeardown);
        for (int s = 0; s < kStages; ++s)
          if (last_issued[s] >= 0 &&
              !mbar_wait(bar(bKVFull + s), (last_issued[s] / kStages) & 1, TO, abort_flag))
            record_error(p.status, p.status_mirror, kSiteTeardown);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (ntiles > 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, 64, false, false);
      // QK(j): wait for KV(j) and for both readers of S(j - 2) to be done with S[j % 2].
      auto issue_qk = [&](int j) -> bool {
        const int st = j % kStages, b2 = j & 1;
        if (!wait_warp(bar(bKVFull + st), (j / kStages) & 1, kSiteMmaKV, false)) return false;
        if (j >= 2 && !wait_warp(bar(bSEmpty + b2), ((j >> 1) - 1) & 1, kSiteMmaS, false)) return false;
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
            *reinterpret_cast<float4*>(smem + kKV + st * kStageBytes + c * 8192 + first_bad * 128 + k * 16) = z;
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t scol = tmem + kColS + 64 * b2;
          for (int c = 0; c < kQSmemChunks; ++c)
            for (int s = 0; s < 4; ++s) {
              const uint64_t ad = smem_desc(sb + kQCkv + c * 16384 + s * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(kv + c * 8192 + s * 32, 16, 1024, 2);
              mma_ss(scol, ad, bd, id_qk, (c | s) ? 1u : 0u);
            }
          for (int s = 0; s < 4; ++s) {  // ckv chunk 3: A from TMEM
            const uint64_t bd = smem_desc(kv + 3 * 8192 + s * 32, 16, 1024, 2);
            mma_ts(scol, tmem + kColQ + 8 * s, bd, id_qk, 1u);
          }
          if (p.rope_dim > 0)
            for (int s = 0; s < 2; ++s) {  // kpe: A from TMEM
              const uint64_t bd = smem_desc(kv + kStageKpe + s * 32, 16, 512, 4);
              mma_ts(scol, tmem + kColQpe + 8 * s, bd, id_qk, 1u);
            }
          mma_commit(bar(bSFull + b2));
        }
        __syncwarp();
        return true;
      };
      bool ok = wait_warp(bar(bQFull), 0, kSiteMmaQ, false) && wait_warp(bar(bQTmem), 0, kSiteMmaQ, false);
      tc_fence_after();
      for (int j = 0; ok && j < ntiles; ++j) ok = issue_qk(j);
      // Every MMA this thread issued must retire before TMEM is released.
      if (lane == 0) {
        mma_commit(bar(bFin));
        if (!mbar_wait(bar(bFin), 0, TO, abort_flag)) record_error(p.status, p.status_mirror, kSiteTeardown);
      }
      __syncwarp();
    }
  } else if (warp == kWarpPv) {
    // ------------------------------------------------------------------ P.V issuer
    if (ntiles > 0) {
      const uint32_t id_pv = idesc_bf16_f32(128, 256, false, true);
      for (int j = 0; j < ntiles; ++j) {
        if (!wait_warp(bar(bPFull + (j & 1)), (j >> 1) & 1, kSiteMmaP, false)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kv = sb + kKV + (j % kStages) * kStageBytes;
          const uint32_t pcol = tmem + kColP + 32 * (j & 1);
          for (int s = 0; s < 4; ++s) {
            const uint64_t bd = smem_desc(kv + s * 2048, 8192, 1024, 2);
            mma_ts(tmem + kColO, pcol + 8 * s, bd, id_pv, (j > 0 || s > 0) ? 1u : 0u);
          }
          mma_commit(bar(bKVEmpty + (j % kStages)));
          mma_commit(bar(bPVDone + (j & 1)));
        }
        __syncwarp();
      }
      if (lane == 0) {
        mma_commit(bar(bFin + 1));
        if (!mbar_wait(bar(bFin + 1), 0, TO, abort_flag)) record_error(p.status, p.status_mirror, kSiteTeardown);
      }
      __syncwarp();
    }
  } else if (warp >= kWarpExchange0) {
    // ------------------------------------------------------------------ score exchange
    // Partial S(j) (our 288 of the 576 contraction columns) goes to the peer, laid out
    // chunk-major per lane quarter: 16-byte chunk c of row (32q + lane) sits at
    // q * 8 KB + (c * 32 + lane) * 16, so one warp store covers 512 contiguous bytes.
    const int q = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const uint32_t xq_peer = map_to_cta(sb + kX + q * 8192 + lane * 16, peer);
    const uint32_t xfull_peer = map_to_cta(bar(bXFull + q), peer);
    for (int j = 0; j < ntiles; ++j) {
      const int b2 = j & 1;
      if (!wait_warp(bar(bSFull + b2), (j >> 1) & 1, kSiteExchange, false)) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(trow + kColS + 64 * b2, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(trow + kColS + 64 * b2 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bSEmpty + b2));
      // the peer must have drained our slot (it held tile j - kXSlots)
      const int xs = j % kXSlots, xph = j / kXSlots;
      if (j >= kXSlots && !wait_warp(bar(bXEmpty + 4 * xs + q), (xph - 1) & 1, kSiteExchange, true)) break;
      const uint32_t dst = xq_peer + xs * kXSlotBytes;
      const uint32_t xbar = xfull_peer + 8u * (4 * xs);
#pragma unroll
      for (int c = 0; c < 16; ++c)
        st_async_v4(dst + c * 512, sr[4 * c], sr[4 * c + 1], sr[4 * c + 2], sr[4 * c + 3], xbar);
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
    const float* xq_ptr = reinterpret_cast<const float*>(smem + kX + q * 8192 + lane * 16);
    const float scale = p.scale_log2;  // > 0 (the planner rejects other scales)
    float m_run = kNegInf, l_run = 0.f;
    bool ok = true;

    // --- the TMEM part of Q: ckv columns [256r + 192, 256r + 256) and kpe columns
    // [32r, 32r + 32) of this row, as packed bf16 pairs (even element in the low half)
    if (ntiles > 0) {
      uint32_t qa[32], qb[16];
      if (r < w.n_rows) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q_nope) +
                                                          static_cast<size_t>(w.q_row0 + r) * kCkv + 256 * rank + 192);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = __ldg(src + i);
          qa[4 * i] = v.x; qa[4 * i + 1] = v.y; qa[4 * i + 2] = v.z; qa[4 * i + 3] = v.w;
        }
        if (p.rope_dim > 0) {
          const uint4* srp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q_pe) +
                                                            static_cast<size_t>(w.q_row0 + r) * kRope + 32 * rank);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(srp + i);
            qb[4 * i] = v.x; qb[4 * i + 1] = v.y; qb[4 * i + 2] = v.z; qb[4 * i + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) qb[i] = 0u;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) qa[i] = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i) qb[i] = 0u;
      }
      tmem_st32(trow + kColQ, qa);
      tmem_st16(trow + kColQpe, qb);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bQTmem));
    }

    for (int j = 0; ok && j < ntiles; ++j) {
      const int b2 = j & 1;
      if (!(ok = wait_warp(bar(bSFull + b2), (j >> 1) & 1, kSiteSoftS, false))) break;
      const int xsl = j % kXSlots, xph = j / kXSlots;
      const uint32_t xfull = bar(bXFull + 4 * xsl + q);
      if (lane == 0) mbar_arrive_expect_tx(xfull, 8192);
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(trow + kColS + 64 * b2, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(trow + kColS + 64 * b2 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bSEmpty + b2));
      if (!(ok = wait_warp(xfull, xph & 1, kSiteSoftX, true))) break;
      // --- raw S(j) = our partial + the peer's (fp32 addition commutes: the pair holds
      // bit-identical scores)
      const float* xs = xq_ptr + xsl * (kXSlotBytes / 4);
      float t[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(xs + c * 128);
        t[4 * c + 0] = __uint_as_float(sr[4 * c + 0]) + x.x;
        t[4 * c + 1] = __uint_as_float(sr[4 * c + 1]) + x.y;
        t[4 * c + 2] = __uint_as_float(sr[4 * c + 2]) + x.z;
        t[4 * c + 3] = __uint_as_float(sr[4 * c + 3]) + x.w;
      }

      // --- mask (partial tiles only), running max in the log2 domain, lazy rescale
      const int nvalid = lim - (w.key_begin + kTileN * j);
      if (__any_sync(0xffffffffu, nvalid < kTileN)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) t[c] = (c < nvalid) ? t[c] : kNegInf;
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(t[i], t[i + 8]);
#pragma unroll
      for (int c = 16; c < 64; c += 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], t[c + i]);
      const float mraw = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float mt = mraw * scale;  // scale > 0 keeps the order; -inf stays -inf
      // Hand the slot back to the peer.  mraw depends on every value loaded from the
      // slot, and the vote needs every lane's mraw, so all of this warp's loads have
      // delivered their data before lane 0's arrive issues; the peer's next push cannot
      // overtake them.  (An arrive issued before the loads completed did let it; a
      // release-ordered arrive also works but costs a cluster-scope fence per tile.)
      if (__any_sync(0xffffffffu, mraw != p.nan_guard) && lane == 0)
        mbar_arrive_remote_relaxed(bar(bXEmpty + 4 * xsl + q), peer);
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
        // every PV so far (the last is PV(j - 1)) must have landed in O
        if (!(ok = wait_warp(bar(bPVDone + ((j - 1) & 1)), ((j - 1) >> 1) & 1, kSiteSoftPV, false))) break;
        tc_fence_after();
        const float a = resc ? alpha : 1.f;
        for (int cc = 0; cc < 256; cc += 32) {
          uint32_t o[32];
          tmem_ld32(trow + kColO + cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
          tmem_st32(trow + kColO + cc, o);
        }
        tmem_wait_st();
      }

      // --- P = exp2(s * scale - m) as bf16 (fp32 running sum); P[j % 2] was last read
      // by PV(j - 2)
      const float msub = (m_run == kNegInf) ? 0.f : m_run;
      uint32_t pk[32];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = ex2_approx(fmaf(t[2 * c], scale, -msub));
        const float p1 = ex2_approx(fmaf(t[2 * c + 1], scale, -msub));
        pk[c] = pack_bf16x2(p0, p1);
        ls[c & 3] += p0 + p1;
      }
      l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (j >= 2 && !(ok = wait_warp(bar(bPVDone + b2), ((j >> 1) - 1) & 1, kSiteSoftPV, false))) break;
      tc_fence_after();
      tmem_st32(trow + kColP + 32 * b2, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bPFull + b2));
    }

    // --- epilogue.  Each warp stages its 32 rows of O / l (bf16) in the KV ring (idle now:
    // every load was consumed by a finished PV) and writes them back one 512-byte half
    // row per warp store, so every store covers whole cache lines.  16-byte piece c of staged row R sits at
    // position c ^ R, which keeps both the row-wise writes and the piece-wise reads free
    // of bank conflicts.
    if (ok) {
      const bool has = l_run > 0.f;
      const float inv_l = has ? 1.f / l_run : 0.f;
      const float lse_nat = has ? (m_run + __log2f(l_run)) * 0.69314718055994531f : kNegInf;
      if (ntiles > 0) {
        ok = wait_warp(bar(bPVDone + ((ntiles - 1) & 1)), ((ntiles - 1) >> 1) & 1, kSiteEpilogue, false);
        tc_fence_after();
      }
      if (ok) {
        const bool part = w.partial >= 0;  // bf16 partial in the workspace, or the output
        uint8_t* stage = smem + kKV + q * 16384;  // 32 rows x 512 B
        for (int cc = 0; cc < 256; cc += 32) {
          uint32_t o[32];
          if (ntiles > 0) {
            tmem_ld32(trow + kColO + cc, o);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          uint8_t* row = stage + (lane << 9);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = (cc >> 3) + i;  // pieces of 8 bf16
            *reinterpret_cast<uint4*>(row + ((c ^ lane) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l),
                pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l),
                pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l),
                pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l));
          }
        }
        __syncwarp();
        const int nrows = min(32, w.n_rows - 32 * q);  // rows of this warp inside the tile
        uint8_t* base = part ? static_cast<uint8_t*>(p.ws_o) + static_cast<size_t>(w.partial) * kCkv * 2
                             : static_cast<uint8_t*>(p.out) + static_cast<size_t>(w.q_row0) * kCkv * 2;
        for (int R = 0; R < nrows; ++R) {
          uint8_t* dst = base + (static_cast<size_t>(32 * q + R) * kCkv + 256 * rank) * 2;
          *reinterpret_cast<uint4*>(dst + (lane << 4)) =
              *reinterpret_cast<const uint4*>(stage + (R << 9) + ((lane ^ R) << 4));
        }
        if (rank == 0 && r < w.n_rows) {
          if (!part) {
            if (p.lse != nullptr) p.lse[w.q_row0 + r] = lse_nat;
          } else {
            p.ws_lse[static_cast<size_t>(w.partial) + r] = lse_nat;
          }
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // The peer may still store into our shared memory or arrive on our barriers.
  cluster_arrive();
  cluster_wait();
}

// Combine the partials of split (or cascaded) query tiles by their log-sum-exp:
// M = max_i lse_i, out = sum_i e^{lse_i - M} o_i / sum_i e^{lse_i - M},
// lse = M + ln sum_i e^{lse_i - M} (FlashInferMLAManager.run: merging key segments).
// One warp per row; lane l owns columns [16l, 16l + 16), so every load and store of a
// row is one contiguous 1 KB access.  Up to eight partials are in flight at a time, and
// a tile with more than 32 partials is merged 32 at a time against a running maximum.
__global__ void __launch_bounds__(256) mla_merge_kernel(const MergeParams p) {
  // The merge list and the reference list are plan data, written before the attention
  // grid started: read them while that grid drains.
  const MergeItem m = p.merge[blockIdx.x >> 4];  // 16 blocks per split query tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = ((blockIdx.x & 15) << 3) + warp;  // 8 rows (one per warp) per block
  if (r >= m.n_rows) return;
  const int n = m.n_refs;
  const int32_t* refs = p.refs + m.first_ref;  // workspace row of each partial's row 0
  int ref_l = lane < n ? refs[lane] : 0;       // lane u holds partial u's reference (u < 32)
  // Launched as a programmatic dependent of the attention grid: wait until that grid has
  // finished and its partials are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float neg_inf = -__int_as_float(0x7f800000);
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  float M = neg_inf, z = 0.f;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int cnt = min(32, n - i0);
    if (i0 > 0) ref_l = lane < cnt ? refs[i0 + lane] : 0;
    const float l_l = lane < cnt ? p.ws_lse[static_cast<size_t>(ref_l) + r] : neg_inf;
    // every partial of this group in flight before any is used (8 at a time)
    for (int k = 0; k < cnt; k += 8) {
      uint4 v[8][2];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int ref_u = __shfl_sync(0xffffffffu, ref_l, (k + u) & 31);
        if (k + u < cnt) {
          const uint4* src = reinterpret_cast<const uint4*>(
              static_cast<const uint8_t*>(p.ws_o) + ((static_cast<size_t>(ref_u) + r) * kCkv + 16 * lane) * 2);
          v[u][0] = src[0];
          v[u][1] = src[1];
        } else {
          v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (k == 0) {
        // the group's running max; earlier groups' sums are rescaled to it
        float Mg = l_l;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) Mg = fmaxf(Mg, __shfl_xor_sync(0xffffffffu, Mg, off));
        const float Mn = fmaxf(M, Mg);
        if (Mn != neg_inf && M != neg_inf && Mn != M) {
          const float s = __expf(M - Mn);
          z *= s;
#pragma unroll
          for (int q = 0; q < 16; ++q) acc[q] *= s;
        }
        M = Mn;
      }
      const float wl = (lane < cnt && M != neg_inf) ? __expf(l_l - M) : 0.f;
      if (k == 0) {
        float zg = wl;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) zg += __shfl_xor_sync(0xffffffffu, zg, off);
        z += zg;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wk = __shfl_sync(0xffffffffu, wl, (k + u) & 31);
        const uint32_t* wv = reinterpret_cast<const uint32_t*>(v[u]);
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) {
          acc[2 * k2] += wk * __uint_as_float(wv[k2] << 16);
          acc[2 * k2 + 1] += wk * __uint_as_float(wv[k2] & 0xffff0000u);
        }
      }
    }
  }
  const float inv = z > 0.f ? 1.f / z : 0.f;
  uint4 o[2];
  uint32_t* ov = reinterpret_cast<uint32_t*>(o);
#pragma unroll
  for (int k2 = 0; k2 < 8; ++k2) ov[k2] = ptx::pack_bf16x2(acc[2 * k2] * inv, acc[2 * k2 + 1] * inv);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(m.q_row0 + r) * kCkv +
                                        16 * lane);
  dst[0] = o[0];
  dst[1] = o[1];
  if (p.lse != nullptr && lane == 0) p.lse[m.q_row0 + r] = z > 0.f ? M + __logf(z) : neg_inf;
}

// ---------------------------------------------------------------------- launchers
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix (row pitch = cols).
bool encode_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream) {
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
  AttnParams p = a.p;
  p.q_nope = a.q_nope;
  p.q_pe = a.q_pe;
  p.nan_guard = __builtin_nanf("");
  p.box_rows = p.page_size < kTileN ? p.page_size : kTileN;
  const uint32_t br = static_cast<uint32_t>(p.box_rows);
  // the cache row is [ckv 512 | kpe rope_dim]; without kpe the kpe map is never used
  const uint64_t width = static_cast<uint64_t>(kCkv + p.rope_dim);
  CUtensorMap tm_q, tm_kv, tm_kpe;
  if (!encode_2d(&tm_q, a.q_nope, a.rows, kCkv, 64, kTileM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tm_kv, a.cache, a.cache_rows, width, 64, br, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (p.rope_dim > 0) {
    if (!encode_2d(&tm_kpe, a.cache, a.cache_rows, width, 32, br, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  } else {
    tm_kpe = tm_kv;
  }
  if (!a.wait_prior_grid) {
    mla_attn_kernel<<<2 * a.num_work, attn::kThreads, attn::kSmemAlloc, stream>>>(tm_q, tm_kv, tm_kpe, p);
    return cudaGetLastError();
  }
  // Programmatic dependent of the append: set-up and query loads overlap it.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2u * static_cast<unsigned>(a.num_work));
  cfg.blockDim = dim3(attn::kThreads);
  cfg.dynamicSmemBytes = attn::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_attn_kernel, tm_q, tm_kv, tm_kpe, p);
}

cudaError_t launch_merge(const MergeParams& p, int num_merge, cudaStream_t stream) {
  // Programmatic dependent launch: the merge grid is set up while the attention grid
  // drains, and its griddepcontrol.wait releases it once that grid has finished.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_merge) * 16u);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_merge_kernel, p);
}

}  // namespace mla

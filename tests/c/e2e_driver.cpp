// End-to-end steps through the library's C ABI (include/mla.h) from a C++ serving
// loop: every step plans from host page tables (mla_plan), copies the step's queries
// from pinned host memory to the device, runs the attention (mla_run), copies the
// output (and lse) back to pinned host memory, and retires the plan of two steps
// earlier (mla_plan_check: its device status word; mla_plan_destroy).  Steps are
// pipelined two deep on three streams (uploads: plan and queries; runs; downloads), each
// parity with its own device buffers guarded by events, as a serving loop overlaps them.
//
//   e2e_driver DIR STEPS WARMUP SM_SCALE [DEVICE]
//
// DIR holds: tables (one step's tables in the int32 layout of plan_timer.cpp),
// q_nope.bin (bf16 [T][H][512]), q_pe.bin (bf16 [T][H][64]), cache.bin (bf16
// [num_pages][page_size][576]) and lse (one int32: 1 to download the lse as well).
// Prints "ms_per_step X", "h2d_bytes_per_step N", "d2h_bytes_per_step N", "status S":
// the device time from an event before the first timed step's plan upload to one after
// its last download, per step.
#include <cuda_runtime.h>

#include <cstdio>
#include <algorithm>
#include <cstdlib>
#include <deque>
#include <string>
#include <vector>

#include "mla.h"

namespace {

bool read_file(const std::string& path, std::vector<unsigned char>* out) {
  FILE* f = std::fopen(path.c_str(), "rb");
  if (!f) return false;
  std::fseek(f, 0, SEEK_END);
  const long n = std::ftell(f);
  std::fseek(f, 0, SEEK_SET);
  out->resize(static_cast<size_t>(n));
  const bool ok = n == 0 || std::fread(out->data(), 1, static_cast<size_t>(n), f) == static_cast<size_t>(n);
  std::fclose(f);
  return ok;
}

#define CK(x)                                                            \
  do {                                                                   \
    cudaError_t e_ = (x);                                                \
    if (e_ != cudaSuccess) {                                             \
      std::fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));      \
      return 3;                                                          \
    }                                                                    \
  } while (0)

}  // namespace

int main(int argc, char** argv) {
  if (argc < 5) {
    std::fprintf(stderr, "usage: %s DIR STEPS WARMUP SM_SCALE\n", argv[0]);
    return 2;
  }
  const std::string dir = argv[1];
  const int steps = std::atoi(argv[2]), warmup = std::atoi(argv[3]);
  const float sm_scale = static_cast<float>(std::atof(argv[4]));
  const int device = argc > 5 ? std::atoi(argv[5]) : 0;
  if (steps < 1 || warmup < 0) return 2;
  CK(cudaSetDevice(device));
  std::vector<unsigned char> tab, qn_f, qp_f, cache_f, lse_f;
  if (!read_file(dir + "/tables", &tab) || !read_file(dir + "/q_nope.bin", &qn_f) ||
      !read_file(dir + "/q_pe.bin", &qp_f) || !read_file(dir + "/cache.bin", &cache_f) ||
      !read_file(dir + "/lse", &lse_f))
    return 2;
  // every size is checked against the tables' header before anything is read
  const size_t n32 = tab.size() / 4;
  if (n32 < 5) return 2;
  const int32_t* t32 = reinterpret_cast<const int32_t*>(tab.data());
  const int32_t H = t32[0], P = t32[1], pages = t32[2], batch = t32[3], causal = t32[4];
  if (H <= 0 || P <= 0 || pages <= 0 || batch < 0 || n32 < 5 + 2 * (static_cast<size_t>(batch) + 1)) return 2;
  const int32_t* qo = t32 + 5;
  const int32_t* kvp = qo + batch + 1;
  if (kvp[batch] < 0 || n32 != 5 + 2 * (static_cast<size_t>(batch) + 1) + static_cast<size_t>(kvp[batch]) + batch)
    return 2;
  const int32_t* kvi = kvp + batch + 1;
  const int32_t* last = kvi + kvp[batch];
  const int32_t T = qo[batch];
  if (T < 0 || qn_f.size() != static_cast<size_t>(T) * H * 512 * 2 || qp_f.size() != static_cast<size_t>(T) * H * 64 * 2 ||
      cache_f.size() != static_cast<size_t>(pages) * P * 576 * 2)
    return 2;
  const bool want_lse = lse_f.size() >= 4 && *reinterpret_cast<const int32_t*>(lse_f.data()) != 0;
  const size_t qn_bytes = qn_f.size(), qp_bytes = qp_f.size();
  const size_t out_bytes = static_cast<size_t>(T) * H * 512 * 2, lse_bytes = static_cast<size_t>(T) * H * 4;

  mla_dims d{H, 512, 64, P, pages, sm_scale};
  // pinned host buffers: the step's queries, and its result
  void *qn_h = nullptr, *qp_h = nullptr, *out_h = nullptr, *lse_h = nullptr;
  CK(cudaMallocHost(&qn_h, qn_bytes));
  CK(cudaMallocHost(&qp_h, qp_bytes));
  CK(cudaMallocHost(&out_h, 2 * out_bytes));
  CK(cudaMallocHost(&lse_h, 2 * lse_bytes));
  std::copy(qn_f.begin(), qn_f.end(), static_cast<unsigned char*>(qn_h));
  std::copy(qp_f.begin(), qp_f.end(), static_cast<unsigned char*>(qp_h));
  // the cache is resident state (written by earlier steps of the layer)
  void* cache = nullptr;
  CK(cudaMalloc(&cache, cache_f.size()));
  CK(cudaMemcpy(cache, cache_f.data(), cache_f.size(), cudaMemcpyHostToDevice));
  struct Buf {
    void *qn, *qp, *out;
    float* lse;
    cudaEvent_t uploaded, computed, downloaded;
  } buf[2];
  for (Buf& b : buf) {
    CK(cudaMalloc(&b.qn, qn_bytes));
    CK(cudaMalloc(&b.qp, qp_bytes));
    CK(cudaMalloc(&b.out, out_bytes));
    CK(cudaMalloc(reinterpret_cast<void**>(&b.lse), lse_bytes));
    CK(cudaEventCreateWithFlags(&b.uploaded, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&b.computed, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&b.downloaded, cudaEventDisableTiming));
  }
  cudaStream_t s_up, s_run, s_down;
  CK(cudaStreamCreateWithFlags(&s_up, cudaStreamNonBlocking));
  CK(cudaStreamCreateWithFlags(&s_run, cudaStreamNonBlocking));
  CK(cudaStreamCreateWithFlags(&s_down, cudaStreamNonBlocking));

  std::deque<mla_plan_t> live;
  int status = 0;
  auto retire = [&]() {
    mla_plan_t p = live.front();
    live.pop_front();
    const mla_status st = mla_plan_check(p);  // waits for its run, reads its status word
    if (st != MLA_OK) status = st;
    mla_plan_destroy(p);
  };
  auto one = [&](int i) -> int {
    Buf& b = buf[i & 1];
    mla_plan_t p = nullptr;
    // the plan's upload goes on the upload stream, ahead of the queries: on the compute
    // stream it would wait for step i-1's run and then queue behind step i+1's query copy
    // in the copy engine; `uploaded` below orders the run after both
    const mla_status st = mla_plan(&d, batch, qo, kvp, kvi, last, causal, s_up, nullptr, &p);
    if (st != MLA_OK) return st;
    CK(cudaStreamWaitEvent(s_up, b.computed, 0));  // step i-2 has finished reading these
    CK(cudaMemcpyAsync(b.qn, qn_h, qn_bytes, cudaMemcpyHostToDevice, s_up));
    CK(cudaMemcpyAsync(b.qp, qp_h, qp_bytes, cudaMemcpyHostToDevice, s_up));
    CK(cudaEventRecord(b.uploaded, s_up));
    CK(cudaStreamWaitEvent(s_run, b.uploaded, 0));
    CK(cudaStreamWaitEvent(s_run, b.downloaded, 0));  // step i-2's result has left `out`
    const mla_status rs = mla_run(p, b.qn, b.qp, cache, b.out, want_lse ? b.lse : nullptr, s_run);
    if (rs != MLA_OK) return rs;
    CK(cudaEventRecord(b.computed, s_run));
    CK(cudaStreamWaitEvent(s_down, b.computed, 0));
    CK(cudaMemcpyAsync(static_cast<unsigned char*>(out_h) + (i & 1) * out_bytes, b.out, out_bytes,
                       cudaMemcpyDeviceToHost, s_down));
    if (want_lse)
      CK(cudaMemcpyAsync(static_cast<unsigned char*>(lse_h) + (i & 1) * lse_bytes, b.lse, lse_bytes,
                         cudaMemcpyDeviceToHost, s_down));
    CK(cudaEventRecord(b.downloaded, s_down));
    live.push_back(p);
    if (live.size() > 2) retire();
    return 0;
  };
  for (int i = 0; i < warmup; ++i)
    if (int r = one(i)) return r;
  while (!live.empty()) retire();
  CK(cudaDeviceSynchronize());
  cudaEvent_t e0, e1;
  CK(cudaEventCreate(&e0));
  CK(cudaEventCreate(&e1));
  CK(cudaEventRecord(e0, s_up));
  for (int i = 0; i < steps; ++i)
    if (int r = one(i)) return r;
  for (Buf& b : buf) CK(cudaStreamWaitEvent(s_down, b.downloaded, 0));
  CK(cudaEventRecord(e1, s_down));
  CK(cudaEventSynchronize(e1));
  while (!live.empty()) retire();
  float ms = 0.f;
  CK(cudaEventElapsedTime(&ms, e0, e1));
  // bytes crossing to the device each step: the queries, and the plan's upload (work
  // and merge lists, merge references, append rows, page table)
  size_t plan_bytes = 0;
  {
    mla_plan_t p = nullptr;
    mla_plan_info info{};
    if (mla_plan(&d, batch, qo, kvp, kvi, last, causal, s_run, nullptr, &p) == MLA_OK &&
        mla_plan_get_info(p, &info) == MLA_OK)
      plan_bytes = 32 * size_t(info.num_work) + 16 * size_t(info.num_merge) + 4 * size_t(info.num_merge_refs) +
                   4 * size_t(T) + 4 * size_t(kvp[batch]);
    mla_plan_destroy(p);
  }
  std::printf("ms_per_step %.6f\nh2d_bytes_per_step %zu\nd2h_bytes_per_step %zu\nstatus %d\n", ms / steps,
              qn_bytes + qp_bytes + plan_bytes, out_bytes + (want_lse ? lse_bytes : 0), status);
  return 0;
}

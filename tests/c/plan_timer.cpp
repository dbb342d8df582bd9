// Host time of the library's planning calls, measured from C++ through the C ABI
// (include/mla.h), with no Python in the loop.
//
//   plan_timer TABLES_FILE ITERS HOST_ONLY
//
// TABLES_FILE holds one step's tables as little-endian int32 values:
//   num_heads page_size num_pages batch causal
//   qo_indptr[batch+1] kv_indptr[batch+1] kv_indices[kv_indptr[batch]] last_page_len[batch]
// then, optionally, a second step in the same layout (the "changed" step for
// mla_plan_update; without it the first step's page ids are rotated by one page).
// HOST_ONLY = 1 plans on the host only (no CUDA call; a machine without a GPU);
// 0 makes real plans on the current device (uploads included, no synchronisation).
//
// Prints "key microseconds" lines: fresh (mla_plan alone; each plan is destroyed two
// plans later, outside the timed call), update_same (mla_plan_update with the tables
// unchanged), update_changed (alternating two steps).
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "mla.h"

namespace {

struct Step {
  int32_t H = 0, P = 0, pages = 0, batch = 0, causal = 1;
  std::vector<int32_t> qo, kvp, kvi, last;
};

bool read_step(FILE* f, Step* s) {
  int32_t hdr[5];
  if (std::fread(hdr, sizeof(int32_t), 5, f) != 5) return false;
  s->H = hdr[0];
  s->P = hdr[1];
  s->pages = hdr[2];
  s->batch = hdr[3];
  s->causal = hdr[4];
  auto rd = [&](std::vector<int32_t>& v, size_t n) {
    v.resize(n);
    return n == 0 || std::fread(v.data(), sizeof(int32_t), n, f) == n;
  };
  if (!rd(s->qo, s->batch + 1) || !rd(s->kvp, s->batch + 1)) return false;
  if (!rd(s->kvi, static_cast<size_t>(s->kvp[s->batch])) || !rd(s->last, s->batch)) return false;
  if (s->kvi.empty()) s->kvi.push_back(0);
  if (s->last.empty()) s->last.push_back(0);
  return true;
}

double now_us() {
  return std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now().time_since_epoch()).count();
}

}  // namespace

int main(int argc, char** argv) {
  if (argc < 4) {
    std::fprintf(stderr, "usage: %s TABLES_FILE ITERS HOST_ONLY\n", argv[0]);
    return 2;
  }
  FILE* f = std::fopen(argv[1], "rb");
  if (!f) return 2;
  Step a, b;
  if (!read_step(f, &a)) return 2;
  if (!read_step(f, &b)) {
    b = a;
    for (auto& x : b.kvi) x = (x + 1) % a.pages;
  }
  std::fclose(f);
  const int iters = std::atoi(argv[2]);
  mla_dims d{a.H, 512, 64, a.P, a.pages > b.pages ? a.pages : b.pages, 0.0721687836f};
  mla_plan_options o{};
  o.host_only = std::atoi(argv[3]) != 0;

  // fresh plans, each destroyed two plans later (as a pipelined serving loop retires
  // them, its buffers returning to the library's pool); only mla_plan is timed
  mla_plan_t p = nullptr, live[3] = {nullptr, nullptr, nullptr};
  double fresh_total = 0.0;
  for (int i = 0; i < iters + 3; ++i) {
    const Step& s = (i & 1) ? b : a;
    const double t0 = now_us();
    if (mla_plan(&d, s.batch, s.qo.data(), s.kvp.data(), s.kvi.data(), s.last.data(), s.causal, nullptr, &o, &p))
      return 3;
    if (i >= 3) fresh_total += now_us() - t0;  // the first three warm the pool
    mla_plan_destroy(live[i % 3]);
    live[i % 3] = p;
  }
  for (mla_plan_t x : live) mla_plan_destroy(x);
  const double fresh = fresh_total / iters;

  if (mla_plan(&d, a.batch, a.qo.data(), a.kvp.data(), a.kvi.data(), a.last.data(), a.causal, nullptr, &o, &p))
    return 3;
  int32_t reused = 0;
  double t0 = now_us();
  for (int i = 0; i < iters; ++i)
    if (mla_plan_update(p, a.batch, a.qo.data(), a.kvp.data(), a.kvi.data(), a.last.data(), nullptr, &reused) ||
        !reused)
      return 4;
  const double same = (now_us() - t0) / iters;
  t0 = now_us();
  for (int i = 0; i < iters; ++i) {
    const Step& s = (i & 1) ? a : b;
    if (mla_plan_update(p, s.batch, s.qo.data(), s.kvp.data(), s.kvi.data(), s.last.data(), nullptr, &reused) ||
        reused)
      return 5;
  }
  const double changed = (now_us() - t0) / iters;
  mla_plan_destroy(p);
  std::printf("fresh %.3f\nupdate_same %.3f\nupdate_changed %.3f\n", fresh, same, changed);
  return 0;
}

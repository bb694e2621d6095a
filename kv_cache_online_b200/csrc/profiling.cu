// Opt-in stage timing and the launch counter (see profiling.h), and their C ABI.
#include <atomic>
#include <mutex>
#include <vector>

#include "iskv.h"
#include "profiling.h"

namespace iskv {

namespace {

struct Pending {
  int stage;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_enabled = false;
std::vector<cudaEvent_t> g_free;
std::vector<Pending> g_pending;
cudaEvent_t g_last = nullptr;  // last event recorded by the current section
double g_ms[ST_COUNT] = {0};
long long g_calls[ST_COUNT] = {0};
std::atomic<long long> g_launches{0};

const char *kNames[ST_COUNT] = {
    "fold.project",   "fold.residual_qr_svd", "fold.core_svd",      "fold.basis_rotate",
    "fold.coord_rotate", "fold.finalize",     "reorth.gram",        "reorth.newton_schulz",
    "reorth.core_svd", "reorth.coord_rotate", "reorth.basis_rotate", "reconstruct.prepare",
    "reconstruct.compressed",
    "reconstruct.exact", "select",            "job_upload",        "attention.prepare",
    "attention.scores", "attention.softmax",  "attention.values", "cache.append",
    "cache.evict"};

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void collect_locked() {
  for (const Pending &p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      g_ms[p.stage] += ms;
      g_calls[p.stage] += 1;
    }
  }
  // Events are shared between neighbouring stages: free each once.
  std::vector<cudaEvent_t> seen;
  for (const Pending &p : g_pending) {
    for (cudaEvent_t e : {p.a, p.b}) {
      bool dup = false;
      for (cudaEvent_t s : seen) dup |= (s == e);
      if (!dup) seen.push_back(e);
    }
  }
  if (g_last) {
    bool dup = false;
    for (cudaEvent_t s : seen) dup |= (s == g_last);
    if (!dup) seen.push_back(g_last);
  }
  for (cudaEvent_t e : seen) g_free.push_back(e);
  g_pending.clear();
  g_last = nullptr;
}

}  // namespace

const char *stage_name(int s) { return (s >= 0 && s < ST_COUNT) ? kNames[s] : ""; }

void stage_begin(cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_enabled) return;
  cudaEvent_t e = take_event();
  cudaEventRecord(e, s);
  if (g_last) {
    // a previous section's last event is no longer needed as a start
    bool used = false;
    for (const Pending &p : g_pending) used |= (p.a == g_last || p.b == g_last);
    if (!used) g_free.push_back(g_last);
  }
  g_last = e;
}

void stage_mark(cudaStream_t s, int id) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_enabled || !g_last) return;
  cudaEvent_t e = take_event();
  cudaEventRecord(e, s);
  g_pending.push_back({id, g_last, e});
  g_last = e;
  if (g_pending.size() > 4096) collect_locked();
}

void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

}  // namespace iskv

using namespace iskv;

extern "C" {

int32_t iskv_stage_timing(int32_t enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  const bool was = g_enabled;
  collect_locked();
  g_enabled = enable != 0;
  return was ? 1 : 0;
}

int32_t iskv_stage_count(void) { return ST_COUNT; }

const char *iskv_stage_name(int32_t i) { return stage_name(i); }

iskv_status iskv_stage_read(double *ms, int64_t *calls) {
  std::lock_guard<std::mutex> lk(g_mu);
  collect_locked();
  for (int i = 0; i < ST_COUNT; ++i) {
    if (ms) ms[i] = g_ms[i];
    if (calls) calls[i] = g_calls[i];
  }
  return ISKV_OK;
}

void iskv_stage_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  collect_locked();
  for (int i = 0; i < ST_COUNT; ++i) {
    g_ms[i] = 0.0;
    g_calls[i] = 0;
  }
}

int64_t iskv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

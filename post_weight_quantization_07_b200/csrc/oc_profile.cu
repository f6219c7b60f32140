// Per-phase device timing and launch counting.  When enabled, each phase of a
// call records a CUDA event pair on the call's stream; oc_profile_read()
// waits for them and returns the accumulated milliseconds and kernel launches
// per phase.  Launches are counted always (a plain counter).
#include <atomic>
#include <vector>

#include "oc_internal.cuh"

namespace oc {
namespace {

struct Rec {
  int phase;
  cudaEvent_t a, b;
  int64_t launches;
};

std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;
bool g_on = false;
std::atomic<int64_t> g_launches{0};

const char* const kPhaseNames[kNumPhases] = {
    "hessian_syrk", "qep_cross", "qep_syrk", "qep_w_delta", "factor",
    "qep_apply", "gptq_prep", "gptq_sweep", "gptq_trailing", "gptq_pack",
    "hessian_fixup", "qep_cross_fixup", "hadamard_rotate", "lpcd_left_project", "dequant_gemv", "qep_diff"};

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  check_cuda(cudaEventCreate(&e), "cudaEventCreate");
  return e;
}

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void count_launches(int64_t k) { g_launches.fetch_add(k, std::memory_order_relaxed); }

PhaseScope::PhaseScope(const Ctx& c, Phase p) : stream_(c.stream), phase_(p) {
  if (!g_on) return;
  a_ = take_event();
  if (cudaEventRecord(a_, stream_) != cudaSuccess) {
    g_pool.push_back(a_);
    return;
  }
  l0_ = g_launches.load(std::memory_order_relaxed);
  active_ = true;
}

PhaseScope::~PhaseScope() {
  if (!active_) return;
  cudaEvent_t b = nullptr;
  if (!g_pool.empty()) {
    b = g_pool.back();
    g_pool.pop_back();
  } else if (cudaEventCreate(&b) != cudaSuccess) {
    return;
  }
  if (cudaEventRecord(b, stream_) != cudaSuccess) return;
  g_recs.push_back({static_cast<int>(phase_), a_, b, g_launches.load(std::memory_order_relaxed) - l0_});
}

void profile_enable(bool on) { g_on = on; }

int profile_read(double* ms, int64_t* launches, int max_phases) {
  const int np = max_phases < kNumPhases ? max_phases : kNumPhases;
  for (int i = 0; i < np; ++i) {
    if (ms) ms[i] = 0.0;
    if (launches) launches[i] = 0;
  }
  for (const Rec& r : g_recs) {
    check_cuda(cudaEventSynchronize(r.b), "cudaEventSynchronize");
    float t = 0.f;
    check_cuda(cudaEventElapsedTime(&t, r.a, r.b), "cudaEventElapsedTime");
    if (r.phase < np) {
      if (ms) ms[r.phase] += t;
      if (launches) launches[r.phase] += r.launches;
    }
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  return kNumPhases;
}

const char* phase_name(int p) { return (p >= 0 && p < kNumPhases) ? kPhaseNames[p] : ""; }

int64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

}  // namespace oc

// Optional per-stage timing with CUDA events and a count of kernel launches.
//
// When stage timing is on, every compress/decode stage is bracketed by two
// events recorded on the caller's stream; anchorkv_stage_times() waits for
// them and adds the elapsed times per stage.  Off (the default), nothing is
// recorded and the only cost is one branch per stage.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

struct Mark {
  int stage;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Mark> g_marks;
std::vector<cudaEvent_t> g_pool;
int64_t g_launches = 0;
static_assert(kStageCount == ANCHORKV_N_STAGES, "stage table and header disagree");
double g_ms[kStageCount];
int64_t g_calls[kStageCount];
cudaEvent_t g_open[kStageCount];

cudaEvent_t get_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

const char* kNames[kStageCount] = {"obs_pass1", "obs_combine", "token_stats", "anchor_select", "assign",
                                   "assign_refine", "project", "select_topR", "quantize", "decode_prep",
                                   "decode_split", "decode_combine", "obs_alpha", "obs_key_term", "decode_attn",
                                   "decode_rope"};

}  // namespace

void stage_begin(int stage, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  g_open[stage] = get_event();
  cudaEventRecord(g_open[stage], s);
}

void stage_end(int stage, cudaStream_t s, int kernels) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_launches += kernels;
  if (!g_on || !g_open[stage]) return;
  cudaEvent_t b = get_event();
  cudaEventRecord(b, s);
  g_marks.push_back({stage, g_open[stage], b});
  g_open[stage] = nullptr;
}

}  // namespace akv

using namespace akv;

extern "C" {

int anchorkv_stage_timing(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = enable != 0;
  for (int i = 0; i < kStageCount; ++i) { g_ms[i] = 0.0; g_calls[i] = 0; }
  return ANCHORKV_OK;
}

int anchorkv_stage_times(double* ms_out, int64_t* calls_out, int32_t n) {
  if (!ms_out || !calls_out || n < kStageCount) return ANCHORKV_EINVAL;
  std::lock_guard<std::mutex> lk(g_mu);
  for (const Mark& m : g_marks) {
    if (cudaEventSynchronize(m.b) != cudaSuccess) return ANCHORKV_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, m.a, m.b) != cudaSuccess) return ANCHORKV_ECUDA;
    g_ms[m.stage] += ms;
    g_calls[m.stage] += 1;
    g_pool.push_back(m.a);
    g_pool.push_back(m.b);
  }
  g_marks.clear();
  for (int i = 0; i < kStageCount; ++i) { ms_out[i] = g_ms[i]; calls_out[i] = g_calls[i]; }
  return ANCHORKV_OK;
}

const char* anchorkv_stage_name(int32_t stage) {
  return (stage >= 0 && stage < kStageCount) ? kNames[stage] : "";
}

int anchorkv_launch_count(int64_t* out) {
  if (!out) return ANCHORKV_EINVAL;
  std::lock_guard<std::mutex> lk(g_mu);
  *out = g_launches;
  return ANCHORKV_OK;
}

}  // extern "C"

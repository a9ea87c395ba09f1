// prof.cu -- optional per-kernel timing with CUDA events on the launching
// stream (off by default; switched on by ttt_profile_begin).
#include <mutex>
#include <vector>

#include "../../include/ttt.h"
#include "kernels.h"

namespace ttt {

static const char* kKindNames[K_NUM] = {
    "ttt_linear_simt", "ttt_linear_umma", "lact_cast",     "lact_keypass",
    "gemm_read",       "gemm_grad",       "lact_update",   "muon_momentum",
    "ns_prep",         "gemm_ns",         "muon_apply",    "lact_keygrad",
    "ttt_linear_segstate", "ttt_linear_bwd_ew", "window_attention", "lact_loop", "lact_bwd_fwd",
    "lact_bwd_gemm"};

struct ProfRec {
  int kind;
  cudaEvent_t e0, e1;
};

static std::mutex g_mu;
static bool g_on = false;
static std::vector<ProfRec> g_recs;
static std::vector<cudaEvent_t> g_pool;
static cudaEvent_t g_pending[K_NUM];

static cudaEvent_t get_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void prof_before(int kind, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  g_pending[kind] = get_event();
  cudaEventRecord(g_pending[kind], s);
}

void prof_after(int kind, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || g_pending[kind] == nullptr) return;
  cudaEvent_t e1 = get_event();
  cudaEventRecord(e1, s);
  g_recs.push_back({kind, g_pending[kind], e1});
  g_pending[kind] = nullptr;
}

}  // namespace ttt

extern "C" {

int ttt_profile_begin(void) {
  std::lock_guard<std::mutex> lk(ttt::g_mu);
  for (auto& r : ttt::g_recs) {
    ttt::g_pool.push_back(r.e0);
    ttt::g_pool.push_back(r.e1);
  }
  ttt::g_recs.clear();
  for (auto& p : ttt::g_pending) p = nullptr;
  ttt::g_on = true;
  return TTT_OK;
}

int ttt_profile_end(ttt_prof_entry* entries, int max_entries, int* n_entries) {
  std::lock_guard<std::mutex> lk(ttt::g_mu);
  ttt::g_on = false;
  if (!n_entries) return TTT_ERR_ARG;
  int launches[ttt::K_NUM] = {0};
  double ms[ttt::K_NUM] = {0};
  for (auto& r : ttt::g_recs) {
    if (cudaEventSynchronize(r.e1) != cudaSuccess) return TTT_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.e0, r.e1) != cudaSuccess) return TTT_ERR_CUDA;
    launches[r.kind] += 1;
    ms[r.kind] += t;
  }
  int n = 0;
  for (int k = 0; k < ttt::K_NUM; ++k) {
    if (launches[k] == 0) continue;
    if (entries && n < max_entries) {
      snprintf(entries[n].name, sizeof(entries[n].name), "%s", ttt::kKindNames[k]);
      entries[n].launches = launches[k];
      entries[n].total_ms = ms[k];
    }
    ++n;
  }
  *n_entries = n;
  return TTT_OK;
}

}  // extern "C"

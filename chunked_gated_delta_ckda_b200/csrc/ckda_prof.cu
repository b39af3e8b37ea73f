// ckda_prof.cu -- optional per-kernel timing with CUDA events recorded on the
// launch stream around each kernel launch (off by default; host only).
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "ckda_internal.cuh"

namespace ckda {
namespace {
struct Rec {
  const char *name;
  cudaEvent_t a, b;
};
struct Agg {
  std::string name;
  int count;
  double total_ms;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_open;      // recorded, not yet collected
std::vector<cudaEvent_t> g_pool;
std::vector<Agg> g_agg;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

ProfScope::ProfScope(const char *name, cudaStream_t s) : idx_(-1), s_(s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  Rec r{name, take_event(), take_event()};
  if (!r.a || !r.b) return;
  if (cudaEventRecord(r.a, s) != cudaSuccess) return;
  g_open.push_back(r);
  idx_ = (int)g_open.size() - 1;
}

ProfScope::~ProfScope() {
  if (idx_ < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (idx_ < (int)g_open.size()) cudaEventRecord(g_open[idx_].b, s_);
}

}  // namespace ckda

using namespace ckda;

extern "C" {

int ckda_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int prev = g_on ? 1 : 0;
  g_on = on != 0;
  return prev;
}

int ckda_profile_collect(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (Rec &r : g_open) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -CKDA_ERR_CUDA;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -CKDA_ERR_CUDA;
    bool found = false;
    for (Agg &a : g_agg)
      if (a.name == r.name) {
        a.count += 1;
        a.total_ms += ms;
        found = true;
        break;
      }
    if (!found) g_agg.push_back(Agg{r.name, 1, (double)ms});
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_open.clear();
  return (int)g_agg.size();
}

int ckda_profile_get(int i, char *name, int name_len, int *count, double *total_ms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (i < 0 || i >= (int)g_agg.size() || !name || name_len < 1) return CKDA_ERR_INVALID_ARG;
  std::strncpy(name, g_agg[i].name.c_str(), name_len - 1);
  name[name_len - 1] = '\0';
  if (count) *count = g_agg[i].count;
  if (total_ms) *total_ms = g_agg[i].total_ms;
  return CKDA_OK;
}

void ckda_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_agg.clear();
  for (Rec &r : g_open) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_open.clear();
}

}  // extern "C"

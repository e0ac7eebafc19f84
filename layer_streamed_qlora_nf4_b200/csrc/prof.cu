// Measurement hooks: kernel-launch counter, per-launch CUDA-event timing of the
// heavy kernel classes (recorded on the stream each kernel is launched on),
// and the standalone AdamW entry point.
#include <atomic>
#include <mutex>
#include <string.h>
#include <string>
#include <vector>

#include "common.cuh"

namespace lsq {

static std::atomic<int64_t> g_launches{0};

cudaError_t launched(cudaError_t e) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

namespace {

struct Rec {
  int cls;
  int e0, e1;
  double flops, bytes;
};

struct Profiler {
  std::mutex mu;
  bool enabled = false;
  std::vector<cudaEvent_t> pool;
  size_t next = 0;
  std::vector<Rec> recs;
  std::vector<std::string> names;
  int event() {
    if (next == pool.size()) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return -1;
      pool.push_back(e);
    }
    return (int)next++;
  }
  int cls(const char* n) {
    for (size_t i = 0; i < names.size(); ++i)
      if (names[i] == n) return (int)i;
    names.push_back(n);
    return (int)names.size() - 1;
  }
};

Profiler& prof() {
  static Profiler p;
  return p;
}

}  // namespace

int prof_begin(cudaStream_t st) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.enabled) return -1;
  const int e = p.event();
  if (e < 0) return -1;
  cudaEventRecord(p.pool[e], st);
  return e;
}

void prof_end(int token, cudaStream_t st, const char* name, double flops, double bytes) {
  if (token < 0) return;
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.enabled) return;
  const int e = p.event();
  if (e < 0) return;
  cudaEventRecord(p.pool[e], st);
  p.recs.push_back(Rec{p.cls(name), token, e, flops, bytes});
}

}  // namespace lsq

using namespace lsq;

extern "C" int64_t lsq_launch_counter(void) { return g_launches.load(); }

extern "C" int lsq_profile_enable(int enable) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (enable) {
    p.recs.clear();
    p.next = 0;
  }
  p.enabled = enable != 0;
  return LSQ_OK;
}

extern "C" int lsq_profile_read(lsq_prof_entry* out, int32_t max, int32_t* n_out) {
  if (!out || !n_out || max < 0) return set_error(LSQ_ERR_INVALID, "lsq_profile_read: null output");
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  std::vector<lsq_prof_entry> agg(p.names.size());
  for (size_t i = 0; i < p.names.size(); ++i) {
    memset(&agg[i], 0, sizeof(lsq_prof_entry));
    strncpy(agg[i].name, p.names[i].c_str(), sizeof(agg[i].name) - 1);
  }
  for (const Rec& r : p.recs) {
    LSQ_CUDA(cudaEventSynchronize(p.pool[r.e1]));
    float ms = 0.f;
    LSQ_CUDA(cudaEventElapsedTime(&ms, p.pool[r.e0], p.pool[r.e1]));
    lsq_prof_entry& a = agg[r.cls];
    a.launches += 1;
    a.total_ms += ms;
    a.flops += r.flops;
    a.bytes += r.bytes;
  }
  int n = 0;
  for (size_t i = 0; i < agg.size() && n < max; ++i)
    if (agg[i].launches > 0) out[n++] = agg[i];
  *n_out = n;
  return LSQ_OK;
}

extern "C" int lora_adamw_step(float* lora, const float* grad, const lsq_adamw* opt, int64_t n,
                               void* stream) {
  if (!lora || !grad || !opt || !opt->m || !opt->v)
    return set_error(LSQ_ERR_INVALID, "lora_adamw_step: null pointer");
  if (n <= 0 || opt->step < 1) return set_error(LSQ_ERR_SHAPE, "lora_adamw_step: n > 0, step >= 1");
  return launch_adamw(lora, grad, opt->m, opt->v, n, opt->lr, opt->beta1, opt->beta2, opt->eps,
                      opt->weight_decay, opt->step, static_cast<cudaStream_t>(stream));
}

// Measurement hooks: kernel-launch counter, per-launch CUDA-event timing of the
// heavy kernel classes (recorded on the stream each kernel is launched on, or,
// for launches captured into a CUDA graph, by event-record nodes of that graph),
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
int64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }
void count_launches(int64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {

struct Rec {
  int cls;
  int e0, e1;
  double flops, bytes;
};

struct Agg {
  int64_t launches = 0;
  double ms = 0, flops = 0, bytes = 0;
};

struct Profiler {
  std::mutex mu;
  bool enabled = false;
  std::vector<cudaEvent_t> pool;
  size_t next = 0;
  std::vector<Rec> recs;
  std::vector<std::string> names;
  std::vector<Agg> graph_acc;  // per class: regions replayed inside CUDA graphs
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

// Capture mode (per thread): the sink of the graph being captured, and the
// begin events of its open regions (a token is kCapTag | index).
thread_local std::vector<ProfRec>* t_sink = nullptr;
thread_local std::vector<cudaEvent_t> t_open;
constexpr int kCapTag = 1 << 30;

}  // namespace

bool prof_enabled() {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  return p.enabled;
}

void prof_capture_sink(std::vector<ProfRec>* sink) {
  t_sink = sink;
  t_open.clear();
}

int prof_begin(cudaStream_t st) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.enabled) return -1;
  if (t_sink) {
    // "external": a real event-record node of the graph (a plain record during
    // capture would only express an ordering dependency)
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    t_open.push_back(e);
    return kCapTag | (int)(t_open.size() - 1);
  }
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
  if (token & kCapTag) {
    const size_t i = (size_t)(token & ~kCapTag);
    if (!t_sink || i >= t_open.size()) return;
    cudaEvent_t e1;
    if (cudaEventCreate(&e1) != cudaSuccess) return;
    cudaEventRecordWithFlags(e1, st, cudaEventRecordExternal);
    t_sink->push_back(ProfRec{p.cls(name), t_open[i], e1, flops, bytes});
    return;
  }
  const int e = p.event();
  if (e < 0) return;
  cudaEventRecord(p.pool[e], st);
  p.recs.push_back(Rec{p.cls(name), token, e, flops, bytes});
}

int prof_accumulate(const std::vector<ProfRec>& recs) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.enabled) return LSQ_OK;
  if (p.graph_acc.size() < p.names.size()) p.graph_acc.resize(p.names.size());
  for (const ProfRec& r : recs) {
    float ms = 0.f;
    LSQ_CUDA(cudaEventElapsedTime(&ms, r.e0, r.e1));
    Agg& a = p.graph_acc[r.cls];
    a.launches += 1;
    a.ms += ms;
    a.flops += r.flops;
    a.bytes += r.bytes;
  }
  return LSQ_OK;
}

void prof_release(std::vector<ProfRec>& recs) {
  for (ProfRec& r : recs) {
    cudaEventDestroy(r.e0);
    cudaEventDestroy(r.e1);
  }
  recs.clear();
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
    p.graph_acc.clear();
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
  for (size_t i = 0; i < p.graph_acc.size() && i < agg.size(); ++i) {
    agg[i].launches += p.graph_acc[i].launches;
    agg[i].total_ms += p.graph_acc[i].ms;
    agg[i].flops += p.graph_acc[i].flops;
    agg[i].bytes += p.graph_acc[i].bytes;
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

// The streamed decoder stack and one SFT optimiser step.
//
// Method (Soup layer-streaming tutorial, "四段資料路徑" parts 2-3; Layer Streaming
// blog, "層流技術：技術實作與記憶體效率"; RepoDaily review, "架构解读"): the frozen
// decoder stack lives in page-locked host memory; two fixed VRAM buffers take
// one layer each; while the GPU computes layer i from one buffer, a dedicated
// copy stream loads the next layer into the other; forward walks 0..L-1,
// backward walks L-1..0 recomputing each layer, so each layer is needed twice
// per micro-batch.  Embedding, lm_head, LoRA, gradients and optimiser state
// stay resident.
//
// Schedule: the sequence of layer visits of the whole step is planned on the
// host.  A visit whose layer is already in a buffer uses it in place (the turn
// from forward to backward, and the first layers of the next step or
// micro-batch, find their layers still resident); otherwise the layer is copied
// into the buffer the previous visit did not use.  Fences: the copy stream
// waits on the event recorded after the last compute that read the target
// buffer ("free"); the compute stream waits on the event recorded after the
// copy ("ready").  Copies run one visit ahead.  Kernels are deterministic, so
// a streamed step is bit-identical to the same step with the stack resident.
//
// Launches: the kernels of each layer visit (a forward, an adapter-off
// reference forward, or a recomputing backward) are captured once into a CUDA
// graph and replayed.  Eager launches would each have their command fetched
// from host memory over the same PCIe link the layer copy saturates, which
// slowed a layer's kernels by about a quarter on B200; a replayed graph's work
// is already on the device.  A graph bakes in the step's buffers, so the cache
// is rebuilt whenever a step passes different ones.
//
// Data-parallel layer sharding (stream_stack_shard): with G ranks, one process
// per GPU, each rank copies only its 1/G slice of a layer from host memory, and
// an in-place NCCL all-gather on the copy stream (NVLink / NVSwitch, far faster
// than each GPU's own host link) assembles the whole layer in every rank's
// buffer before the "ready" event.  Per-GPU host->device bytes fall by G.  The
// NCCL library is loaded at run time (the one torch already loaded, else the
// system's), so the library has no link-time dependency on it.
#include <cstdlib>
#include <dlfcn.h>
#include <nccl.h>
#include <string.h>

#include <algorithm>
#include <chrono>
#include <cmath>
#include <map>
#include <mutex>
#include <thread>
#include <tuple>
#include <vector>

#include "common.cuh"

struct lsq_stack {
  lsq_cfg cfg;
  lsq::LayerShapes shapes;
  lsq_layer_layout layout;
  lsq_lora_layout lora_layout;
  std::vector<const void*> blobs;
  void* buf[2];
  int resident;
  int device;
  cudaStream_t copy_stream;
  cudaEvent_t ready[2], freed[2];
  int buf_layer[2];            // layer held by each buffer (after the enqueued copies)
  std::vector<cudaEvent_t> wait_ev;  // pairs around each compute-side wait (timing)
  cudaEvent_t t_start, t_end, done;
  float* loss_host;            // pinned: [0] loss, [1 ..] DPO log-probabilities
  lsq_step_stats stats;
  int n_waits_last;
  // data-parallel layer sharding (stream_stack_shard); shard == 0: every layer
  // is copied whole from this rank's host blob
  int world = 1, rank = 0;
  size_t shard = 0;            // bytes of a layer each rank fetches from host
  void* comm = nullptr;        // ncclComm_t
  int aborted = 0;             // the communicator was aborted after a timeout
  // data-parallel gradient averaging (stream_stack_reduce_grads): its own
  // communicator and stream, so the per-layer all-reduces overlap the backward
  void* grad_comm = nullptr;   // ncclComm_t
  int grad_world = 1;
  cudaStream_t red_stream = nullptr;
  cudaEvent_t red_ev = nullptr, red_done = nullptr;
  // CUDA graphs of the layer visits, keyed by (kind: 0 forward, 1 adapter-off
  // reference forward, 2 backward; layer; buffer; accumulate; micro-batch when
  // profiling), valid while the step's pointers and sizes (graph_sig) are unchanged
  struct GraphEntry {
    cudaGraphExec_t exec = nullptr;
    int64_t launches = 0;               // kernels in the graph
    std::vector<lsq::ProfRec> recs;     // profiler regions inside it
  };
  std::map<std::tuple<int, int, int, int, int>, GraphEntry> graphs;
  std::vector<uintptr_t> graph_sig;
  cudaStream_t cap_stream = nullptr;    // capture only (nothing runs on it)
};

namespace {
void drop_graphs(lsq_stack* h) {
  for (auto& kv : h->graphs) {
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
    lsq::prof_release(kv.second.recs);
  }
  h->graphs.clear();
  h->graph_sig.clear();
}
}  // namespace

namespace lsq {
namespace {

struct StackWs {
  float* xs;         // [L+1][T][D] fp32: layer inputs (saved for backward) and final hidden
  uint16_t* hf;      // [T][D] final-norm output
  float* rstd_f;     // [T]
  int64_t head_T;    // tokens per lm_head / cross-entropy chunk (whole sequences)
  float* logits;     // [head_T][V]
  uint16_t* dlogits; // [head_T][V]
  float* row_loss;   // [T]
  float* loss_dev;   // [1]
  float* dhf;        // [T][D]
  float2* rope_cs;   // [seq][d/2] RoPE cos/sin table, built once per step
  uint16_t* lora16;  // [L][lora16 elems] LoRA operands in product types, once per step
  uint8_t* saved_u;  // [L][saved_u_bytes] each layer's rank-r products u, forward -> backward
  size_t saved_u_bytes;
  float* dh[2];      // [T][D] fp32 residual-stream gradient (ping-pong)
  uint16_t* dhb[2];  // bf16 copies
  void* gemm;
  size_t gemm_bytes;
  void* layer_ws;
  size_t layer_ws_bytes;
  // DPO step only
  float* xr[2];      // [T][D] fp32: the reference (adapter-off) hidden state, ping-pong
  float* row_ref;    // [T] reference per-row -log p
  float* seq_scale;  // [2 * pairs] dlogits coefficient per sequence
  float* logps;      // [4 * pairs]
};

constexpr int kMaxPairs = 32;

GemmDesc head_fwd(const uint16_t* lm_head, int64_t V, int64_t D, const uint16_t* hf, int64_t T,
                  float* logits) {
  GemmDesc d;
  d.wmode = W_BF16_N;
  d.M = V;
  d.T = T;
  d.Kc = D;
  d.w = lm_head;
  d.w_rows = V;
  d.w_cols = D;
  d.act = hf;
  d.act_ld = D;
  d.out = logits;
  d.out_f32 = 1;
  d.ldo = V;
  d.prof_name = "gemm_bf16_head";
  return d;
}

GemmDesc head_dx(const uint16_t* lm_head, int64_t V, int64_t D, const uint16_t* dlogits,
                 int64_t T, float* dhf) {
  GemmDesc d;
  d.wmode = W_BF16_T;
  d.M = D;
  d.T = T;
  d.Kc = V;
  d.w = lm_head;
  d.w_rows = V;
  d.w_cols = D;
  d.act = dlogits;
  d.act_ld = V;
  d.out = dhf;
  d.out_f32 = 1;
  d.ldo = D;
  d.prof_name = "gemm_bf16_head_dx";
  return d;
}

// Tokens per lm_head chunk: whole sequences, as many as keep the chunk's fp32
// logits and bf16 logit gradients within 4 GiB (at least one sequence), or
// LSQ_HEAD_CHUNK_SEQS sequences when that is set in the environment; the DPO
// step needs every row's loss before any logit gradient, so it takes all T.
int64_t head_chunk_tokens(const lsq_cfg* cfg, int64_t T, int seq, bool dpo) {
  if (dpo || seq <= 0) return T;
  const int64_t per_seq = (int64_t)cfg->vocab * 6 * seq;
  int64_t seqs = std::max<int64_t>(1, (int64_t(4) << 30) / std::max<int64_t>(per_seq, 1));
  if (const char* e = std::getenv("LSQ_HEAD_CHUNK_SEQS")) {
    const long v = std::strtol(e, nullptr, 10);
    if (v > 0) seqs = v;
  }
  return std::min<int64_t>(T, seqs * seq);
}

size_t plan_stack_ws(const lsq_cfg* cfg, const LayerShapes& s, int64_t T, int seq, void* base,
                     StackWs* w, bool dpo = false) {
  Arena a;
  a.base = static_cast<uint8_t*>(base);
  a.cap = SIZE_MAX;
  StackWs x{};
  const int64_t V = cfg->vocab, D = s.D;
  x.xs = a.take<float>((size_t)(cfg->n_layers + 1) * T * D);
  x.hf = a.take<uint16_t>(T * D);
  x.rstd_f = a.take<float>(T);
  x.head_T = head_chunk_tokens(cfg, T, seq, dpo);
  x.logits = a.take<float>((size_t)x.head_T * V);
  x.dlogits = a.take<uint16_t>((size_t)x.head_T * V);
  x.row_loss = a.take<float>(T);
  x.loss_dev = a.take<float>(64);
  x.dhf = a.take<float>(T * D);
  x.rope_cs = a.take<float2>(T * s.hd / 2);  // >= seq * d/2 entries
  x.lora16 = a.take<uint16_t>((size_t)cfg->n_layers * lora16_elems_per_layer(cfg));
  x.saved_u_bytes = layer_saved_u_bytes(cfg, T);
  x.saved_u = a.take<uint8_t>((size_t)cfg->n_layers * x.saved_u_bytes);
  for (int i = 0; i < 2; ++i) {
    x.dh[i] = a.take<float>(T * D);
    x.dhb[i] = a.take<uint16_t>(T * D);
  }
  const size_t gb =
      std::max(gemm_workspace_bytes(head_fwd(nullptr, V, D, nullptr, x.head_T, nullptr)),
               gemm_workspace_bytes(head_dx(nullptr, V, D, nullptr, x.head_T, nullptr)));
  x.gemm = a.take<uint8_t>(gb + 256);
  x.gemm_bytes = gb + 256;
  x.layer_ws_bytes = layer_ws_bytes(cfg, T);
  x.layer_ws = a.take<uint8_t>(x.layer_ws_bytes);
  if (dpo) {
    x.xr[0] = a.take<float>(T * D);
    x.xr[1] = a.take<float>(T * D);
    x.row_ref = a.take<float>(T);
    x.seq_scale = a.take<float>(2 * kMaxPairs);
    x.logps = a.take<float>(4 * kMaxPairs);
  }
  if (w) *w = x;
  return a.used;
}

struct Visit {
  int layer;
  int fwd;
  int buf;
  int copy;
};

// Plans buffer use for the visit sequence, starting from the buffers' contents.
std::vector<Visit> plan_visits(int L, int micro_batches, int bl0, int bl1) {
  std::vector<Visit> v;
  int held[2] = {bl0, bl1};
  int prev_buf = 1;  // so that the first copy goes to buffer 0
  for (int mb = 0; mb < micro_batches; ++mb) {
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = 0; k < L; ++k) {
        const int layer = pass == 0 ? k : L - 1 - k;
        Visit x{layer, pass == 0, 0, 0};
        if (held[0] == layer)
          x.buf = 0;
        else if (held[1] == layer)
          x.buf = 1;
        else {
          x.buf = 1 - prev_buf;
          x.copy = 1;
          held[x.buf] = layer;
        }
        prev_buf = x.buf;
        v.push_back(x);
      }
    }
  }
  return v;
}

// NCCL entry points, resolved once from libnccl.so.2 at run time.
struct NcclFns {
  decltype(&ncclGetUniqueId) get_unique_id = nullptr;
  decltype(&ncclCommInitRank) init_rank = nullptr;
  decltype(&ncclAllGather) all_gather = nullptr;
  decltype(&ncclAllReduce) all_reduce = nullptr;
  decltype(&ncclCommDestroy) destroy = nullptr;
  decltype(&ncclCommAbort) abort = nullptr;
  decltype(&ncclGetErrorString) error_string = nullptr;
};

int nccl_fns(const NcclFns** out) {
  static std::mutex mu;
  static NcclFns f;
  static int state = 0;  // 0 not tried, 1 loaded, -1 missing
  std::lock_guard<std::mutex> g(mu);
  if (state == 0) {
    state = -1;
    void* lib = dlopen("libnccl.so.2", RTLD_NOW | RTLD_LOCAL);
    if (lib) {
      f.get_unique_id = reinterpret_cast<decltype(f.get_unique_id)>(dlsym(lib, "ncclGetUniqueId"));
      f.init_rank = reinterpret_cast<decltype(f.init_rank)>(dlsym(lib, "ncclCommInitRank"));
      f.all_gather = reinterpret_cast<decltype(f.all_gather)>(dlsym(lib, "ncclAllGather"));
      f.all_reduce = reinterpret_cast<decltype(f.all_reduce)>(dlsym(lib, "ncclAllReduce"));
      f.destroy = reinterpret_cast<decltype(f.destroy)>(dlsym(lib, "ncclCommDestroy"));
      f.abort = reinterpret_cast<decltype(f.abort)>(dlsym(lib, "ncclCommAbort"));
      f.error_string =
          reinterpret_cast<decltype(f.error_string)>(dlsym(lib, "ncclGetErrorString"));
      if (f.get_unique_id && f.init_rank && f.all_gather && f.all_reduce && f.destroy && f.abort &&
          f.error_string)
        state = 1;
    }
  }
  if (state != 1)
    return set_error(LSQ_ERR_CUDA, "NCCL (libnccl.so.2) is not loadable or lacks an entry point");
  *out = &f;
  return LSQ_OK;
}

// This rank's slice of a layer of `bytes`: [off, off + len) of the blob.
void shard_slice(const lsq_stack* h, size_t bytes, size_t* off, size_t* len) {
  *off = (size_t)h->rank * h->shard;
  *len = *off < bytes ? std::min(h->shard, bytes - *off) : 0;
}

// Sharded fetch of `layer` into buffer b, on the copy stream: this rank's slice
// from host, then the in-place all-gather of every rank's slice.
int shard_fetch(lsq_stack* h, int b, int layer, size_t bytes) {
  const NcclFns* f = nullptr;
  LSQ_TRY(nccl_fns(&f));
  size_t off = 0, len = 0;
  shard_slice(h, bytes, &off, &len);
  uint8_t* dst = static_cast<uint8_t*>(h->buf[b]);
  if (len)
    LSQ_CUDA(cudaMemcpyAsync(dst + off, static_cast<const uint8_t*>(h->blobs[layer]) + off, len,
                             cudaMemcpyHostToDevice, h->copy_stream));
  const ncclResult_t r = f->all_gather(dst + off, dst, h->shard, ncclUint8,
                                       static_cast<ncclComm_t>(h->comm), h->copy_stream);
  if (r != ncclSuccess)
    return set_error(LSQ_ERR_CUDA, "ncclAllGather: %s", f->error_string(r));
  return LSQ_OK;
}

// After a step timed out: abort the communicators, which ends any all-gather
// or all-reduce still waiting for a peer, and refuse further steps on this stack.
void shard_abort(lsq_stack* h) {
  const NcclFns* f = nullptr;
  if (nccl_fns(&f) == LSQ_OK) {
    if (h->comm) f->abort(static_cast<ncclComm_t>(h->comm));
    if (h->grad_comm) f->abort(static_cast<ncclComm_t>(h->grad_comm));
  }
  h->comm = nullptr;
  h->grad_comm = nullptr;
  h->aborted = 1;
}

int wait_event_timeout(cudaEvent_t ev, int64_t timeout_ms) {
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return LSQ_OK;
    if (e != cudaErrorNotReady) return cuda_status(e, "cudaEventQuery");
    const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(
                        std::chrono::steady_clock::now() - t0)
                        .count();
    if (timeout_ms >= 0 && ms > timeout_ms)
      return set_error(LSQ_ERR_TIMEOUT, "stream_stack_step: no completion after %lld ms",
                       (long long)timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

}  // namespace
}  // namespace lsq

using namespace lsq;

extern "C" size_t stream_stack_workspace_bytes(const lsq_cfg* cfg, int32_t batch, int32_t seq) {
  LayerShapes s;
  if (batch <= 0 || seq <= 0 || layer_shapes(cfg, &s) != LSQ_OK || cfg->n_layers <= 0 ||
      cfg->vocab <= 0)
    return 0;
  return plan_stack_ws(cfg, s, (int64_t)batch * seq, seq, nullptr, nullptr);
}

extern "C" int stream_stack_create(const lsq_cfg* cfg, const void* const* layer_blobs,
                                   int32_t n_layers, void* vram_buf0, void* vram_buf1,
                                   int32_t resident, lsq_stack** out) {
  if (!out) return set_error(LSQ_ERR_INVALID, "stream_stack_create: null output");
  *out = nullptr;
  LayerShapes s;
  LSQ_TRY(layer_shapes(cfg, &s));
  if (n_layers != cfg->n_layers || n_layers <= 0)
    return set_error(LSQ_ERR_SHAPE, "stream_stack_create: n_layers %d != cfg.n_layers %d", n_layers,
                     cfg->n_layers);
  if (cfg->vocab <= 0 || cfg->vocab % 8 != 0)
    return set_error(LSQ_ERR_SHAPE, "stream_stack_create: vocab must be a positive multiple of 8");
  if (!layer_blobs) return set_error(LSQ_ERR_INVALID, "stream_stack_create: null layer list");
  for (int i = 0; i < n_layers; ++i)
    if (!layer_blobs[i] || !aligned16(layer_blobs[i]))
      return set_error(LSQ_ERR_INVALID, "stream_stack_create: layer %d blob null or unaligned", i);
  if (resident != 0 && resident != 1) return set_error(LSQ_ERR_INVALID, "resident must be 0 or 1");
  if (!resident && (!vram_buf0 || !vram_buf1 || !aligned16(vram_buf0) || !aligned16(vram_buf1)))
    return set_error(LSQ_ERR_INVALID, "stream_stack_create: two aligned VRAM buffers are needed");
  if (!resident) {
    for (int i = 0; i < n_layers; ++i) {
      cudaPointerAttributes at;
      if (cudaPointerGetAttributes(&at, layer_blobs[i]) != cudaSuccess ||
          at.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return set_error(LSQ_ERR_INVALID,
                         "stream_stack_create: layer %d blob is not page-locked host memory", i);
      }
    }
  }
  lsq_stack* h = new lsq_stack();
  h->cfg = *cfg;
  h->shapes = s;
  lsq_layer_layout_get(cfg, &h->layout);
  lsq_lora_layout_get(cfg, &h->lora_layout);
  h->blobs.assign(layer_blobs, layer_blobs + n_layers);
  h->buf[0] = vram_buf0;
  h->buf[1] = vram_buf1;
  h->resident = resident;
  h->buf_layer[0] = h->buf_layer[1] = -1;
  h->n_waits_last = 0;
  h->stats = lsq_step_stats{};
  cudaGetDevice(&h->device);
  int rc = LSQ_OK;
  if (cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    rc = set_error(LSQ_ERR_CUDA, "stream_stack_create: cannot create streams");
  for (int i = 0; rc == LSQ_OK && i < 2; ++i)
    if (cudaEventCreateWithFlags(&h->ready[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->freed[i], cudaEventDisableTiming) != cudaSuccess)
      rc = set_error(LSQ_ERR_CUDA, "stream_stack_create: cannot create events");
  if (rc == LSQ_OK &&
      (cudaEventCreate(&h->t_start) != cudaSuccess || cudaEventCreate(&h->t_end) != cudaSuccess ||
       cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming) != cudaSuccess))
    rc = set_error(LSQ_ERR_CUDA, "stream_stack_create: cannot create events");
  if (rc == LSQ_OK && cudaMallocHost(&h->loss_host, (1 + 4 * kMaxPairs) * sizeof(float)) != cudaSuccess)
    rc = set_error(LSQ_ERR_CUDA, "stream_stack_create: cannot allocate the pinned loss slot");
  if (rc != LSQ_OK) {
    delete h;
    return rc;
  }
  *out = h;
  return LSQ_OK;
}

extern "C" int stream_stack_destroy(lsq_stack* h) {
  if (!h) return LSQ_OK;
  cudaStreamSynchronize(h->copy_stream);
  cudaStreamDestroy(h->copy_stream);
  drop_graphs(h);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  for (int i = 0; i < 2; ++i) {
    cudaEventDestroy(h->ready[i]);
    cudaEventDestroy(h->freed[i]);
  }
  for (auto e : h->wait_ev) cudaEventDestroy(e);
  cudaEventDestroy(h->t_start);
  cudaEventDestroy(h->t_end);
  cudaEventDestroy(h->done);
  cudaFreeHost(h->loss_host);
  const NcclFns* f = nullptr;
  if (h->comm && nccl_fns(&f) == LSQ_OK) f->destroy(static_cast<ncclComm_t>(h->comm));
  if (h->grad_comm && nccl_fns(&f) == LSQ_OK) f->destroy(static_cast<ncclComm_t>(h->grad_comm));
  if (h->red_stream) {
    cudaStreamSynchronize(h->red_stream);
    cudaStreamDestroy(h->red_stream);
  }
  if (h->red_ev) cudaEventDestroy(h->red_ev);
  if (h->red_done) cudaEventDestroy(h->red_done);
  delete h;
  return LSQ_OK;
}

extern "C" int stream_stack_last_stats(const lsq_stack* h, lsq_step_stats* out) {
  if (!h || !out) return set_error(LSQ_ERR_INVALID, "stream_stack_last_stats: null pointer");
  *out = h->stats;
  return LSQ_OK;
}

extern "C" int lsq_stream_plan(int32_t n_layers, int32_t micro_batches, int32_t held0,
                               int32_t held1, int32_t* layer, int32_t* buf, int32_t* copy,
                               int32_t max_visits, int32_t* n_visits) {
  if (!layer || !buf || !copy || !n_visits)
    return set_error(LSQ_ERR_INVALID, "lsq_stream_plan: null output");
  if (n_layers <= 0 || micro_batches <= 0 || held0 < -1 || held0 >= n_layers || held1 < -1 ||
      held1 >= n_layers || (held0 >= 0 && held0 == held1))
    return set_error(LSQ_ERR_SHAPE, "lsq_stream_plan: bad layer count or buffer contents");
  const int64_t n = (int64_t)2 * n_layers * micro_batches;
  if (n > max_visits)
    return set_error(LSQ_ERR_WORKSPACE, "lsq_stream_plan: %lld visits, room for %d",
                     (long long)n, max_visits);
  const std::vector<Visit> v = plan_visits(n_layers, micro_batches, held0, held1);
  for (size_t i = 0; i < v.size(); ++i) {
    layer[i] = v[i].layer;
    buf[i] = v[i].buf;
    copy[i] = v[i].copy;
  }
  *n_visits = (int32_t)v.size();
  return LSQ_OK;
}

extern "C" int64_t lsq_shard_bytes(int64_t layer_bytes, int32_t world) {
  if (layer_bytes <= 0 || world < 1) return 0;
  const int64_t s = (layer_bytes + world - 1) / world;
  return (s + 255) / 256 * 256;
}

extern "C" int lsq_nccl_unique_id(void* id_out, int64_t id_bytes) {
  if (!id_out || id_bytes != (int64_t)sizeof(ncclUniqueId))
    return set_error(LSQ_ERR_INVALID, "lsq_nccl_unique_id: need a %d-byte output",
                     (int)sizeof(ncclUniqueId));
  const NcclFns* f = nullptr;
  LSQ_TRY(nccl_fns(&f));
  ncclUniqueId id;
  const ncclResult_t r = f->get_unique_id(&id);
  if (r != ncclSuccess) return set_error(LSQ_ERR_CUDA, "ncclGetUniqueId: %s", f->error_string(r));
  memcpy(id_out, &id, sizeof(id));
  return LSQ_OK;
}

extern "C" int stream_stack_shard(lsq_stack* h, const void* nccl_id, int64_t id_bytes,
                                  int32_t world, int32_t rank, int64_t buf_bytes) {
  if (!h || !nccl_id) return set_error(LSQ_ERR_INVALID, "stream_stack_shard: null pointer");
  if (id_bytes != (int64_t)sizeof(ncclUniqueId))
    return set_error(LSQ_ERR_INVALID, "stream_stack_shard: the id has %d bytes",
                     (int)sizeof(ncclUniqueId));
  if (h->resident)
    return set_error(LSQ_ERR_INVALID, "stream_stack_shard: a resident stack copies no layers");
  if (h->shard || h->comm || h->aborted)
    return set_error(LSQ_ERR_INVALID, "stream_stack_shard: the stack is already sharded");
  if (world < 1 || rank < 0 || rank >= world)
    return set_error(LSQ_ERR_INVALID, "stream_stack_shard: rank %d of world %d", rank, world);
  const int64_t S = lsq_shard_bytes((int64_t)h->layout.bytes, world);
  if (buf_bytes < S * world)
    return set_error(LSQ_ERR_WORKSPACE,
                     "stream_stack_shard: layer buffers of %lld bytes, %lld needed (world x %lld)",
                     (long long)buf_bytes, (long long)(S * world), (long long)S);
  int dev = -1;
  LSQ_CUDA(cudaGetDevice(&dev));
  if (dev != h->device)
    return set_error(LSQ_ERR_INVALID, "stream_stack_shard: call on the stack's device (%d, not %d)",
                     h->device, dev);
  const NcclFns* f = nullptr;
  LSQ_TRY(nccl_fns(&f));
  ncclUniqueId id;
  memcpy(&id, nccl_id, sizeof(id));
  ncclComm_t comm = nullptr;
  const ncclResult_t r = f->init_rank(&comm, world, id, rank);
  if (r != ncclSuccess)
    return set_error(LSQ_ERR_CUDA, "ncclCommInitRank: %s", f->error_string(r));
  h->comm = comm;
  h->world = world;
  h->rank = rank;
  h->shard = (size_t)S;
  return LSQ_OK;
}

extern "C" int stream_stack_reduce_grads(lsq_stack* h, const void* nccl_id, int64_t id_bytes,
                                         int32_t world, int32_t rank) {
  if (!h || !nccl_id) return set_error(LSQ_ERR_INVALID, "stream_stack_reduce_grads: null pointer");
  if (id_bytes != (int64_t)sizeof(ncclUniqueId))
    return set_error(LSQ_ERR_INVALID, "stream_stack_reduce_grads: the id has %d bytes",
                     (int)sizeof(ncclUniqueId));
  if (h->grad_comm || h->aborted)
    return set_error(LSQ_ERR_INVALID,
                     "stream_stack_reduce_grads: gradients are already reduced, or the stack's "
                     "communicators were aborted");
  if (world < 1 || rank < 0 || rank >= world)
    return set_error(LSQ_ERR_INVALID, "stream_stack_reduce_grads: rank %d of world %d", rank,
                     world);
  int dev = -1;
  LSQ_CUDA(cudaGetDevice(&dev));
  if (dev != h->device)
    return set_error(LSQ_ERR_INVALID,
                     "stream_stack_reduce_grads: call on the stack's device (%d, not %d)",
                     h->device, dev);
  const NcclFns* f = nullptr;
  LSQ_TRY(nccl_fns(&f));
  if (!h->red_stream) {
    LSQ_CUDA(cudaStreamCreateWithFlags(&h->red_stream, cudaStreamNonBlocking));
    LSQ_CUDA(cudaEventCreateWithFlags(&h->red_ev, cudaEventDisableTiming));
    LSQ_CUDA(cudaEventCreateWithFlags(&h->red_done, cudaEventDisableTiming));
  }
  ncclUniqueId id;
  memcpy(&id, nccl_id, sizeof(id));
  ncclComm_t comm = nullptr;
  const ncclResult_t r = f->init_rank(&comm, world, id, rank);
  if (r != ncclSuccess)
    return set_error(LSQ_ERR_CUDA, "ncclCommInitRank: %s", f->error_string(r));
  h->grad_comm = comm;
  h->grad_world = world;
  return LSQ_OK;
}

namespace lsq {
namespace {

struct DpoArgs {
  int pairs;
  float beta;
  float* logps_out;  // host [4 * pairs] or null
};

// One optimiser step over the streamed stack: SFT (dpo == null) or DPO.  The
// DPO step runs the reference (adapter off) forward of each layer right after
// the policy forward, from the same resident layer buffer, so it reads the
// stack as often as an SFT step does.
int step_impl(lsq_stack* h, const int32_t* tokens, int32_t micro_batches, int32_t batch,
              int32_t seq, const uint16_t* emb, const uint16_t* lm_head,
              const uint16_t* final_norm, float* lora, float* lora_grad, const lsq_adamw* opt,
              float* loss_out, float* logits_out, void* ws, size_t ws_bytes, void* stream,
              int64_t timeout_ms, const DpoArgs* dpo) {
  if (!h) return set_error(LSQ_ERR_INVALID, "stream_stack_step: null handle");
  if (h->aborted)
    return set_error(LSQ_ERR_INVALID,
                     "stream_stack_step: the stack's communicator was aborted after a timeout");
  if (!tokens || !emb || !lm_head || !final_norm || !lora || !lora_grad || !loss_out)
    return set_error(LSQ_ERR_INVALID, "stream_stack_step: null pointer");
  if (micro_batches <= 0 || batch <= 0 || seq < 2)
    return set_error(LSQ_ERR_SHAPE, "stream_stack_step: need micro_batches, batch >= 1, seq >= 2");
  if (opt && (!opt->m || !opt->v || opt->step < 1))
    return set_error(LSQ_ERR_INVALID, "stream_stack_step: AdamW needs m, v and step >= 1");
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != h->device) return set_error(LSQ_ERR_INVALID, "stream_stack_step: wrong current device");
  const lsq_cfg* cfg = &h->cfg;
  const LayerShapes& s = h->shapes;
  const int L = cfg->n_layers;
  const int64_t T = (int64_t)batch * seq, D = s.D, V = cfg->vocab;
  const size_t need = plan_stack_ws(cfg, s, T, seq, nullptr, nullptr, dpo != nullptr);
  if (!ws || ws_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "stream_stack_step: workspace %zu < %zu", ws_bytes, need);
  StackWs w;
  plan_stack_ws(cfg, s, T, seq, ws, &w, dpo != nullptr);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int64_t layer_floats = h->lora_layout.floats_per_layer;
  const float inv_count = 1.f / (float)((double)micro_batches * batch * (seq - 1));

  // The buffers' contents are only trusted after a step that completed; a
  // failed step leaves them unknown.
  const int held0 = h->buf_layer[0], held1 = h->buf_layer[1];
  h->buf_layer[0] = h->buf_layer[1] = -1;
  std::vector<Visit> visits;
  if (!h->resident) visits = plan_visits(L, micro_batches, held0, held1);
  const size_t n_vis = (size_t)2 * L * micro_batches;
  while (h->wait_ev.size() < 2 * n_vis) {
    cudaEvent_t e;
    LSQ_CUDA(cudaEventCreate(&e));
    h->wait_ev.push_back(e);
  }
  const size_t bytes = h->layout.bytes;
  int copies = 0;
  auto enqueue_copy = [&](size_t j) -> int {
    const Visit& x = visits[j];
    if (!x.copy) return LSQ_OK;
    LSQ_CUDA(cudaStreamWaitEvent(h->copy_stream, h->freed[x.buf], 0));
    if (h->shard)
      LSQ_TRY(shard_fetch(h, x.buf, x.layer, bytes));
    else
      LSQ_CUDA(cudaMemcpyAsync(h->buf[x.buf], h->blobs[x.layer], bytes, cudaMemcpyHostToDevice,
                               h->copy_stream));
    LSQ_CUDA(cudaEventRecord(h->ready[x.buf], h->copy_stream));
    ++copies;
    return LSQ_OK;
  };
  // The layer visits run as replays of cached CUDA graphs.  A graph bakes in
  // every pointer its kernels get, so the cache is dropped whenever this step's
  // buffers, sizes or profiling state differ from the ones it was captured with.
  const bool profiling = prof_enabled();
  {
    const std::vector<uintptr_t> sig = {
        (uintptr_t)lora, (uintptr_t)lora_grad, (uintptr_t)ws, (uintptr_t)ws_bytes,
        (uintptr_t)batch, (uintptr_t)seq, (uintptr_t)micro_batches, (uintptr_t)profiling,
        (uintptr_t)(dpo != nullptr), (uintptr_t)w.head_T};  // (head_T moves the layer workspace)
    if (sig != h->graph_sig) {
      drop_graphs(h);
      h->graph_sig = sig;
    }
  }
  if (!device_status_ptr()) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  std::vector<const std::vector<ProfRec>*> replayed;  // profiled graphs launched in this step
  // Replays the graph of key k, capturing it first with enqueue(capture stream).
  auto visit = [&](std::tuple<int, int, int, int, int> k, auto&& enqueue) -> int {
    auto it = h->graphs.find(k);
    if (it == h->graphs.end()) {
      lsq_stack::GraphEntry e;
      LSQ_CUDA(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeRelaxed));
      if (profiling) prof_capture_sink(&e.recs);
      const int64_t n0 = launch_count();
      const int rc = enqueue(h->cap_stream);
      e.launches = launch_count() - n0;
      prof_capture_sink(nullptr);
      cudaGraph_t g = nullptr;
      cudaError_t ce = cudaStreamEndCapture(h->cap_stream, &g);
      if (rc == LSQ_OK && ce == cudaSuccess) ce = cudaGraphInstantiate(&e.exec, g, 0);
      if (g) cudaGraphDestroy(g);
      if (rc != LSQ_OK || ce != cudaSuccess) {
        prof_release(e.recs);
        cudaGetLastError();
        return rc != LSQ_OK ? rc : cuda_status(ce, "layer visit graph");
      }
      it = h->graphs.emplace(k, std::move(e)).first;
    } else {
      count_launches(it->second.launches);  // the graph's kernels run again
    }
    LSQ_CUDA(cudaGraphLaunch(it->second.exec, cs));
    if (profiling) replayed.push_back(&it->second.recs);
    return LSQ_OK;
  };

  // Returns the device pointer of visit j's layer, after fencing the compute stream.
  auto acquire = [&](size_t j, const void** blob) -> int {
    if (h->resident) return LSQ_OK;
    const Visit& x = visits[j];
    if (j + 1 < visits.size()) LSQ_TRY(enqueue_copy(j + 1));
    LSQ_CUDA(cudaEventRecord(h->wait_ev[2 * j], cs));
    LSQ_CUDA(cudaStreamWaitEvent(cs, h->ready[x.buf], 0));
    LSQ_CUDA(cudaEventRecord(h->wait_ev[2 * j + 1], cs));
    *blob = h->buf[x.buf];
    return LSQ_OK;
  };

  LSQ_CUDA(cudaEventRecord(h->t_start, cs));
  LSQ_TRY(launch_rope_table(seq, s.hd, cfg->rope_theta, w.rope_cs, cs));
  // the LoRA masters in their product types, for every layer (they change only at
  // the optimiser step, after the last visit)
  LSQ_TRY(prepare_lora16(cfg, lora, L, w.lora16, cs));
  const size_t l16 = lora16_elems_per_layer(cfg);
  // Sharded: the step's first all-gather waits for everything the caller put on
  // the compute stream before the step (e.g. a gradient all-reduce on another
  // communicator), so that collectives of the two never run interleaved.
  if (h->shard) LSQ_CUDA(cudaStreamWaitEvent(h->copy_stream, h->t_start, 0));
  if (!h->resident && !visits.empty()) LSQ_TRY(enqueue_copy(0));
  size_t j = 0;
  for (int mb = 0; mb < micro_batches; ++mb) {
    const int32_t* tok = tokens + (int64_t)mb * T;
    LSQ_TRY(launch_embedding(tok, T, emb, D, V, w.xs, cs));
    const int mbk = profiling ? mb : 0;  // profiled graphs are replayed once per step
    for (int i = 0; i < L; ++i, ++j) {
      const void* blob = h->blobs[i];
      if (!h->resident) LSQ_TRY(acquire(j, &blob));
      const int b = h->resident ? -1 : visits[j].buf;
      LSQ_TRY(visit(std::make_tuple(0, i, b, 0, mbk), [&](cudaStream_t s) {
        return layer_fwd_impl(cfg, blob, lora + (int64_t)i * layer_floats,
                              w.xs + (size_t)i * T * D, batch, seq, w.xs + (size_t)(i + 1) * T * D,
                              w.layer_ws, w.layer_ws_bytes, s, w.rope_cs, w.lora16 + i * l16,
                              w.saved_u + (size_t)i * w.saved_u_bytes);
      }));
      if (dpo)  // reference model: the same layer with its adapter off
        LSQ_TRY(visit(std::make_tuple(1, i, b, 0, mbk), [&](cudaStream_t s) {
          return layer_fwd_impl(cfg, blob, nullptr, i == 0 ? w.xs : w.xr[(i - 1) & 1], batch, seq,
                                w.xr[i & 1], w.layer_ws, w.layer_ws_bytes, s, w.rope_cs);
        }));
      if (!h->resident) LSQ_CUDA(cudaEventRecord(h->freed[visits[j].buf], cs));
    }
    const float* xL = w.xs + (size_t)L * T * D;
    if (dpo) {
      LSQ_TRY(launch_rmsnorm_fwd(w.xr[(L - 1) & 1], final_norm, T, D, cfg->rms_eps, w.hf, OUT_BF16,
                                 w.rstd_f, cs));
      LSQ_TRY(gemm_run(head_fwd(lm_head, V, D, w.hf, T, w.logits), w.gemm, w.gemm_bytes, cs));
      LSQ_TRY(launch_cross_entropy(w.logits, tok, T, seq, V, 0.f, nullptr, w.row_ref, cs));
    }
    LSQ_TRY(launch_rmsnorm_fwd(xL, final_norm, T, D, cfg->rms_eps, w.hf, OUT_BF16, w.rstd_f, cs));
    if (!dpo) {
      // lm_head, cross-entropy and the head's input gradient, a chunk of whole
      // sequences at a time, so that the [T, V] logits never exist at once
      const bool last_mb = mb == micro_batches - 1;
      for (int64_t c0 = 0; c0 < T; c0 += w.head_T) {
        const int64_t tc = std::min<int64_t>(w.head_T, T - c0);
        LSQ_TRY(gemm_run(head_fwd(lm_head, V, D, w.hf + c0 * D, tc, w.logits), w.gemm,
                         w.gemm_bytes, cs));
        if (logits_out && last_mb)
          LSQ_CUDA(cudaMemcpyAsync(logits_out + c0 * V, w.logits, (size_t)tc * V * sizeof(float),
                                   cudaMemcpyDeviceToDevice, cs));
        LSQ_TRY(launch_cross_entropy(w.logits, tok + c0, tc, seq, V, inv_count, w.dlogits,
                                     w.row_loss + c0, cs));
        LSQ_TRY(gemm_run(head_dx(lm_head, V, D, w.dlogits, tc, w.dhf + c0 * D), w.gemm,
                         w.gemm_bytes, cs));
      }
      LSQ_TRY(launch_sum_rows(w.row_loss, T, inv_count, mb > 0 ? 1 : 0, w.loss_dev, cs));
    } else {
      LSQ_TRY(gemm_run(head_fwd(lm_head, V, D, w.hf, T, w.logits), w.gemm, w.gemm_bytes, cs));
      LSQ_TRY(launch_cross_entropy(w.logits, tok, T, seq, V, 0.f, nullptr, w.row_loss, cs));
      LSQ_TRY(launch_dpo_loss(w.row_loss, w.row_ref, dpo->pairs, seq, dpo->beta, w.seq_scale,
                              w.logps, w.loss_dev, cs));
      LSQ_TRY(launch_cross_entropy(w.logits, tok, T, seq, V, 0.f, w.dlogits, w.row_loss, cs,
                                   w.seq_scale));
      LSQ_TRY(gemm_run(head_dx(lm_head, V, D, w.dlogits, T, w.dhf), w.gemm, w.gemm_bytes, cs));
      if (logits_out)
        LSQ_CUDA(cudaMemcpyAsync(logits_out, w.logits, (size_t)T * V * sizeof(float),
                                 cudaMemcpyDeviceToDevice, cs));
    }
    LSQ_TRY(launch_rmsnorm_bwd(w.dhf, xL, final_norm, w.rstd_f, nullptr, T, D, w.dh[0], w.dhb[0], cs));
    int cur = 0;
    for (int i = L - 1; i >= 0; --i, ++j) {
      const void* blob = h->blobs[i];
      if (!h->resident) LSQ_TRY(acquire(j, &blob));
      const int b = h->resident ? -1 : visits[j].buf;
      const int acc = mb > 0 ? 1 : 0;
      LSQ_TRY(visit(std::make_tuple(2, i, b, acc, mbk), [&](cudaStream_t s) {
        return layer_bwd_impl(cfg, blob, lora + (int64_t)i * layer_floats,
                              w.xs + (size_t)i * T * D, w.dh[cur], w.dhb[cur], batch, seq,
                              w.dh[1 - cur], w.dhb[1 - cur], lora_grad + (int64_t)i * layer_floats,
                              acc, w.layer_ws, w.layer_ws_bytes, s, w.rope_cs, w.lora16 + i * l16,
                              w.saved_u + (size_t)i * w.saved_u_bytes);
      }));
      if (!h->resident) LSQ_CUDA(cudaEventRecord(h->freed[visits[j].buf], cs));
      if (h->grad_comm && mb == micro_batches - 1) {
        // layer i's gradient is final: average it over the ranks on the reduction
        // stream while the backward of layer i - 1 runs
        const NcclFns* f = nullptr;
        LSQ_TRY(nccl_fns(&f));
        LSQ_CUDA(cudaEventRecord(h->red_ev, cs));
        LSQ_CUDA(cudaStreamWaitEvent(h->red_stream, h->red_ev, 0));
        float* g = lora_grad + (int64_t)i * layer_floats;
        const ncclResult_t r = f->all_reduce(g, g, (size_t)layer_floats, ncclFloat, ncclAvg,
                                             static_cast<ncclComm_t>(h->grad_comm), h->red_stream);
        if (r != ncclSuccess)
          return set_error(LSQ_ERR_CUDA, "ncclAllReduce: %s", f->error_string(r));
      }
      cur = 1 - cur;
    }
  }
  if (h->grad_comm) {  // the optimiser (and the step's end) waits for the last all-reduce
    LSQ_CUDA(cudaEventRecord(h->red_done, h->red_stream));
    LSQ_CUDA(cudaStreamWaitEvent(cs, h->red_done, 0));
  }
  if (opt)
    LSQ_TRY(launch_adamw(lora, lora_grad, opt->m, opt->v, layer_floats * L, opt->lr, opt->beta1,
                         opt->beta2, opt->eps, opt->weight_decay, opt->step, cs));
  LSQ_CUDA(cudaMemcpyAsync(h->loss_host, w.loss_dev, sizeof(float), cudaMemcpyDeviceToHost, cs));
  if (dpo)
    LSQ_CUDA(cudaMemcpyAsync(h->loss_host + 1, w.logps, 4 * dpo->pairs * sizeof(float),
                             cudaMemcpyDeviceToHost, cs));
  LSQ_CUDA(cudaEventRecord(h->t_end, cs));
  LSQ_CUDA(cudaEventRecord(h->done, cs));
  {
    const int rc = wait_event_timeout(h->done, timeout_ms);
    if (rc != LSQ_OK) {
      if (rc == LSQ_ERR_TIMEOUT && (h->comm || h->grad_comm)) shard_abort(h);
      return rc;
    }
  }
  for (const std::vector<ProfRec>* r : replayed) LSQ_TRY(prof_accumulate(*r));
  int flags = 0;
  int* st = device_status_ptr();
  if (st) {
    LSQ_CUDA(cudaMemcpy(&flags, st, sizeof(int), cudaMemcpyDeviceToHost));
    if (flags) return set_error(LSQ_ERR_DEVICE, "stream_stack_step: device status 0x%x", flags);
  }
  if (!h->resident) {
    int held[2] = {held0, held1};
    for (const Visit& x : visits)
      if (x.copy) held[x.buf] = x.layer;
    h->buf_layer[0] = held[0];
    h->buf_layer[1] = held[1];
  }
  *loss_out = *h->loss_host;
  if (dpo && dpo->logps_out)
    for (int k = 0; k < 4 * dpo->pairs; ++k) dpo->logps_out[k] = h->loss_host[1 + k];
  h->stats.layer_copies = copies;
  size_t fetched = bytes;
  if (h->shard) {
    size_t off = 0;
    shard_slice(h, bytes, &off, &fetched);
  }
  h->stats.h2d_bytes = (int64_t)copies * (int64_t)fetched;
  cudaEventElapsedTime(&h->stats.step_ms, h->t_start, h->t_end);
  float wait_ms = 0.f;
  if (!h->resident) {
    for (size_t k = 0; k < visits.size(); ++k) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, h->wait_ev[2 * k], h->wait_ev[2 * k + 1]) == cudaSuccess)
        wait_ms += ms;
    }
  }
  h->stats.copy_wait_ms = wait_ms;
  return LSQ_OK;
}

}  // namespace
}  // namespace lsq

extern "C" int stream_stack_step(lsq_stack* h, const int32_t* tokens, int32_t micro_batches,
                                 int32_t batch, int32_t seq, const uint16_t* emb,
                                 const uint16_t* lm_head, const uint16_t* final_norm, float* lora,
                                 float* lora_grad, const lsq_adamw* opt, float* loss_out,
                                 float* logits_out, void* ws, size_t ws_bytes, void* stream,
                                 int64_t timeout_ms) {
  return step_impl(h, tokens, micro_batches, batch, seq, emb, lm_head, final_norm, lora, lora_grad,
                   opt, loss_out, logits_out, ws, ws_bytes, stream, timeout_ms, nullptr);
}

extern "C" size_t stream_stack_dpo_workspace_bytes(const lsq_cfg* cfg, int32_t pairs, int32_t seq) {
  LayerShapes s;
  if (pairs <= 0 || pairs > kMaxPairs || seq <= 0 || layer_shapes(cfg, &s) != LSQ_OK ||
      cfg->n_layers <= 0 || cfg->vocab <= 0)
    return 0;
  return plan_stack_ws(cfg, s, (int64_t)2 * pairs * seq, seq, nullptr, nullptr, true);
}

extern "C" int stream_stack_dpo_step(lsq_stack* h, const int32_t* tokens, int32_t pairs,
                                     int32_t seq, float beta, const uint16_t* emb,
                                     const uint16_t* lm_head, const uint16_t* final_norm,
                                     float* lora, float* lora_grad, const lsq_adamw* opt,
                                     float* loss_out, float* logps_out, float* logits_out,
                                     void* ws, size_t ws_bytes, void* stream, int64_t timeout_ms) {
  if (pairs <= 0 || pairs > kMaxPairs)
    return set_error(LSQ_ERR_SHAPE, "stream_stack_dpo_step: pairs must be 1..%d", kMaxPairs);
  if (!(beta > 0.f) || !std::isfinite(beta))
    return set_error(LSQ_ERR_INVALID, "stream_stack_dpo_step: beta must be positive and finite");
  DpoArgs d{pairs, beta, logps_out};
  return step_impl(h, tokens, 1, 2 * pairs, seq, emb, lm_head, final_norm, lora, lora_grad, opt,
                   loss_out, logits_out, ws, ws_bytes, stream, timeout_ms, &d);
}

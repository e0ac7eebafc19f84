// C ABI: error reporting, device status, and the single NF4 + LoRA linear.
//
// y = x W~^T + s (x A^T) B^T and its backward dX = dY W~ + s (dY B) A,
// dA = s (dY B)^T x, dB = s dY^T (x A^T) (Soup layer-streaming tutorial,
// "四段資料路徑" parts 1 and 3, FAQ 4).  The forward takes fp16 activations (the
// fused GEMM's forward operand type) and writes fp16, or fp32 with an fp32
// residual; the backward takes bf16 gradients.
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace lsq {

static thread_local char t_msg[512] = "";

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return LSQ_OK;
  return set_error(LSQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

namespace {

struct LinearWs {
  float* u;       // u = x A^T, fp32 (the forward's optional output)
  uint16_t* u16;  // bf16 copies of u, v for the dA / dB products ([r][lora16_ld(T)])
  uint16_t* v16;
  uint16_t* uh;   // the GEMMs' LoRA slab operands: u in fp16 [T][r], v in bf16 [T][r],
  uint16_t* vh;   //   s B in fp16 [N][r], s A^T in bf16 [K][r]
  uint16_t* sb;
  uint16_t* sat;
  float* scratch;
  size_t scratch_bytes;
  void* gemm;
  size_t gemm_bytes;
};

GemmDesc fwd_desc(const uint16_t* x, int64_t T, int64_t K, int64_t N, const uint8_t* codes,
                  const float* absmax, const uint16_t* sb, int r, const uint16_t* uh,
                  const float* residual, void* y, int y_f32) {
  GemmDesc d;
  d.wmode = W_NF4_N;
  d.M = N;
  d.T = T;
  d.Kc = K;
  d.w = codes;
  d.absmax = absmax;
  d.w_rows = N;
  d.w_cols = K;
  d.act = x;
  d.act_ld = K;
  d.slab_w = r;
  d.la16 = sb;
  d.la16_ld = r;
  d.lb16 = uh;
  d.lb16_ld = r;
  d.out = y;
  d.out_f32 = y_f32;
  d.ldo = N;
  d.residual = residual;
  d.ldr = N;
  return d;
}

GemmDesc bwd_desc(const uint16_t* dy, int64_t T, int64_t K, int64_t N, const uint8_t* codes,
                  const float* absmax, const uint16_t* sat, int r, const uint16_t* vh,
                  uint16_t* dx) {
  GemmDesc d;
  d.wmode = W_NF4_T;
  d.M = K;
  d.T = T;
  d.Kc = N;
  d.w = codes;
  d.absmax = absmax;
  d.w_rows = N;
  d.w_cols = K;
  d.act = dy;
  d.act_ld = N;
  d.slab_w = r;
  d.la16 = sat;
  d.la16_ld = r;
  d.lb16 = vh;
  d.lb16_ld = r;
  d.out = dx;
  d.ldo = K;
  return d;
}

size_t linear_ws_plan(int64_t T, int64_t K, int64_t N, int r, LinearWs* w, void* base) {
  const size_t sb = std::max(lora_scratch_bytes(T, K, r), lora_scratch_bytes(T, N, r));
  const size_t gb = std::max(
      gemm_workspace_bytes(fwd_desc(nullptr, T, K, N, nullptr, nullptr, nullptr, r, nullptr,
                                    nullptr, nullptr, 0)),
      gemm_workspace_bytes(bwd_desc(nullptr, T, K, N, nullptr, nullptr, nullptr, r, nullptr,
                                    nullptr)));
  Arena b;
  b.base = static_cast<uint8_t*>(base);
  b.cap = SIZE_MAX;
  float* u = b.take<float>((size_t)T * r);
  uint16_t* u16 = b.take<uint16_t>((size_t)lora16_ld(T) * r);  // [r][lora16_ld(T)]
  uint16_t* v16 = b.take<uint16_t>((size_t)lora16_ld(T) * r);
  uint16_t* uh = b.take<uint16_t>((size_t)T * r);
  uint16_t* vh = b.take<uint16_t>((size_t)T * r);
  uint16_t* sbm = b.take<uint16_t>((size_t)N * r);
  uint16_t* sat = b.take<uint16_t>((size_t)K * r);
  float* s = b.take<float>(sb / sizeof(float) + 1);
  void* g = b.take<uint8_t>(gb + 256);
  if (w) {
    w->u = base ? u : nullptr;
    w->u16 = base ? u16 : nullptr;
    w->v16 = base ? v16 : nullptr;
    w->uh = base ? uh : nullptr;
    w->vh = base ? vh : nullptr;
    w->sb = base ? sbm : nullptr;
    w->sat = base ? sat : nullptr;
    w->scratch = base ? s : nullptr;
    w->scratch_bytes = sb;
    w->gemm = base ? g : nullptr;
    w->gemm_bytes = gb + 256;
  }
  return b.used;
}

// The slab operand s B (fp16 [N][r], kind 2) or s A^T (bf16 [K][r] from A [r][K],
// kind 3) of one linear, rounded from the caller's fp32 matrix.
int prepare_slab(const float* src, int kind, int64_t rows, int r, float scale, uint16_t* out,
                 cudaStream_t st) {
  LoraPrepSegs g{};
  LoraPrepSeg& e = g.seg[0];
  e.kind = kind;
  e.src_off = 0;
  e.dst_off = 0;
  e.rows = rows;
  e.cols = r;
  e.ld_out = r;
  e.n_parts = 1;
  e.part_end[0] = rows;
  e.scale = scale;
  g.n = 1;
  return launch_lora_prepare(src, 0, 1, out, 0, g, st);
}

int check_linear(const void* x, int64_t T, int64_t K, int64_t N, const void* codes,
                 const void* absmax, int32_t block, const void* A, const void* B, int32_t r,
                 const char* who) {
  if (!x || !codes || !absmax || !A || !B) return set_error(LSQ_ERR_INVALID, "%s: null input", who);
  if (block != 64) return set_error(LSQ_ERR_SHAPE, "%s: block must be 64", who);
  if (T <= 0 || K <= 0 || N <= 0) return set_error(LSQ_ERR_SHAPE, "%s: empty shape", who);
  if (K % 64 != 0) return set_error(LSQ_ERR_SHAPE, "%s: K %% 64 != 0", who);
  if (N % 8 != 0) return set_error(LSQ_ERR_SHAPE, "%s: N %% 8 != 0", who);
  if (r <= 0 || r % 16 != 0 || r > 256)
    return set_error(LSQ_ERR_SHAPE, "%s: r must be a positive multiple of 16 (<= 256)", who);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(absmax) || !aligned16(A) || !aligned16(B))
    return set_error(LSQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned", who);
  return LSQ_OK;
}

}  // namespace
}  // namespace lsq

using namespace lsq;

extern "C" const char* lsq_last_error(void) { return t_msg; }
extern "C" int lsq_version(void) { return 201; }

extern "C" int lsq_device_status(int* flags, int clear) {
  if (!flags) return set_error(LSQ_ERR_INVALID, "lsq_device_status: null output");
  int* p = device_status_ptr();
  if (!p) return set_error(LSQ_ERR_CUDA, "lsq_device_status: no device status word");
  LSQ_CUDA(cudaDeviceSynchronize());
  LSQ_CUDA(cudaMemcpy(flags, p, sizeof(int), cudaMemcpyDeviceToHost));
  if (clear) LSQ_CUDA(cudaMemset(p, 0, sizeof(int)));
  return LSQ_OK;
}

extern "C" size_t nf4_lora_linear_workspace_bytes(int64_t T, int64_t K, int64_t N, int32_t r) {
  if (T <= 0 || K <= 0 || N <= 0 || r <= 0) return 0;
  return linear_ws_plan(T, K, N, r, nullptr, nullptr);
}

extern "C" int nf4_lora_linear_fwd(const uint16_t* x, int64_t T, int64_t K, int64_t N,
                                   const uint8_t* codes, const float* absmax, int32_t block,
                                   const float* A, const float* B, int32_t r, float scale,
                                   const float* residual, void* y, int32_t y_fp32, float* u_out,
                                   void* ws, size_t ws_bytes, void* stream) {
  LSQ_TRY(check_linear(x, T, K, N, codes, absmax, block, A, B, r, "nf4_lora_linear_fwd"));
  if (!y) return set_error(LSQ_ERR_INVALID, "nf4_lora_linear_fwd: null output");
  if (y_fp32 != 0 && y_fp32 != 1)
    return set_error(LSQ_ERR_INVALID, "nf4_lora_linear_fwd: y_fp32 must be 0 or 1");
  if (residual && !y_fp32)
    return set_error(LSQ_ERR_INVALID, "nf4_lora_linear_fwd: a residual needs an fp32 output");
  if (!aligned16(y) || (residual && !aligned16(residual)) || (u_out && !aligned16(u_out)))
    return set_error(LSQ_ERR_ALIGN, "nf4_lora_linear_fwd: pointers must be 16-byte aligned");
  const size_t need = linear_ws_plan(T, K, N, r, nullptr, nullptr);
  if (!ws || ws_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "nf4_lora_linear_fwd: workspace %zu < %zu", ws_bytes, need);
  LinearWs w;
  linear_ws_plan(T, K, N, r, &w, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* u = u_out ? u_out : w.u;
  LSQ_TRY(launch_lora_down(x, K, A, T, K, r, u, nullptr, w.scratch, w.scratch_bytes, st, w.uh));
  LSQ_TRY(prepare_slab(B, 2, N, r, scale, w.sb, st));
  GemmDesc d = fwd_desc(x, T, K, N, codes, absmax, w.sb, r, w.uh, residual, y, y_fp32);
  return gemm_run(d, w.gemm, w.gemm_bytes, st);
}

extern "C" int nf4_lora_linear_bwd(const uint16_t* dy, const uint16_t* x, int64_t T, int64_t K,
                                   int64_t N, const uint8_t* codes, const float* absmax,
                                   int32_t block, const float* A, const float* B, int32_t r,
                                   float scale, uint16_t* dx, float* dA, float* dB,
                                   int32_t accumulate, void* ws, size_t ws_bytes, void* stream) {
  LSQ_TRY(check_linear(x, T, K, N, codes, absmax, block, A, B, r, "nf4_lora_linear_bwd"));
  if (!dy || !dx || !dA || !dB) return set_error(LSQ_ERR_INVALID, "nf4_lora_linear_bwd: null pointer");
  const size_t need = linear_ws_plan(T, K, N, r, nullptr, nullptr);
  if (!ws || ws_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "nf4_lora_linear_bwd: workspace %zu < %zu", ws_bytes, need);
  LinearWs w;
  linear_ws_plan(T, K, N, r, &w, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t pe[1] = {N};
  LSQ_TRY(launch_lora_down(x, K, A, T, K, r, nullptr, w.u16, w.scratch, w.scratch_bytes, st));
  LSQ_TRY(launch_lora_vproj(dy, T, N, B, r, nullptr, w.v16, w.scratch, w.scratch_bytes, st, w.vh));
  LSQ_TRY(prepare_slab(A, 3, K, r, scale, w.sat, st));
  GemmDesc d = bwd_desc(dy, T, K, N, codes, absmax, w.sat, r, w.vh, dx);
  LSQ_TRY(gemm_run(d, w.gemm, w.gemm_bytes, st));
  return launch_lora_grad_ab16(w.v16, x, K, dA, dy, w.u16, N, r, 1, pe, T, scale, accumulate, dB,
                               st);
}

// Internal (non-ABI) declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <vector>

#include "../../include/lsq.h"

namespace lsq {

// ---------------------------------------------------------------- errors
int set_error(int code, const char* fmt, ...);   // records a message, returns code
int cuda_status(cudaError_t e, const char* what); // LSQ_OK or LSQ_ERR_CUDA with message
#define LSQ_TRY(expr)            \
  do {                           \
    int _rc = (expr);            \
    if (_rc != LSQ_OK) return _rc; \
  } while (0)
#define LSQ_CUDA(expr) LSQ_TRY(::lsq::cuda_status((expr), #expr))

// Counts a kernel launch (wraps the cudaGetLastError check after every launch).
cudaError_t launched(cudaError_t e);
// Launches issued so far, and n more (the kernels of a replayed CUDA graph).
int64_t launch_count();
void count_launches(int64_t n);
// Per-launch event timing of heavy kernels (no-ops unless lsq_profile_enable).
int prof_begin(cudaStream_t st);
void prof_end(int token, cudaStream_t st, const char* name, double flops, double bytes);
bool prof_enabled();
// A region recorded inside a captured CUDA graph: its events belong to the graph
// and are re-recorded at every replay.
struct ProfRec {
  int cls;
  cudaEvent_t e0, e1;
  double flops, bytes;
};
// While a sink is set on the calling thread (during a stream capture),
// prof_begin/prof_end record into fresh events and append the region to *sink.
void prof_capture_sink(std::vector<ProfRec>* sink);
// After a replay of a graph has completed: adds its regions' event times to the
// profile (a no-op unless profiling is enabled).
int prof_accumulate(const std::vector<ProfRec>& recs);
// Destroys the regions' events.
void prof_release(std::vector<ProfRec>& recs);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device status word bits (latched by kernels, read by lsq_device_status).
enum { DEV_ERR_WAIT_GEMM = 1, DEV_ERR_NONFINITE = 2 };
int* device_status_ptr();  // device address of the status word (current device)

// NF4 levels and fp32 decision midpoints, derived on the host from the
// definition of the data type (see nf4_quant.cu).
const float* nf4_levels();     // 16
const float* nf4_midpoints();  // 15

// ---------------------------------------------------------------- workspace
// Bump allocator over a caller-provided device workspace (256-B granules).
struct Arena {
  uint8_t* base = nullptr;
  size_t cap = 0, used = 0;
  bool overflow = false;
  template <class T>
  T* take(size_t n) {
    size_t bytes = (n * sizeof(T) + 255) & ~size_t(255);
    if (used + bytes > cap) {
      overflow = true;
      used += bytes;
      return nullptr;
    }
    T* p = reinterpret_cast<T*>(base + used);
    used += bytes;
    return p;
  }
};

// ---------------------------------------------------------------- tensor-core GEMM
// out[t, m] = sum_c Wop[m, c] * act[t, c] + sum_j la[m, j] * lb[t, j]  (+ residual[t, m])
// Wop is produced per tile by the operand stage:
//   W_NF4_N : Wop[m, c] = deq(W)[m, c]   (W [w_rows = M, w_cols = Kc] NF4; forward)
//   W_NF4_T : Wop[m, c] = deq(W)[c, m]   (W [w_rows = Kc, w_cols = M] NF4; dX)
//   W_BF16_N: Wop[m, c] = W[m, c]        (W bf16 [M, Kc])
//   W_BF16_T: Wop[m, c] = W[c, m]        (W bf16 [Kc, M])
//   W_BF16C_N: Wop[m, c] = W[m, c]       (W bf16 [M, Kc], converted to an fp16 operand)
// Operand precision: the forward modes of the decoder layer (W_NF4_N, W_BF16C_N)
// multiply fp16 operands (the weight rounded to fp16, fp16 activations and LoRA
// slab) and write fp16 (or fp32) outputs; the input-gradient modes (W_NF4_T,
// W_BF16_T) and the lm_head forward (W_BF16_N) multiply bf16 operands and write
// bf16 (or fp32).  Accumulation is fp32 in every mode.
enum WMode { W_NF4_N = 0, W_NF4_T = 1, W_BF16_N = 2, W_BF16_T = 3, W_BF16C_N = 4 };
__host__ __device__ constexpr bool wmode_f16(int m) { return m == W_NF4_N || m == W_BF16C_N; }

struct GemmDesc {
  int wmode = W_NF4_N;
  int64_t M = 0, T = 0, Kc = 0;
  const void* w = nullptr;          // NF4 codes or bf16 weight
  const float* absmax = nullptr;    // NF4 only: fp32 absmax per 64-block, or
  const uint8_t* absmax_q = nullptr;  // 8-bit absmax (double quantised) with
  const float* absmax_s = nullptr;    // one fp32 scale per 256 blocks
  int64_t w_rows = 0, w_cols = 0;   // storage shape of W
  const uint16_t* act = nullptr;    // bf16 [T, act_ld], contraction over the first Kc columns
  int64_t act_ld = 0;
  // LoRA slab: an extra K range of slab_w columns appended to split 0, with
  // operands la16 and lb16 below (for a stacked weight, la16's rows hold only their
  // own part's columns, zeros elsewhere, so that every row uses the same lb16, as a
  // CTA pair's shared B operand requires)
  int slab_w = 0;
  // epilogue: out is fp32 when out_f32, else 16-bit in the mode's operand type;
  // residual (fp32 [T, ldr], added before the store) needs an fp32 output
  void* out = nullptr;
  int out_f32 = 0;
  int64_t ldo = 0;
  const float* residual = nullptr;
  int64_t ldr = 0;
  int force_splits = 0;             // 0 = heuristic
  const char* prof_name = nullptr;  // profiler class (default: by operand mode)
  // Partials left to the next kernel: with parts_out set, a product split over K
  // skips its reduce and reports the fp32 partials ([splits][T][M], in the
  // workspace, valid until the next GEMM on it) and their count; an unsplit
  // product writes out as usual and reports 1.  The residual is then the
  // consumer's to add.
  const float** parts_out = nullptr;
  int* splits_out = nullptr;
  // The LoRA slab's operands, loaded by TMA: la16 [M][la16_ld] (the scale applied)
  // and lb16 [T][lb16_ld], slab_w columns of each, in the mode's operand type (fp16
  // forward, bf16 input gradient).
  const uint16_t* la16 = nullptr;
  int64_t la16_ld = 0;
  const uint16_t* lb16 = nullptr;
  int64_t lb16_ld = 0;
};
size_t gemm_workspace_bytes(const GemmDesc& d);
int gemm_run(const GemmDesc& d, void* ws, size_t ws_bytes, cudaStream_t st);
int gemm_num_sms();

// ---------------------------------------------------------------- small kernels
// Output kinds of a reduce or normalisation kernel.
enum OutKind { OUT_BF16 = 0, OUT_F32 = 1, OUT_F16 = 2 };
// Kernels that take a split product's partials (n_parts slices T * width apart,
// summed in slice order, then the residual, as launch_splitk_reduce would):
//   launch_rmsnorm_fwd_sum: x_out = sum + res (fp32), y = RMSNorm(x_out), rstd;
//   launch_rmsnorm_bwd_sum: launch_rmsnorm_bwd with dy = the sum;
//   launch_reduce_rope: qkv (fp16) = the sum rounded to fp16, q and k heads rotated.
int launch_rmsnorm_fwd_sum(const float* parts, int n_parts, const float* res, int64_t T,
                           int64_t D, float* x_out, const uint16_t* g, float eps, uint16_t* y,
                           int y_kind, float* rstd, cudaStream_t st);
int launch_rmsnorm_bwd_sum(const float* parts, int n_parts, const float* x, const uint16_t* g,
                           const float* rstd, const float* dres, int64_t T, int64_t D, float* dx,
                           uint16_t* dx_bf16, cudaStream_t st);
int launch_reduce_rope(const float* parts, int n_parts, int64_t T, int seq, int H, int Hkv, int d,
                       const float2* cs, uint16_t* qkv, cudaStream_t st);
int launch_splitk_reduce(const float* partial, int splits, int64_t T, int64_t M, void* out,
                         int out_kind, int64_t ldo, const float* residual, int64_t ldr,
                         cudaStream_t st);
// y = x (mean(x^2) + eps)^-1/2 g; x fp32 (the residual stream), y fp16 (OUT_F16,
// a forward GEMM operand) or bf16 (OUT_BF16, the lm_head operand)
int launch_rmsnorm_fwd(const float* x, const uint16_t* g, int64_t T, int64_t D, float eps,
                       uint16_t* y, int y_kind, float* rstd, cudaStream_t st);
// dx = dres + rmsnorm_bwd(dy);  writes fp32 dx and (optionally) its bf16 copy
int launch_rmsnorm_bwd(const float* dy, const float* x, const uint16_t* g, const float* rstd,
                       const float* dres, int64_t T, int64_t D, float* dx, uint16_t* dx_bf16,
                       cudaStream_t st);
// cos/sin table [seq][d/2] for rotate-half RoPE
int launch_rope_table(int seq, int d, float theta, float2* cs, cudaStream_t st);
// in place on the fp16 q and k heads of the fused qkv buffer
int launch_rope(uint16_t* qkv, int64_t T, int seq, int H, int Hkv, int d, const float2* cs,
                cudaStream_t st);
// dk, dv are per query head [T, H d] (summed over each kv group here)
int launch_rope_grad(const float* dq, const float* dk, const float* dv, int64_t T, int seq, int H,
                     int Hkv, int d, const float2* cs, uint16_t* dqkv, cudaStream_t st);
// m = silu(gate) * up: gu fp16 [T, 2F] -> m fp16 [T, F]; backward: dgu bf16
int launch_swiglu_fwd(const uint16_t* gu, int64_t T, int64_t F, uint16_t* m, cudaStream_t st);
int launch_swiglu_bwd(const float* dm, const uint16_t* gu, int64_t T, int64_t F, uint16_t* dgu,
                      cudaStream_t st);
// out fp32 [T, D] = emb (bf16) rows of the tokens
int launch_embedding(const int32_t* tokens, int64_t T, const uint16_t* emb, int64_t D,
                     int64_t V, float* out, cudaStream_t st);
// dlogits may be null (row losses only); seq_scale (per sequence) replaces inv_count.
int launch_cross_entropy(const float* logits, const int32_t* tokens, int64_t T, int seq,
                         int64_t V, float inv_count, uint16_t* dlogits, float* row_loss,
                         cudaStream_t st, const float* seq_scale = nullptr);
int launch_dpo_loss(const float* row_pol, const float* row_ref, int pairs, int seq, float beta,
                    float* seq_scale, float* logps, float* loss_out, cudaStream_t st);
int launch_sum_rows(const float* row_loss, int64_t T, float scale, int accumulate, float* out,
                    cudaStream_t st);
int launch_adamw(float* p, const float* g, float* m, float* v, int64_t n, float lr, float b1,
                 float b2, float eps, float wd, int step, cudaStream_t st);
int launch_f32_to_bf16(const float* x, int64_t n, uint16_t* y, cudaStream_t st);

// LoRA rank-r products (tcgen05 tensor cores, fp32 accumulation, fixed-order
// reductions).  Operands in their product types: u = x A^T multiplies fp16 (x an
// fp16 forward activation, A rounded to fp16); v, dA, dB multiply bf16 (each has a
// gradient operand).  Widths R are multiples of 8.  The products that
// feed another write its operand too, rounded to bf16 and transposed: u16, v16
// [R][lora16_ld(T)].
// scratch: lora_scratch_bytes(T, K, R) bytes for the fixed-order partials of a
// product split along its reduction (and, in the fp32-operand forms, the 16-bit
// copy of the LoRA operand).
int64_t lora16_ld(int64_t T);  // row stride of u16 / v16: T rounded up to 8
size_t lora_scratch_bytes(int64_t T, int64_t K, int R);
// u[t, j] = sum_k x[t, k] A[j, k]        x fp16 [T, ldx], A16 fp16 [R, K] -> u fp32 [T, R]
// (u may be null), and uh (nullable) the same rounded to fp16, [T, R]: the fused
// GEMM's LoRA slab operand
int launch_lora_down16(const uint16_t* x, int64_t ldx, const uint16_t* A16, int64_t T, int64_t K,
                       int R, float* u, uint16_t* u16, float* scratch, size_t scratch_bytes,
                       cudaStream_t st, uint16_t* uh = nullptr);
// v[t, c] = sum_n dy[t, n] Bt[c, n]      dy bf16 [T, N], Bt bf16 [R, N]: the block-diagonal
// stack of the parts' B transposed (column n of part p holds B_p's row n in rows
// [p r, (p + 1) r), zeros elsewhere)
// (v may be null; vh, nullable: the same rounded to bf16, [T, R], the slab operand)
int launch_lora_vproj16(const uint16_t* dy, int64_t T, int64_t N, const uint16_t* Bs, int R,
                        float* v, uint16_t* v16, float* scratch, size_t scratch_bytes,
                        cudaStream_t st, uint16_t* vh = nullptr);
// Both of a projection group's trainable gradients in one launch, R = n_parts r:
//   dA[j, k] (+)= s sum_t v[t, j] x[t, k]        v16 bf16 [R, lora16_ld(T)], x fp16 [T, K]
//                                                (converted to bf16 as it is loaded);
//   dB[n, j] (+)= s sum_t dy[t, n] u[t, part(n) r + j]   dy bf16 [T, N], u16 bf16
//                                                [R, lora16_ld(T)], the rows of dB split into
//                                                parts ending at part_end[].
int launch_lora_grad_ab16(const uint16_t* v16, const uint16_t* x, int64_t K, float* dA,
                          const uint16_t* dy, const uint16_t* u16, int64_t N, int r, int n_parts,
                          const int64_t* part_end, int64_t T, float s, int accumulate, float* dB,
                          cudaStream_t st);
// fp32-operand forms for a single linear (one part): the LoRA operand is rounded
// once into the scratch first
int launch_lora_down(const uint16_t* x, int64_t ldx, const float* A, int64_t T, int64_t K, int R,
                     float* u, uint16_t* u16, float* scratch, size_t scratch_bytes,
                     cudaStream_t st, uint16_t* uh = nullptr);
int launch_lora_vproj(const uint16_t* dy, int64_t T, int64_t N, const float* B, int r, float* v,
                      uint16_t* v16, float* scratch, size_t scratch_bytes, cudaStream_t st,
                      uint16_t* vh = nullptr);
// One layer's LoRA operands rounded once into their product types: a list of
// blocks, each
//   kind 0: an fp16 copy of an A matrix, [rows][cols];
//   kind 1: a bf16 block-diagonal stack of a B matrix, transposed ([ld_out][rows],
//           the rows split into parts ending at part_end[], part p's rows holding
//           B in rows [p cols, (p + 1) cols) of the stack);
//   kind 2: scale * the same stack untransposed, fp16 [rows][ld_out] (the forward
//           GEMM's LoRA slab);
//   kind 3: scale * A transposed, bf16 [rows][ld_out] from A [ld_out][rows] (the
//           input-gradient GEMM's LoRA slab).
// Offsets in elements within one layer's LoRA block / output.
struct LoraPrepSeg {
  int64_t src_off, dst_off, rows, cols, ld_out;
  int kind, n_parts;
  int64_t part_end[4];
  float scale;  // kinds 2 and 3
};
struct LoraPrepSegs {
  LoraPrepSeg seg[16];
  int n;
};
// Converts n_layers LoRA blocks (stride lora_stride floats) into out (stride
// out_stride elements per layer).
int launch_lora_prepare(const float* lora, int64_t lora_stride, int n_layers, uint16_t* out,
                        int64_t out_stride, const LoraPrepSegs& segs, cudaStream_t st);

// attention (causal GQA), q/k/v read from the fused fp16 qkv buffer [T, (H + 2 Hkv) d];
// o fp16 [T, H d]; dout bf16
int launch_attention_fwd(const uint16_t* qkv, int64_t T, int seq, int H, int Hkv, int d,
                         uint16_t* o, float* lse, cudaStream_t st);
// dk, dv are written per query head: [T, H d] fp32 (the kv-group sum happens in rope_grad)
int launch_attention_bwd(const uint16_t* qkv, const uint16_t* o, const uint16_t* dout,
                         const float* lse, int64_t T, int seq, int H, int Hkv, int d, float* delta,
                         float* dq, float* dk, float* dv, cudaStream_t st);

// ---------------------------------------------------------------- layer internals
struct LayerShapes {
  int64_t D, F, qd, kvd, qkv_n, gu_n;
  int H, Hkv, hd, r;
  float s;
  int absmax_bits;  // 32 or 8
  int weight_bits;  // 4 (NF4) or 16 (bf16)
};
int layer_shapes(const lsq_cfg* cfg, LayerShapes* out);
size_t layer_ws_bytes(const lsq_cfg* cfg, int64_t T);
// dx_out_bf16 may be null (then converted internally).
// rope_cs: the cos/sin table of launch_rope_table for this seq, or null (then the
// layer builds it in its workspace); lora16: this layer's LoRA operands rounded by
// prepare_lora16, or null (then the layer rounds its masters in its workspace)
// saved_u (layer_saved_u_bytes, 256-byte aligned): where the forward leaves this
// layer's rank-r products u = x A^T, and from where the backward of the same
// inputs reads them instead of recomputing them; null in both keeps them in the
// workspace and recomputes them.
int layer_fwd_impl(const lsq_cfg* cfg, const void* blob, const float* lora, const float* x_in,
                   int batch, int seq, float* x_out, void* ws, size_t ws_bytes,
                   cudaStream_t st, const float2* rope_cs = nullptr,
                   const uint16_t* lora16 = nullptr, void* saved_u = nullptr);
size_t layer_saved_u_bytes(const lsq_cfg* cfg, int64_t T);
// The LoRA operands of one layer in their product types (fp16 A, bf16 block-
// diagonal B stacks): elements per layer, and the rounding of n_layers
// consecutive LoRA blocks into out (that many elements apart).
size_t lora16_elems_per_layer(const lsq_cfg* cfg);
int prepare_lora16(const lsq_cfg* cfg, const float* lora, int n_layers, uint16_t* out,
                   cudaStream_t st);
int layer_bwd_impl(const lsq_cfg* cfg, const void* blob, const float* lora, const float* x_in,
                   const float* dx_out, const uint16_t* dx_out_bf16, int batch, int seq,
                   float* dx_in, uint16_t* dx_in_bf16, float* lora_grad, int accumulate,
                   void* ws, size_t ws_bytes, cudaStream_t st, const float2* rope_cs = nullptr,
                   const uint16_t* lora16 = nullptr, const void* saved_u = nullptr);

}  // namespace lsq

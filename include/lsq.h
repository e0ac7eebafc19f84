/*
 * lsq.h - C ABI of the layer-streamed QLoRA (NF4) library for NVIDIA B200 (sm_100a).
 *
 * The library computes the hot path of layer-streamed QLoRA fine-tuning as the
 * pages on "Exact Layer Streaming" describe it:
 *   - the frozen decoder weights are stored as blockwise-absmax NF4 (Soup
 *     layer-streaming tutorial, "Soup layer streaming 的四段資料路徑", part 1 "NF4");
 *   - each frozen linear carries a trainable LoRA branch, y = x W^T + s (x A^T) B^T,
 *     and its backward still reads W: dX = dY W + s (dY B) A (same page, part 3
 *     "Forward＋backward" and FAQ 4);
 *   - the decoder stack sits in page-locked host memory and is fed to the GPU one
 *     layer at a time through two fixed VRAM buffers, the copy running on its own
 *     stream so that it overlaps compute (same page, part 2 "Pinned memory";
 *     Layer Streaming blog, "層流技術：技術實作與記憶體效率");
 *   - every layer is recomputed in backward (tutorial, part 3 and the
 *     "gradient_checkpointing: true" bullet), so each layer is read twice per
 *     micro-batch.
 *
 * Conventions (all entry points):
 *   - Return value: LSQ_OK (0) or one of the LSQ_ERR_* codes below; nothing
 *     aborts or throws.  lsq_last_error() gives a message for the calling thread.
 *   - Memory: the caller owns every buffer (device tensors, pinned host blobs,
 *     workspaces, streams).  The library never allocates or frees caller memory
 *     and allocates no device memory per call.  Opaque handles (lsq_stack) own
 *     only their CUDA events, copy stream and pinned loss slot, and (once
 *     stream_stack_shard has run) an NCCL communicator.
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Unless stated otherwise a call only enqueues work on it; pointers must stay
 *     valid until that work completes.
 *   - Layouts are row-major and contiguous.  bf16 and fp16 tensors are passed as
 *     uint16_t bit patterns.  Device pointers must be 16-byte aligned.
 *   - Precision.  Forward activations that feed tensor cores are fp16, and the
 *     forward GEMMs multiply the dequantised weight rounded to fp16 (an 11-bit
 *     significand: 8x less rounding error than bf16, which keeps a deep stack's
 *     gradients within tolerance); gradients are bf16 (their range needs bf16's
 *     8-bit exponent), the residual stream between layers is fp32, and every
 *     accumulation is fp32.  A forward value beyond the fp16 range (|x| > 65504:
 *     a weight, an absmax, or an activation) latches LSQ_DEV_ERR_NONFINITE in the
 *     device status word.
 *   - Kernel-side errors (a bounded wait that gave up) are latched in a device
 *     status word; lsq_device_status() reads it, the synchronous calls check it.
 */
#ifndef LSQ_H
#define LSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  LSQ_OK = 0,
  LSQ_ERR_INVALID = 1,   /* null pointer, bad enum, non-finite input */
  LSQ_ERR_SHAPE = 2,     /* a size that violates the documented constraints */
  LSQ_ERR_CUDA = 3,      /* a CUDA runtime error (launch or asynchronous) */
  LSQ_ERR_TIMEOUT = 4,   /* a host wait passed its deadline */
  LSQ_ERR_WORKSPACE = 5, /* workspace smaller than the *_workspace_bytes query */
  LSQ_ERR_ALIGN = 6,     /* a pointer that is not 16-byte aligned */
  LSQ_ERR_DEVICE = 7     /* a kernel latched an error in the device status word */
};

/* Message for the last error raised on the calling thread ("" if none). */
const char* lsq_last_error(void);
/* ABI version (major * 100 + minor). */
int lsq_version(void);
/* Reads (and, if clear != 0, resets) the device status word of the current
 * device into *flags.  Synchronises the device.  Returns LSQ_OK or LSQ_ERR_CUDA.
 * Bits: LSQ_DEV_ERR_WAIT (a bounded in-kernel wait gave up), LSQ_DEV_ERR_NONFINITE
 * (a non-finite quantiser input, or a forward value beyond the fp16 range). */
#define LSQ_DEV_ERR_WAIT 1
#define LSQ_DEV_ERR_NONFINITE 2
int lsq_device_status(int* flags, int clear);

/* ------------------------------------------------------------------- NF4 */

/* The 16 NF4 levels as fp32, ascending, derived inside the library from the
 * definition of 4-bit NormalFloat (normal quantiles with an exact zero, scaled
 * to [-1, 1]); host only, needs no GPU. */
int lsq_nf4_codebook(float out_levels[16]);

/* nf4_quantize - blockwise-absmax NF4 quantisation of a frozen weight.
 * Tutorial, "四段資料路徑" part 1 (weights are quantised offline to NF4 shards).
 *   W       device fp32 [N, K] row-major.
 *   block   elements per absmax block; must be 64.  K % 64 == 0, N*K even.
 *   codes   device uint8 [N*K/2]: element 2j in the high nibble of byte j,
 *           element 2j+1 in the low nibble.  Code = index of the nearest level
 *           of w/absmax (fp32 division, exact midpoint -> lower code).
 *   absmax  device fp32 [N*K/64]: max |w| of each block (0 -> all codes 7).
 * Synchronous: waits for the stream, then returns LSQ_ERR_INVALID if W held a
 * NaN, an Inf, or a value beyond 65504 in magnitude (the fp16 range of the
 * fused GEMM's forward operand); codes/absmax are then unspecified.
 * Deterministic. */
int nf4_quantize(const float* W, int64_t N, int64_t K, int32_t block, uint8_t* codes,
                 float* absmax, void* stream);

/* lsq_bf16_from_f32 - round fp32 to bf16 (nearest, ties to even): the storage
 * of an unquantised frozen weight.  x device fp32 [n], y device uint16 [n].
 * Asynchronous. */
int lsq_bf16_from_f32(const float* x, int64_t n, uint16_t* y, void* stream);

/* nf4_dequantize - w~ = fl32(level[code] * absmax) into fp32 W_out [N, K].
 * Same layouts and constraints as nf4_quantize; asynchronous. */
int nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t N, int64_t K,
                   int32_t block, float* W_out, void* stream);

/* nf4_absmax_quantize8 - second-stage (double) quantisation of an NF4 absmax
 * array to 8 bits.  The pages give the stored sizes only (a 3.60 GB store for
 * 32 Llama-3.1-8B layers, 113 MB layer buffers: article "架构解读：layer streaming
 * 如何塞进 4 GB"), which an 8-bit absmax with one fp32 scale per 256 blocks
 * reproduces; the linear scheme below is this library's reading.
 *   absmax    device fp32 [n_blocks], values finite and >= 0 (nf4_quantize's output).
 *   q         device uint8 [n_blocks], 16-byte aligned.
 *   scale     device fp32 [ceil(n_blocks / 256)].
 * For each run of 256 consecutive values (the last may be shorter):
 * scale = fl32(max / 255), q = rint(fl32(a / scale)) half to even, at most 255;
 * a run of zeros gets scale 0, q 0.  Asynchronous, deterministic.  The NF4 codes
 * stay those chosen with the fp32 absmax. */
int nf4_absmax_quantize8(const float* absmax, int64_t n_blocks, uint8_t* q, float* scale,
                         void* stream);

/* nf4_dequantize_dq - w~ = fl32(level[code] * fl32(q[b] * scale[b / 256])) into
 * fp32 W_out [N, K], b = element / 64.  Constraints of nf4_quantize; asynchronous. */
int nf4_dequantize_dq(const uint8_t* codes, const uint8_t* q, const float* scale, int64_t N,
                      int64_t K, int32_t block, float* W_out, void* stream);

/* ------------------------------------------------------- NF4 + LoRA linear */

/* Workspace bytes needed by nf4_lora_linear_fwd/bwd for these sizes. */
size_t nf4_lora_linear_workspace_bytes(int64_t T, int64_t K, int64_t N, int32_t r);

/* nf4_lora_linear_fwd - y = x W~^T + scale * (x A^T) B^T (+ residual).
 * Tutorial part 1 (LoRA A/B trained on top of the frozen NF4 base).
 *   x        device fp16 [T, K];  T >= 1, K % 64 == 0.
 *   codes, absmax  the NF4 weight W [N, K] (layout of nf4_quantize); N % 8 == 0.
 *   A        device fp32 [r, K];  B  device fp32 [N, r];  r % 16 == 0, 16 <= r <= 256.
 *   residual device fp32 [T, N] or NULL (needs y_fp32 = 1).
 *   y        device [T, N] (output): fp16 when y_fp32 == 0, fp32 when y_fp32 == 1.
 *   u_out    device fp32 [T, r] = x A^T, or NULL.
 *   ws       device workspace of nf4_lora_linear_workspace_bytes(T, K, N, r).
 * The dequantised weight, A, scale * B and u are rounded to fp16 for the tensor
 * cores; accumulation is fp32.  Asynchronous, deterministic. */
int nf4_lora_linear_fwd(const uint16_t* x, int64_t T, int64_t K, int64_t N,
                        const uint8_t* codes, const float* absmax, int32_t block,
                        const float* A, const float* B, int32_t r, float scale,
                        const float* residual, void* y, int32_t y_fp32, float* u_out, void* ws,
                        size_t ws_bytes, void* stream);

/* nf4_lora_linear_bwd - backward of the linear above (W frozen).
 * Tutorial part 3 and FAQ 4: dX still needs W.
 *   dy [T, N] bf16 (the gradient), x [T, K] fp16 (the forward input).
 *   dx  device bf16 [T, K] = dy W~ + scale (dy B) A (bf16 products of dy, W~, dy B and
 *       scale A^T; fp32 sums).
 *   dA  device fp32 [r, K] (+)= scale (dy B)^T x;  dB device fp32 [N, r] (+)= scale dy^T (x A^T).
 *   accumulate  0: overwrite dA/dB, 1: add to them.
 * Asynchronous, deterministic (fixed-order reductions, no atomics). */
int nf4_lora_linear_bwd(const uint16_t* dy, const uint16_t* x, int64_t T, int64_t K, int64_t N,
                        const uint8_t* codes, const float* absmax, int32_t block,
                        const float* A, const float* B, int32_t r, float scale, uint16_t* dx,
                        float* dA, float* dB, int32_t accumulate, void* ws, size_t ws_bytes,
                        void* stream);

/* --------------------------------------------------------- decoder layer */

/* Llama-style decoder configuration.  The pages name the model (Llama-3.1-8B,
 * tutorial "維護者的 4GB／8B 成績"); the hyper-parameters are the caller's. */
typedef struct lsq_cfg {
  int64_t hidden;      /* D */
  int64_t ffn;         /* F, SwiGLU inner size */
  int64_t vocab;       /* V */
  int32_t n_heads;     /* H */
  int32_t n_kv_heads;  /* Hkv, H % Hkv == 0 */
  int32_t head_dim;    /* d, must be 128 or 64 */
  int32_t n_layers;    /* L */
  int32_t lora_r;      /* r, multiple of 16 */
  int32_t block;       /* NF4 block, must be 64 */
  float lora_alpha;    /* s = alpha / r */
  float rope_theta;    /* rotate-half RoPE base */
  float rms_eps;       /* RMSNorm epsilon */
  int32_t absmax_bits; /* 0 or 32: fp32 absmax per block; 8: 8-bit absmax with one
                          fp32 scale per 256 blocks (nf4_absmax_quantize8) */
  int32_t weight_bits; /* 0 or 4: NF4 frozen weights; 16: unquantised bf16 weights
                          (the streamed bf16 stacks of the Layer Streaming blog, e.g.
                          Qwen2.5-3B); absmax_bits is then ignored */
} lsq_cfg;

/* Byte layout of one layer's blob (the unit that is streamed).  Projection
 * order q, k, v, o, gate, up, down.  All codes come first, contiguous, so q|k|v
 * and gate|up each form one stacked NF4 matrix; then all absmax arrays (fp32,
 * or uint8 with absmax_bits = 8, then all their fp32 scale arrays); then the
 * two RMSNorm gains (bf16 [D]).  Every section starts 256-byte aligned.  For
 * Llama-3.1-8B shapes a layer is 122,699,776 bytes with fp32 absmax and
 * 112,529,408 bytes (the pages' 113 MB; 3.60 GB for 32 layers) with 8-bit.
 * With weight_bits = 16, codes_off[p] is the offset of the bf16 weight [N, K]
 * (row-major, back to back) and there are no absmax arrays. */
typedef struct lsq_layer_layout {
  uint64_t codes_off[7];
  uint64_t absmax_off[7];   /* fp32 [N*K/64], or uint8 [N*K/64] with absmax_bits 8 */
  uint64_t g1_off, g2_off;
  int64_t rows[7], cols[7]; /* N, K of each projection */
  uint64_t bytes;           /* total blob size (multiple of 256) */
  uint64_t scale_off[7];    /* absmax_bits 8: fp32 [N*K/64/256]; else 0 */
  int32_t absmax_bits;      /* 32 or 8 (NF4 only) */
  int32_t weight_bits;      /* 4 or 16 */
} lsq_layer_layout;

/* Fills *out for cfg.  Host only.  LSQ_ERR_SHAPE unless D, F, H*d, Hkv*d are
 * multiples of 128 and head_dim is 64 or 128. */
int lsq_layer_layout_get(const lsq_cfg* cfg, lsq_layer_layout* out);

/* Layout of one layer's LoRA masters (fp32), offsets in floats:
 *   A_qkv [3r, D] (A_q; A_k; A_v), B_qkv [H*d + 2*Hkv*d, r] (B_q; B_k; B_v),
 *   A_o [r, H*d], B_o [D, r], A_gu [2r, D] (A_gate; A_up), B_gu [2F, r],
 *   A_down [r, F], B_down [D, r].
 * A stack's LoRA buffer is n_layers such blocks back to back (floats_per_layer
 * each); gradients and AdamW moments use the same layout. */
typedef struct lsq_lora_layout {
  int64_t a_off[7], b_off[7]; /* per projection, q..down */
  int64_t floats_per_layer;
} lsq_lora_layout;
int lsq_lora_layout_get(const lsq_cfg* cfg, lsq_lora_layout* out);

/* Workspace for decoder_layer_fwd/bwd with T = batch * seq tokens. */
size_t decoder_layer_workspace_bytes(const lsq_cfg* cfg, int32_t batch, int32_t seq);

/* decoder_layer_fwd - one decoder layer: RMSNorm -> q/k/v (NF4 + LoRA) -> RoPE
 * -> causal GQA attention -> o (+residual) -> RMSNorm -> gate/up -> SwiGLU ->
 * down (+residual).
 *   blob    device pointer to the layer blob (lsq_layer_layout).
 *   lora    device fp32, one layer's LoRA block (lsq_lora_layout), or NULL to
 *           run the layer with its adapter off (every LoRA branch removed: the
 *           reference model of the DPO step).
 *   x_in    device fp32 [batch*seq, D]; x_out device fp32 [batch*seq, D] (the
 *           residual stream is fp32; see the precision convention above).
 * Asynchronous, deterministic. */
int decoder_layer_fwd(const lsq_cfg* cfg, const void* blob, const float* lora,
                      const float* x_in, int32_t batch, int32_t seq, float* x_out,
                      void* ws, size_t ws_bytes, void* stream);

/* decoder_layer_bwd - recomputes the layer's forward from x_in (fp32 [T, D]),
 * then backpropagates dx_out (fp32 [T, D], gradient w.r.t. x_out) into dx_in
 * (fp32 [T, D]) and the LoRA gradients (fp32, lsq_lora_layout; accumulate 0/1).
 * The frozen weights and gains get no gradient.  Asynchronous, deterministic. */
int decoder_layer_bwd(const lsq_cfg* cfg, const void* blob, const float* lora,
                      const float* x_in, const float* dx_out, int32_t batch, int32_t seq,
                      float* dx_in, float* lora_grad, int32_t accumulate, void* ws,
                      size_t ws_bytes, void* stream);

/* ---------------------------------------------------------- streamed stack */

typedef struct lsq_stack lsq_stack;

/* stream_stack_create - binds a decoder stack to two VRAM layer buffers.
 *   layer_blobs  n_layers pointers to layer blobs (lsq_layer_layout).  With
 *                resident == 0 they are page-locked host memory (pinned with
 *                cudaHostAlloc/cudaHostRegister by the caller) and are copied
 *                into vram_buf0/vram_buf1 on the stack's own copy stream; with
 *                resident == 1 they are device memory and are used in place
 *                (the two buffers are then ignored and may be NULL).
 *   vram_buf0/1  device buffers of lsq_layer_layout.bytes each.
 * Creates the handle's copy stream and events on the current device.
 * Buffer contract: while the handle lives, vram_buf0 and vram_buf1 belong to
 * it.  Between steps they keep the layers the last completed step left in them,
 * and the next step uses those layers in place instead of copying them again;
 * so the caller must not write either buffer, nor give it to another handle,
 * until stream_stack_destroy (after a failed step the handle trusts neither
 * buffer and copies every layer it needs). */
int stream_stack_create(const lsq_cfg* cfg, const void* const* layer_blobs, int32_t n_layers,
                        void* vram_buf0, void* vram_buf1, int32_t resident, lsq_stack** out);
int stream_stack_destroy(lsq_stack* stack);

/* AdamW on the LoRA masters (decoupled weight decay, bias correction with
 * step >= 1).  m and v are device fp32 in the LoRA layout. */
typedef struct lsq_adamw {
  float lr, beta1, beta2, eps, weight_decay;
  int32_t step;
  float* m;
  float* v;
} lsq_adamw;

/* Workspace for stream_stack_step with micro-batches of batch x seq tokens. */
size_t stream_stack_workspace_bytes(const lsq_cfg* cfg, int32_t batch, int32_t seq);

/* stream_stack_step - one SFT optimiser step through the streamed stack.
 *   tokens      device int32 [micro_batches, batch, seq], ids in [0, vocab).
 *   emb, lm_head  device bf16 [V, D] (untied, resident); final_norm bf16 [D].
 *   lora        device fp32 stack LoRA buffer (updated in place if opt != NULL).
 *   lora_grad   device fp32, same layout; overwritten with the gradient of the
 *               mean loss over all micro-batches.
 *   opt         AdamW state, or NULL for no update.
 *   loss_out    host float: mean cross-entropy over every predicted position
 *               (positions 0..seq-2 of each sequence, target = next token).
 *   logits_out  device fp32 [batch*seq, V] of the last micro-batch, or NULL.
 * Each micro-batch streams layers 0..L-1 forward, then the lm_head and loss,
 * then L-1..0 backward with per-layer recomputation (the layer's rank-r LoRA
 * products x A^T are kept from its forward; everything else is recomputed).
 * The lm_head, the loss and the head's input gradient run over chunks of whole
 * sequences whose fp32 logits and bf16 logit gradients fit 4 GiB, so the full
 * [batch*seq, V] logits are never held in the workspace.  A layer already in a
 * buffer when it is needed again is not copied again.  Synchronous: returns once
 * the loss is on the host, LSQ_ERR_TIMEOUT if that takes longer than
 * timeout_ms (the work is then still in flight on the streams). */
int stream_stack_step(lsq_stack* stack, const int32_t* tokens, int32_t micro_batches,
                      int32_t batch, int32_t seq, const uint16_t* emb, const uint16_t* lm_head,
                      const uint16_t* final_norm, float* lora, float* lora_grad,
                      const lsq_adamw* opt, float* loss_out, float* logits_out, void* ws,
                      size_t ws_bytes, void* stream, int64_t timeout_ms);

/* Workspace for stream_stack_dpo_step with `pairs` chosen/rejected pairs of seq tokens. */
size_t stream_stack_dpo_workspace_bytes(const lsq_cfg* cfg, int32_t pairs, int32_t seq);

/* stream_stack_dpo_step - one DPO optimiser step through the streamed stack,
 * with the same streamed base and its adapter off as the reference model
 * (Soup release notes, preference losses under layer streaming; Layer
 * Streaming blog, "無記憶體消耗的參考模型").  The pages name DPO and that
 * reference; the loss is the published Direct Preference Optimization one:
 * z = beta ((lp(c) - lr(c)) - (lp(r) - lr(r))), loss = mean over pairs of
 * -log sigmoid(z), where a sequence's log-probability is the sum over positions
 * 0..seq-2 of log softmax(logits)[next token] (no prompt mask).
 *   tokens      device int32 [pairs, 2, seq]: chosen then rejected of each pair.
 *   pairs       1..32; beta > 0.
 *   logps_out   host float [4 * pairs] or NULL: per pair (policy chosen, policy
 *               rejected, reference chosen, reference rejected).
 *   logits_out  device fp32 [2*pairs*seq, V] policy logits, or NULL.
 *   other arguments as stream_stack_step (one micro-batch of 2*pairs sequences).
 * Each layer's reference forward runs right after its policy forward from the
 * same VRAM buffer, so the step copies each layer as often as an SFT step.
 * Synchronous like stream_stack_step. */
int stream_stack_dpo_step(lsq_stack* stack, const int32_t* tokens, int32_t pairs, int32_t seq,
                          float beta, const uint16_t* emb, const uint16_t* lm_head,
                          const uint16_t* final_norm, float* lora, float* lora_grad,
                          const lsq_adamw* opt, float* loss_out, float* logps_out,
                          float* logits_out, void* ws, size_t ws_bytes, void* stream,
                          int64_t timeout_ms);

/* Per-step counters of the last stream_stack_step or stream_stack_dpo_step. */
typedef struct lsq_step_stats {
  int32_t layer_copies;     /* host->device layer copies issued */
  int64_t h2d_bytes;        /* bytes those copies moved */
  float step_ms;            /* device time of the step (events on the compute stream) */
  float copy_wait_ms;       /* summed stall of the compute stream on copy-ready events */
} lsq_step_stats;
int stream_stack_last_stats(const lsq_stack* stack, lsq_step_stats* out);

/* lsq_stream_plan - the layer-visit schedule every streamed step follows
 * (host only; exported so that the schedule can be inspected and tested).
 * A step with micro_batches micro-batches visits layers 0..L-1 (forward), then
 * L-1..0 (backward, recomputing each layer), per micro-batch.  A visit uses a
 * buffer that already holds its layer; otherwise its layer is copied into the
 * buffer the previous visit did not use (the first copy of a step goes to
 * buffer 0 when neither holds the layer).  held0/held1: the layers the two
 * buffers hold before the step (-1: none; a stack starts with -1, -1 and keeps
 * the contents between steps).  Writes, for visit i of 2 * L * micro_batches,
 * layer[i], buf[i] (0 or 1) and copy[i] (1: copied into buf[i] before use),
 * and *n_visits.  LSQ_ERR_SHAPE for n_layers or micro_batches < 1 or bad
 * buffer contents, LSQ_ERR_WORKSPACE if max_visits is too small. */
int lsq_stream_plan(int32_t n_layers, int32_t micro_batches, int32_t held0, int32_t held1,
                    int32_t* layer, int32_t* buf, int32_t* copy, int32_t max_visits,
                    int32_t* n_visits);

/* ------------------------------------------- data-parallel layer sharding */
/* The pages run layer streaming on one GPU and compare it with multi-GPU
 * sharded training (translated project README, the v3 change list: the
 * DeepSpeed ZeRO-3 comparison; RepoDaily review, the feature list's horizontal
 * scaling item); they give no multi-GPU streaming design.  This one is the
 * library's own: with G data-parallel ranks (one process per GPU) each rank
 * copies 1/G of a layer over its own host link and an NCCL all-gather over
 * NVLink / NVSwitch assembles the layer on every GPU. */

#define LSQ_NCCL_ID_BYTES 128

/* lsq_shard_bytes - the slice S of a layer of layer_bytes that each of world
 * ranks copies from host memory: ceil(layer_bytes / world) rounded up to 256
 * bytes.  A sharded stack's two VRAM layer buffers need world * S bytes each.
 * Host only.  Returns 0 if layer_bytes <= 0 or world < 1. */
int64_t lsq_shard_bytes(int64_t layer_bytes, int32_t world);

/* lsq_nccl_unique_id - writes a new NCCL communicator id (id_bytes must be
 * LSQ_NCCL_ID_BYTES) to id_out.  One rank calls it and sends the bytes to every
 * other rank over any host channel.  NCCL is loaded at run time (libnccl.so.2);
 * LSQ_ERR_CUDA if it cannot be loaded or the call fails. */
int lsq_nccl_unique_id(void* id_out, int64_t id_bytes);

/* stream_stack_shard - spreads every later layer copy of a streamed stack
 * (resident == 0) over world data-parallel ranks.  Rank r copies bytes
 * [r S, min((r + 1) S, layout bytes)) of each layer from its own host blob (the
 * rest of its host blobs is never read), then an in-place NCCL all-gather on
 * the stack's copy stream, before the layer's ready event, fills the whole
 * buffer on every rank; S = lsq_shard_bytes(layout bytes, world).
 *   nccl_id    LSQ_NCCL_ID_BYTES from lsq_nccl_unique_id, the same on every rank.
 *   world, rank  this rank among world (0 <= rank < world); world 1 is allowed
 *              (the all-gather is then a local no-op).
 *   buf_bytes  size of each of the stack's two VRAM buffers, >= world * S.
 * Collective and blocking: every rank calls it once, on its stack's device, and
 * it returns when all have joined the communicator.  Afterwards each layer copy
 * is a collective, so every rank must run the same steps (same kind, counts and
 * order).  A step's first copy waits for the work the caller queued on the
 * compute stream before the step (for example a gradient all-reduce on another
 * communicator).  If a step times out (LSQ_ERR_TIMEOUT) the communicator is
 * aborted, which ends any all-gather still waiting for a peer, and the stack
 * refuses further steps (LSQ_ERR_INVALID); destroy it.  stream_stack_destroy
 * also destroys the communicator.  NCCL allocates the communicator's own
 * device buffers once, in this call; steps allocate nothing.  Errors: LSQ_ERR_INVALID (null, wrong id
 * size, resident or already sharded stack, bad rank, wrong device),
 * LSQ_ERR_WORKSPACE (buffers too small), LSQ_ERR_CUDA (NCCL). */
int stream_stack_shard(lsq_stack* stack, const void* nccl_id, int64_t id_bytes, int32_t world,
                       int32_t rank, int64_t buf_bytes);

/* stream_stack_reduce_grads - data-parallel gradient averaging inside the step.
 * With world ranks each streaming the same frozen stack on its own tokens (one
 * process per GPU), the only exchange the method needs is the mean of the LoRA
 * gradients before the optimiser.  After this call every later step of the stack
 * does it itself: as soon as the backward of layer i has finished (in the step's
 * last micro-batch), that layer's gradient block (lsq_lora_layout
 * floats_per_layer floats) is all-reduced in place with NCCL's average on the
 * stack's own reduction stream and communicator, so the exchange overlaps the
 * backward of layers i-1..0; the step's AdamW (opt) waits for the last one and
 * then applies the same update on every rank.  loss_out stays this rank's own
 * loss.  The pages run one GPU; this is the library's data-parallel form.
 *   nccl_id  LSQ_NCCL_ID_BYTES from lsq_nccl_unique_id, the same on every rank
 *            (not the id given to stream_stack_shard: this is a second communicator).
 *   world, rank  this rank among world (world 1 is allowed: the average is a copy).
 * Collective and blocking like stream_stack_shard; every rank must then run the
 * same steps.  A step that times out aborts this communicator too.  Errors:
 * LSQ_ERR_INVALID (null, wrong id size, already set up, bad rank, wrong device),
 * LSQ_ERR_CUDA (NCCL). */
int stream_stack_reduce_grads(lsq_stack* stack, const void* nccl_id, int64_t id_bytes,
                              int32_t world, int32_t rank);

/* ------------------------------------------------------------ optimiser */

/* lora_adamw_step - one AdamW update of n LoRA parameters (fp32, any layout
 * shared by lora, grad, opt->m, opt->v): m = b1 m + (1-b1) g, v = b2 v + (1-b2) g^2,
 * p = p (1 - lr wd) - lr (m / (1-b1^step)) / (sqrt(v / (1-b2^step)) + eps).
 * The same update stream_stack_step applies; exported so that data-parallel
 * callers can reduce gradients across ranks between the step and the update.
 * Asynchronous. */
int lora_adamw_step(float* lora, const float* grad, const lsq_adamw* opt, int64_t n, void* stream);

/* ------------------------------------------------------------ measurement */

/* Number of kernel launches the library has issued in this process. */
int64_t lsq_launch_counter(void);

/* Per-launch device timing of the library's kernels.  While enabled, every
 * tensor-core GEMM (with its split-K reduce), attention, rank-r LoRA product and
 * memory-bound kernel (RMSNorm, RoPE, SwiGLU, embedding, cross-entropy, AdamW)
 * launch is bracketed by CUDA events recorded on the stream it is launched on,
 * together with its algorithmic work (FLOPs, and the minimum DRAM bytes it must
 * move).  Enabling costs two event records per such launch. */
typedef struct lsq_prof_entry {
  char name[32];       /* kernel class, e.g. "gemm_nf4_fwd" */
  int64_t launches;
  double total_ms;     /* summed event time of those launches */
  double flops;        /* summed algorithmic FLOPs */
  double bytes;        /* summed algorithmic DRAM bytes */
} lsq_prof_entry;
/* enable != 0 starts recording (and clears earlier records); 0 stops. */
int lsq_profile_enable(int enable);
/* Synchronises the recorded events and fills up to max entries (one per class). */
int lsq_profile_read(lsq_prof_entry* out, int32_t max, int32_t* n_out);

/* lsq_gemm_plan_get - the launch plan of the fused tensor-core GEMM behind every
 * frozen projection (host only; exported so that the planner can be inspected and
 * tested without a GPU).  The product is out[T, M] = act[T, Kc] . Wop[M, Kc]^T with
 * the operand mode:
 *   LSQ_GEMM_NF4_FWD  Wop = deq(W), W NF4 [M, Kc] (forward, fp16 operands);
 *   LSQ_GEMM_NF4_DX   Wop = deq(W)^T, W NF4 [Kc, M] (input gradient, bf16 operands);
 *   LSQ_GEMM_BF16_FWD, LSQ_GEMM_BF16_DX  the same with a bf16 W (lm_head);
 *   LSQ_GEMM_BF16_AS_F16_FWD  a bf16 W [M, Kc] converted to fp16 in the operand stage.
 * num_sms is the GPU's SM count (148 on B200); allow_pair = 0 asks for one-CTA tiles
 * (the library uses CTA pairs unless LSQ_GEMM_PAIR=0 is set in the environment).
 * LSQ_ERR_INVALID for a bad mode or a null out; LSQ_ERR_SHAPE for a non-positive
 * size or num_sms, or a size beyond 2^31 - 1.  Added in ABI 2.1. */
#define LSQ_GEMM_NF4_FWD 0
#define LSQ_GEMM_NF4_DX 1
#define LSQ_GEMM_BF16_FWD 2
#define LSQ_GEMM_BF16_DX 3
#define LSQ_GEMM_BF16_AS_F16_FWD 4
typedef struct lsq_gemm_plan {
  int32_t pair;               /* 1: CTA pairs (cta_group::2 MMAs, 256 features per pair) */
  int32_t bn, nacc;           /* tokens per TMEM accumulator; accumulators per tile (1, 2) */
  int32_t m_tiles, t_tiles, splits;  /* grid: 128-feature tiles x token tiles x K slices */
  int32_t kt_total, kt_per_split;    /* 64-wide contraction tiles: all, per slice */
  int32_t stages, ring_stages;       /* operand stages; NF4 code-ring slots */
  int32_t x_stage_bytes;      /* activation bytes of one stage, per CTA */
  int32_t w_stage_bytes;      /* weight-operand bytes of one stage */
  int32_t ring_bytes;         /* bytes of one code-ring slot (0: no ring) */
  int32_t absmax_ring_bytes;  /* the absmax prefetch ring */
  int32_t smem_bytes;         /* dynamic shared memory of the launch */
  int32_t smem_limit;         /* the most dynamic shared memory the kernel is given */
  int32_t epilogue_bytes;     /* shared memory the epilogue's staging slots use */
  int32_t tmem_cols;          /* TMEM columns allocated per CTA */
  int64_t partial_bytes;      /* split-K workspace (fp32 partials; 0 when unsplit) */
} lsq_gemm_plan;
int lsq_gemm_plan_get(int32_t mode, int64_t M, int64_t T, int64_t Kc, int32_t num_sms,
                      int32_t allow_pair, lsq_gemm_plan* out);

/* lsq_lora_plan_get - the launch plan of the tensor-core kernel behind the LoRA
 * rank-r products (u = x A^T, v = dY B, dA, dB): C [M, N] = A [M, K] . B [N, K]^T
 * (host only; exported so that the planner can be inspected and tested without a
 * GPU).  num_sms is the GPU's SM count.  A product whose tiles leave at least half
 * of the resident CTA slots empty splits its reduction over a thread-block
 * cluster of `splits` CTAs, whose accumulators are summed in shared memory.
 * LSQ_ERR_INVALID for a null out; LSQ_ERR_SHAPE for a non-positive size or
 * num_sms.  Added in ABI 2.1. */
typedef struct lsq_lora_plan {
  int32_t n_pad;              /* columns per CTA: N rounded up to 16, at most 256 */
  int32_t row_tiles, col_tiles, splits;  /* grid: 128-row tiles x column tiles x slices */
  int32_t kt_total;           /* 64-wide reduction stages */
  int32_t stages;             /* operand stages in flight */
  int32_t stage_bytes;        /* bytes of one stage (A tile + B tile) */
  int32_t smem_bytes;         /* dynamic shared memory of the launch */
  int32_t smem_limit;         /* the most dynamic shared memory the kernel is given */
  int32_t ctas_per_sm;        /* resident CTAs per SM the plan assumes */
  int32_t tmem_cols;          /* TMEM columns allocated per CTA */
  int32_t reduce_bytes;       /* shared memory of the cluster sum (0 when unsplit) */
} lsq_lora_plan;
int lsq_lora_plan_get(int64_t M, int64_t N, int64_t K, int32_t num_sms, lsq_lora_plan* out);

/* --------------------------------------------------- allocation-free variant */

/* nf4_lora_linear_fwd_noalloc - the same computation and kernels as
 * nf4_lora_linear_fwd, for callers that cannot provide a device workspace (a
 * host framework that keeps all device memory in its own pool and gives plugins
 * no allocator, or a latency-critical caller that cannot afford the device-wide
 * synchronisation cudaMalloc/cudaFree may cause).  This entry point is an
 * engineering addition with no counterpart on the pages the method comes from.
 *   Arguments as nf4_lora_linear_fwd, without ws/ws_bytes.
 *   Scratch: a fixed 32 MiB device array built into the library.  Sizes whose
 *   nf4_lora_linear_workspace_bytes exceeds 32 MiB are rejected with
 *   LSQ_ERR_WORKSPACE.  Calls after the first on a device allocate nothing.
 *   The first call on each device looks up the array's device address (with
 *   that device current).  With CUDA's lazy module loading (the default since
 *   CUDA 12.2) that lookup is also what loads the array onto the device, i.e.
 *   it reserves 32 MiB of device memory there and can fail (LSQ_ERR_CUDA) if the
 *   device is full.  So make the first call on each device early: before the
 *   caller's own pool takes all device memory, and before any stream capture.
 *   The array then stays on that device until the process exits.
 *   All calls share the one array: calls that can overlap on the GPU (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.  Nothing in the array needs to start at zero. */
int nf4_lora_linear_fwd_noalloc(const uint16_t* x, int64_t T, int64_t K, int64_t N,
                                const uint8_t* codes, const float* absmax, int32_t block,
                                const float* A, const float* B, int32_t r, float scale,
                                const float* residual, void* y, int32_t y_fp32, float* u_out,
                                void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LSQ_H */

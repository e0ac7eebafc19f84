// One Llama-style decoder layer whose seven frozen projections are NF4 with a
// LoRA branch each: forward, and backward with the layer recomputed from its
// saved input (Soup layer-streaming tutorial, "四段資料路徑" part 3, and the
// "gradient_checkpointing: true" bullet: the streaming wrapper checkpoints
// every layer, so backward re-reads the layer and rebuilds its activations).
//
// Fusions: q|k|v and gate|up are stored back to back in the layer blob, so each
// group is one NF4 GEMM; the LoRA up-projections ride in those GEMMs as an
// extra K slab; the o and down GEMMs add the residual in their epilogue.
//
// Precision: the residual stream (the layer's input and output, and h) is fp32;
// the forward activations that feed tensor cores (n1, q|k|v, attention output,
// n2, gate|up, the SwiGLU product) are fp16, as is the dequantised weight in the
// forward GEMMs; gradients that feed tensor cores are bf16; every accumulation,
// norm and softmax is fp32.
#include "common.cuh"

namespace lsq {

int layer_shapes(const lsq_cfg* cfg, LayerShapes* o) {
  if (!cfg) return set_error(LSQ_ERR_INVALID, "null config");
  if (cfg->absmax_bits != 0 && cfg->absmax_bits != 32 && cfg->absmax_bits != 8)
    return set_error(LSQ_ERR_INVALID, "cfg.absmax_bits must be 0, 32 or 8");
  if (cfg->weight_bits != 0 && cfg->weight_bits != 4 && cfg->weight_bits != 16)
    return set_error(LSQ_ERR_INVALID, "cfg.weight_bits must be 0, 4 or 16");
  if (cfg->block != 64) return set_error(LSQ_ERR_SHAPE, "cfg.block must be 64");
  if (cfg->head_dim != 64 && cfg->head_dim != 128)
    return set_error(LSQ_ERR_SHAPE, "cfg.head_dim must be 64 or 128");
  if (cfg->n_heads <= 0 || cfg->n_kv_heads <= 0 || cfg->n_heads % cfg->n_kv_heads != 0)
    return set_error(LSQ_ERR_SHAPE, "cfg: n_heads must be a positive multiple of n_kv_heads");
  if (cfg->n_heads + cfg->n_kv_heads > 4 * cfg->n_heads)
    return set_error(LSQ_ERR_SHAPE, "cfg: bad head counts");
  if (cfg->lora_r <= 0 || cfg->lora_r % 16 != 0 || cfg->lora_r > 64)
    return set_error(LSQ_ERR_SHAPE, "cfg.lora_r must be 16, 32, 48 or 64");
  const int64_t qd = (int64_t)cfg->n_heads * cfg->head_dim;
  const int64_t kvd = (int64_t)cfg->n_kv_heads * cfg->head_dim;
  if (cfg->hidden <= 0 || cfg->hidden % 128 || cfg->ffn <= 0 || cfg->ffn % 128 || qd % 128 ||
      kvd % 128)
    return set_error(LSQ_ERR_SHAPE, "cfg: hidden, ffn, n_heads*head_dim and n_kv_heads*head_dim "
                                    "must be multiples of 128");
  o->D = cfg->hidden;
  o->F = cfg->ffn;
  o->qd = qd;
  o->kvd = kvd;
  o->qkv_n = qd + 2 * kvd;
  o->gu_n = 2 * cfg->ffn;
  o->H = cfg->n_heads;
  o->Hkv = cfg->n_kv_heads;
  o->hd = cfg->head_dim;
  o->r = cfg->lora_r;
  o->s = cfg->lora_alpha / (float)cfg->lora_r;
  // With 8-bit absmax every projection has a multiple of 256 blocks (its rows
  // and columns are multiples of 128), so a scale run never straddles two
  // projections and the stacked q|k|v and gate|up matrices index one array.
  o->absmax_bits = cfg->absmax_bits == 8 ? 8 : 32;
  o->weight_bits = cfg->weight_bits == 16 ? 16 : 4;
  return LSQ_OK;
}

namespace {

struct AbsmaxRef {  // fp32 absmax, or 8-bit absmax with its run scales; or a bf16 weight
  const float* f32 = nullptr;
  const uint8_t* q = nullptr;
  const float* s = nullptr;
  bool bf16 = false;  // the weight is unquantised bf16 (no absmax)
};

struct Views {  // pointers into one layer blob / one LoRA block
  const uint8_t* codes[7];
  AbsmaxRef absmax[7];
  const uint16_t* g1;
  const uint16_t* g2;
  const float *A_qkv, *B_qkv, *A_o, *B_o, *A_gu, *B_gu, *A_d, *B_d;
  // the same operands rounded once into their product types (Lora16)
  const uint16_t *A16_qkv, *A16_o, *A16_gu, *A16_d, *B16_qkv, *B16_o, *B16_gu, *B16_d;
  // the fused GEMMs' LoRA slab operands: s B stacks (fp16, forward) and s A^T (bf16, dX)
  const uint16_t *Bs16_qkv, *Bs16_o, *Bs16_gu, *Bs16_d, *At16_qkv, *At16_o, *At16_gu, *At16_d;
  bool lora_on;  // false: adapter disabled, every LoRA branch removed
};

void fill_layout(const LayerShapes& s, lsq_layer_layout* L, lsq_lora_layout* R) {
  const int64_t rows[7] = {s.qd, s.kvd, s.kvd, s.D, s.F, s.F, s.D};
  const int64_t cols[7] = {s.D, s.D, s.D, s.qd, s.D, s.D, s.F};
  uint64_t off = 0;
  const bool bf16 = s.weight_bits == 16;
  for (int p = 0; p < 7; ++p) {
    L->rows[p] = rows[p];
    L->cols[p] = cols[p];
    L->codes_off[p] = off;
    off += (uint64_t)rows[p] * cols[p] * (bf16 ? 2 : 1) / (bf16 ? 1 : 2);
  }
  off = (off + 255) & ~uint64_t(255);
  L->absmax_bits = s.absmax_bits;
  L->weight_bits = s.weight_bits;
  for (int p = 0; p < 7; ++p) {
    L->absmax_off[p] = 0;
    if (bf16) continue;
    L->absmax_off[p] = off;
    off += (uint64_t)rows[p] * cols[p] / 64 * (s.absmax_bits == 8 ? 1 : 4);
  }
  off = (off + 255) & ~uint64_t(255);
  for (int p = 0; p < 7; ++p) {
    L->scale_off[p] = 0;
    if (!bf16 && s.absmax_bits == 8) {
      L->scale_off[p] = off;
      off += ((uint64_t)rows[p] * cols[p] / 64 + 255) / 256 * 4;
    }
  }
  off = (off + 255) & ~uint64_t(255);
  L->g1_off = off;
  off += (uint64_t)s.D * 2;
  off = (off + 255) & ~uint64_t(255);
  L->g2_off = off;
  off += (uint64_t)s.D * 2;
  L->bytes = (off + 255) & ~uint64_t(255);
  // LoRA block, each piece 64-float aligned
  auto al = [](int64_t x) { return (x + 63) & ~int64_t(63); };
  const int64_t r = s.r;
  int64_t f = 0;
  const int64_t a_qkv = f;  f = al(f + 3 * r * s.D);
  const int64_t b_qkv = f;  f = al(f + s.qkv_n * r);
  const int64_t a_o = f;    f = al(f + r * s.qd);
  const int64_t b_o = f;    f = al(f + s.D * r);
  const int64_t a_gu = f;   f = al(f + 2 * r * s.D);
  const int64_t b_gu = f;   f = al(f + s.gu_n * r);
  const int64_t a_d = f;    f = al(f + r * s.F);
  const int64_t b_d = f;    f = al(f + s.D * r);
  R->a_off[0] = a_qkv;             R->b_off[0] = b_qkv;
  R->a_off[1] = a_qkv + r * s.D;   R->b_off[1] = b_qkv + s.qd * r;
  R->a_off[2] = a_qkv + 2 * r * s.D; R->b_off[2] = b_qkv + (s.qd + s.kvd) * r;
  R->a_off[3] = a_o;               R->b_off[3] = b_o;
  R->a_off[4] = a_gu;              R->b_off[4] = b_gu;
  R->a_off[5] = a_gu + r * s.D;    R->b_off[5] = b_gu + s.F * r;
  R->a_off[6] = a_d;               R->b_off[6] = b_d;
  R->floats_per_layer = f;
}

// One layer's LoRA operands in their product types, rounded once from the fp32
// masters (per optimiser step in the stack): fp16 A_qkv [3r, D], A_o [r, H d],
// A_gu [2r, D], A_down [r, F] for u = x A^T; bf16 block-diagonal B stacks for
// v = dY B, one product per projection group: B_qkv -> [qkv rows, 3r],
// B_o [D, r], B_gu -> [2F, 2r], B_down [D, r]; and the fused GEMMs' LoRA slab
// operands: the scaled B stacks s B in fp16, [qkv rows, 3r] ... (the forward),
// and the scaled transposed A stacks s A^T in bf16, [D, 3r], [H d, r], [D, 2r],
// [F, r] (the input gradient).  Offsets in elements, each block 128-element
// (256-byte) aligned.
struct Lora16 {
  int64_t a[4], b[4], bs[4], at[4], elems;
};
Lora16 lora16_layout(const LayerShapes& s) {
  auto al = [](int64_t x) { return (x + 127) & ~int64_t(127); };
  const int64_t r = s.r;
  Lora16 o;
  int64_t f = 0;
  o.a[0] = f; f = al(f + 3 * r * s.D);
  o.a[1] = f; f = al(f + r * s.qd);
  o.a[2] = f; f = al(f + 2 * r * s.D);
  o.a[3] = f; f = al(f + r * s.F);
  o.b[0] = f; f = al(f + s.qkv_n * 3 * r);
  o.b[1] = f; f = al(f + s.D * r);
  o.b[2] = f; f = al(f + s.gu_n * 2 * r);
  o.b[3] = f; f = al(f + s.D * r);
  o.bs[0] = f; f = al(f + s.qkv_n * 3 * r);
  o.bs[1] = f; f = al(f + s.D * r);
  o.bs[2] = f; f = al(f + s.gu_n * 2 * r);
  o.bs[3] = f; f = al(f + s.D * r);
  o.at[0] = f; f = al(f + s.D * 3 * r);
  o.at[1] = f; f = al(f + s.qd * r);
  o.at[2] = f; f = al(f + s.D * 2 * r);
  o.at[3] = f; f = al(f + s.F * r);
  o.elems = f;
  return o;
}
LoraPrepSegs lora16_segs(const LayerShapes& s, const lsq_lora_layout& R, const Lora16& o) {
  LoraPrepSegs g{};
  const int64_t r = s.r;
  const int64_t arows[4] = {3 * r, r, 2 * r, r}, acols[4] = {s.D, s.qd, s.D, s.F};
  const int64_t asrc[4] = {R.a_off[0], R.a_off[3], R.a_off[4], R.a_off[6]};
  for (int i = 0; i < 4; ++i) {
    LoraPrepSeg& e = g.seg[i];
    e.kind = 0;
    e.src_off = asrc[i];
    e.dst_off = o.a[i];
    e.rows = arows[i];
    e.cols = acols[i];
    e.ld_out = acols[i];
    e.n_parts = 1;
  }
  const int64_t brows[4] = {s.qkv_n, s.D, s.gu_n, s.D};
  const int64_t bsrc[4] = {R.b_off[0], R.b_off[3], R.b_off[4], R.b_off[6]};
  const int bparts[4] = {3, 1, 2, 1};
  const int64_t pe[4][3] = {{s.qd, s.qd + s.kvd, s.qkv_n}, {s.D, 0, 0}, {s.F, s.gu_n, 0},
                            {s.D, 0, 0}};
  for (int i = 0; i < 4; ++i) {
    LoraPrepSeg& e = g.seg[4 + i];
    e.kind = 1;
    e.src_off = bsrc[i];
    e.dst_off = o.b[i];
    e.rows = brows[i];
    e.cols = r;
    e.ld_out = bparts[i] * r;
    e.n_parts = bparts[i];
    for (int p = 0; p < bparts[i]; ++p) e.part_end[p] = pe[i][p];
    LoraPrepSeg& f = g.seg[8 + i];  // s B, untransposed, fp16
    f = e;
    f.kind = 2;
    f.dst_off = o.bs[i];
    f.scale = s.s;
  }
  for (int i = 0; i < 4; ++i) {  // s A^T, bf16
    LoraPrepSeg& e = g.seg[12 + i];
    e.kind = 3;
    e.src_off = asrc[i];
    e.dst_off = o.at[i];
    e.rows = acols[i];
    e.cols = arows[i];
    e.ld_out = arows[i];
    e.n_parts = 1;
    e.scale = s.s;
  }
  g.n = 16;
  return g;
}

Views views(const LayerShapes& s, const void* blob, const float* lora) {
  lsq_layer_layout L;
  lsq_lora_layout R;
  fill_layout(s, &L, &R);
  Views v;
  const uint8_t* b = static_cast<const uint8_t*>(blob);
  for (int p = 0; p < 7; ++p) {
    v.codes[p] = b + L.codes_off[p];
    if (s.weight_bits == 16) {
      v.absmax[p].bf16 = true;
    } else if (s.absmax_bits == 8) {
      v.absmax[p].q = b + L.absmax_off[p];
      v.absmax[p].s = reinterpret_cast<const float*>(b + L.scale_off[p]);
    } else {
      v.absmax[p].f32 = reinterpret_cast<const float*>(b + L.absmax_off[p]);
    }
  }
  v.g1 = reinterpret_cast<const uint16_t*>(b + L.g1_off);
  v.g2 = reinterpret_cast<const uint16_t*>(b + L.g2_off);
  v.lora_on = lora != nullptr;
  v.A_qkv = v.B_qkv = v.A_o = v.B_o = v.A_gu = v.B_gu = v.A_d = v.B_d = nullptr;
  v.A16_qkv = v.A16_o = v.A16_gu = v.A16_d = v.B16_qkv = v.B16_o = v.B16_gu = v.B16_d = nullptr;
  v.Bs16_qkv = v.Bs16_o = v.Bs16_gu = v.Bs16_d = nullptr;
  v.At16_qkv = v.At16_o = v.At16_gu = v.At16_d = nullptr;
  if (v.lora_on) {
    v.A_qkv = lora + R.a_off[0];
    v.B_qkv = lora + R.b_off[0];
    v.A_o = lora + R.a_off[3];
    v.B_o = lora + R.b_off[3];
    v.A_gu = lora + R.a_off[4];
    v.B_gu = lora + R.b_off[4];
    v.A_d = lora + R.a_off[6];
    v.B_d = lora + R.b_off[6];
  }
  return v;
}

// Workspace carve-up (identical for the forward and the backward).
struct Buffers {
  uint16_t* lora16;                                  // this layer's Lora16 (when not given)
  uint16_t *u16_qkv, *u16_o, *u16_gu, *u16_d;        // bf16 copies of u, for dB ([R][ld])
  uint16_t *v16_qkv, *v16_o, *v16_gu, *v16_d;        // bf16 copies of v, for dA ([R][ld])
  float* h;                                          // fp32 residual stream after attention
  uint16_t *n1, *qkv, *ao, *n2, *gu, *m;             // fp16 forward activations
  uint16_t *dgu, *dqkv, *da, *dout_b, *dh_b;         // bf16 gradients
  uint16_t *uh_qkv, *uh_o, *uh_gu, *uh_d;  // u in fp16, [T][R]: the forward GEMMs' LoRA slab
  uint16_t *vh_qkv, *vh_o, *vh_gu, *vh_d;  // v in bf16, [T][R]: the dX GEMMs' LoRA slab
  float *rstd1, *rstd2, *lse;
  float *dm, *dn2, *dh, *dn1, *dq, *dk, *dv, *delta;
  float2* rope_cs;
  float* lscratch;
  size_t lscratch_bytes;
  void* gemm;
  size_t gemm_bytes;
};

// Forward of a stacked frozen weight W [N, K] (NF4, or bf16 when absmax is
// empty, converted to fp16 in the operand stage): out [T, N] = act W^T + u Bs^T,
// fp16; or, with a residual, out = that + residual in fp32.  The LoRA branch is
// the GEMM's slab of R columns: Bs = s B (fp16 [N][R], each row's part's columns
// only, zeros elsewhere) and u (fp16 [T][R]); R = 0 without an adapter.
GemmDesc nf4_fwd(const uint8_t* codes, const AbsmaxRef& absmax, int64_t N, int64_t K,
                 const uint16_t* act, int64_t T, const uint16_t* Bs, const uint16_t* u, int R,
                 const float* res, void* out, int64_t ldo) {
  GemmDesc d;
  const bool bf16 = absmax.bf16;
  d.wmode = bf16 ? W_BF16C_N : W_NF4_N;
  d.M = N;
  d.T = T;
  d.Kc = K;
  d.w = codes;
  d.absmax = absmax.f32;
  d.absmax_q = absmax.q;
  d.absmax_s = absmax.s;
  d.w_rows = N;
  d.w_cols = K;
  d.act = act;
  d.act_ld = K;
  d.slab_w = R;
  d.la16 = Bs;
  d.la16_ld = R;
  d.lb16 = u;
  d.lb16_ld = R;
  d.out = out;
  d.ldo = ldo;
  d.out_f32 = res != nullptr;
  d.residual = res;
  d.ldr = ldo;
  return d;
}

// dX of a stacked weight W [N, K]: out [T, K] = dy W + v At^T, with At = s A_stack^T
// (bf16 [K][R]) and v (bf16 [T][R]) as the GEMM's slab.
GemmDesc nf4_dx(const uint8_t* codes, const AbsmaxRef& absmax, int64_t N, int64_t K,
                const uint16_t* dy, int64_t T, const uint16_t* At, const uint16_t* v, int R,
                void* out, int out_f32) {
  GemmDesc d;
  const bool bf16 = absmax.bf16;
  d.wmode = bf16 ? W_BF16_T : W_NF4_T;
  d.M = K;
  d.T = T;
  d.Kc = N;
  d.w = codes;
  d.absmax = absmax.f32;
  d.absmax_q = absmax.q;
  d.absmax_s = absmax.s;
  d.w_rows = N;
  d.w_cols = K;
  d.act = dy;
  d.act_ld = N;
  d.slab_w = R;
  d.la16 = At;
  d.la16_ld = R;
  d.lb16 = v;
  d.lb16_ld = R;
  d.out = out;
  d.out_f32 = out_f32;
  d.ldo = K;
  return d;
}

size_t plan_buffers(const LayerShapes& s, int64_t T, void* base, Buffers* b) {
  Arena a;
  a.base = static_cast<uint8_t*>(base);
  a.cap = SIZE_MAX;
  const int r = s.r;
  Buffers x{};
  x.n1 = a.take<uint16_t>(T * s.D);
  x.qkv = a.take<uint16_t>(T * s.qkv_n);
  x.ao = a.take<uint16_t>(T * s.qd);
  x.h = a.take<float>(T * s.D);
  x.n2 = a.take<uint16_t>(T * s.D);
  x.gu = a.take<uint16_t>(T * s.gu_n);
  x.m = a.take<uint16_t>(T * s.F);
  x.dgu = a.take<uint16_t>(T * s.gu_n);
  x.dqkv = a.take<uint16_t>(T * s.qkv_n);
  x.da = a.take<uint16_t>(T * s.qd);
  x.dout_b = a.take<uint16_t>(T * s.D);
  x.dh_b = a.take<uint16_t>(T * s.D);
  x.rstd1 = a.take<float>(T);
  x.rstd2 = a.take<float>(T);
  x.lora16 = a.take<uint16_t>(lora16_layout(s).elems);
  const int64_t t16 = lora16_ld(T);  // u16, v16: [R][t16], transposed
  x.u16_qkv = a.take<uint16_t>(t16 * 3 * r);
  x.u16_o = a.take<uint16_t>(t16 * r);
  x.u16_gu = a.take<uint16_t>(t16 * 2 * r);
  x.u16_d = a.take<uint16_t>(t16 * r);
  x.v16_qkv = a.take<uint16_t>(t16 * 3 * r);
  x.v16_o = a.take<uint16_t>(t16 * r);
  x.v16_gu = a.take<uint16_t>(t16 * 2 * r);
  x.v16_d = a.take<uint16_t>(t16 * r);
  x.uh_qkv = a.take<uint16_t>(T * 3 * r);
  x.uh_o = a.take<uint16_t>(T * r);
  x.uh_gu = a.take<uint16_t>(T * 2 * r);
  x.uh_d = a.take<uint16_t>(T * r);
  x.lse = a.take<float>(T * s.H);
  x.vh_qkv = a.take<uint16_t>(T * 3 * r);
  x.vh_o = a.take<uint16_t>(T * r);
  x.vh_gu = a.take<uint16_t>(T * 2 * r);
  x.vh_d = a.take<uint16_t>(T * r);
  x.dm = a.take<float>(T * s.F);
  x.dn2 = a.take<float>(T * s.D);
  x.dh = a.take<float>(T * s.D);
  x.dn1 = a.take<float>(T * s.D);
  x.dq = a.take<float>(T * s.qd);
  x.dk = a.take<float>(T * s.qd);   // per query head, summed per kv head in rope_grad
  x.dv = a.take<float>(T * s.qd);
  x.delta = a.take<float>(T * s.H);
  x.rope_cs = a.take<float2>(T * s.hd / 2);  // >= seq * d/2 entries
  // LoRA K-split scratch: the largest of every skinny product in the layer
  size_t ls = 0;
  const int64_t Ks[4] = {s.D, s.qd, s.F, std::max(s.qkv_n, s.gu_n)};
  for (int i = 0; i < 4; ++i) ls = std::max(ls, lora_scratch_bytes(T, Ks[i], 3 * r));
  x.lscratch = a.take<float>(ls / sizeof(float) + 1);
  x.lscratch_bytes = ls;
  // GEMM split-K partials: the largest of the layer's GEMMs
  const int64_t pe3[3] = {s.qd, s.qd + s.kvd, s.qkv_n};
  const int64_t pe2[2] = {s.F, s.gu_n};
  size_t gb = 0;
  GemmDesc ds[8] = {
      nf4_fwd(nullptr, AbsmaxRef{}, s.qkv_n, s.D, nullptr, T, nullptr, nullptr, 3 * r, nullptr,
              nullptr, s.qkv_n),
      nf4_fwd(nullptr, AbsmaxRef{}, s.D, s.qd, nullptr, T, nullptr, nullptr, r, nullptr, nullptr,
              s.D),
      nf4_fwd(nullptr, AbsmaxRef{}, s.gu_n, s.D, nullptr, T, nullptr, nullptr, 2 * r, nullptr,
              nullptr, s.gu_n),
      nf4_fwd(nullptr, AbsmaxRef{}, s.D, s.F, nullptr, T, nullptr, nullptr, r, nullptr, nullptr,
              s.D),
      nf4_dx(nullptr, AbsmaxRef{}, s.D, s.F, nullptr, T, nullptr, nullptr, r, nullptr, 1),
      nf4_dx(nullptr, AbsmaxRef{}, s.gu_n, s.D, nullptr, T, nullptr, nullptr, 2 * r, nullptr, 1),
      nf4_dx(nullptr, AbsmaxRef{}, s.D, s.qd, nullptr, T, nullptr, nullptr, r, nullptr, 0),
      nf4_dx(nullptr, AbsmaxRef{}, s.qkv_n, s.D, nullptr, T, nullptr, nullptr, 3 * r, nullptr, 1)};
  for (auto& d : ds) gb = std::max(gb, gemm_workspace_bytes(d));
  x.gemm = a.take<uint8_t>(gb + 256);
  x.gemm_bytes = gb + 256;
  if (b) *b = x;
  return a.used;
}

// The rank-r products u = x A^T of one forward (fp16 [T][R] per projection group,
// read by the GEMMs' LoRA slab, and their bf16 [R][lora16_ld(T)] copies, read by
// dB), carved from a region the caller keeps from the forward to the backward.
size_t carve_saved_u(const LayerShapes& s, int64_t T, void* base, Buffers* b) {
  Arena a;
  a.base = static_cast<uint8_t*>(base);
  a.cap = SIZE_MAX;
  const int r = s.r;
  const int64_t t16 = lora16_ld(T);
  uint16_t* uh_qkv = a.take<uint16_t>(T * 3 * r);
  uint16_t* uh_o = a.take<uint16_t>(T * r);
  uint16_t* uh_gu = a.take<uint16_t>(T * 2 * r);
  uint16_t* uh_d = a.take<uint16_t>(T * r);
  uint16_t* u16_qkv = a.take<uint16_t>(t16 * 3 * r);
  uint16_t* u16_o = a.take<uint16_t>(t16 * r);
  uint16_t* u16_gu = a.take<uint16_t>(t16 * 2 * r);
  uint16_t* u16_d = a.take<uint16_t>(t16 * r);
  if (b && base) {
    b->uh_qkv = uh_qkv;
    b->uh_o = uh_o;
    b->uh_gu = uh_gu;
    b->uh_d = uh_d;
    b->u16_qkv = u16_qkv;
    b->u16_o = u16_o;
    b->u16_gu = u16_gu;
    b->u16_d = u16_d;
  }
  return a.used;
}

// Points v at this layer's LoRA operands in product types: the given lora16, or
// (lora16 null) the masters rounded into the workspace first.
int attach_lora16(const LayerShapes& s, const float* lora, const uint16_t* lora16,
                  const Buffers& b, Views* v, cudaStream_t st) {
  if (!v->lora_on) return LSQ_OK;
  const Lora16 o = lora16_layout(s);
  if (!lora16) {
    lsq_layer_layout L;
    lsq_lora_layout R;
    fill_layout(s, &L, &R);
    LSQ_TRY(launch_lora_prepare(lora, R.floats_per_layer, 1, b.lora16, o.elems,
                                lora16_segs(s, R, o), st));
    lora16 = b.lora16;
  }
  v->A16_qkv = lora16 + o.a[0];
  v->A16_o = lora16 + o.a[1];
  v->A16_gu = lora16 + o.a[2];
  v->A16_d = lora16 + o.a[3];
  v->B16_qkv = lora16 + o.b[0];
  v->B16_o = lora16 + o.b[1];
  v->B16_gu = lora16 + o.b[2];
  v->B16_d = lora16 + o.b[3];
  v->Bs16_qkv = lora16 + o.bs[0];
  v->Bs16_o = lora16 + o.bs[1];
  v->Bs16_gu = lora16 + o.bs[2];
  v->Bs16_d = lora16 + o.bs[3];
  v->At16_qkv = lora16 + o.at[0];
  v->At16_o = lora16 + o.at[1];
  v->At16_gu = lora16 + o.at[2];
  v->At16_d = lora16 + o.at[3];
  return LSQ_OK;
}

int check_layer_args(const lsq_cfg* cfg, const void* blob, const float* lora, const void* x,
                     int batch, int seq, const void* out, LayerShapes* s, const char* who,
                     bool lora_optional = false) {
  LSQ_TRY(layer_shapes(cfg, s));
  if (!blob || (!lora && !lora_optional) || !x || !out)
    return set_error(LSQ_ERR_INVALID, "%s: null pointer", who);
  if (batch <= 0 || seq <= 0) return set_error(LSQ_ERR_SHAPE, "%s: batch and seq must be >= 1", who);
  if (!aligned16(blob) || (lora && !aligned16(lora)) || !aligned16(x) || !aligned16(out))
    return set_error(LSQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned", who);
  return LSQ_OK;
}

// Forward through the SwiGLU product (everything the backward needs) and,
// when x_out is given, the down projection with its residual.
int forward_core(const LayerShapes& s, const Views& v, const float* x, int batch, int seq,
                 const float2* rope_cs, float eps, const Buffers& b, float* x_out,
                 cudaStream_t st, bool have_u = false) {
  const int64_t T = (int64_t)batch * seq;
  const int r = v.lora_on ? s.r : 0;  // r = 0: no LoRA slab in the GEMMs
  const bool down = v.lora_on && !have_u;  // compute u = x A^T here
  LSQ_TRY(launch_rmsnorm_fwd(x, v.g1, T, s.D, eps, b.n1, OUT_F16, b.rstd1, st));
  if (down)
    LSQ_TRY(launch_lora_down16(b.n1, s.D, v.A16_qkv, T, s.D, 3 * r, nullptr, b.u16_qkv,
                               b.lscratch, b.lscratch_bytes, st, b.uh_qkv));
  // A product split over K leaves its partials to the kernel after it (RoPE here,
  // the second RMSNorm after the o projection), which sums them in slice order.
  const float* parts = nullptr;
  int np = 1;
  GemmDesc g_qkv = nf4_fwd(v.codes[0], v.absmax[0], s.qkv_n, s.D, b.n1, T, v.Bs16_qkv, b.uh_qkv,
                           3 * r, nullptr, b.qkv, s.qkv_n);
  g_qkv.parts_out = &parts;
  g_qkv.splits_out = &np;
  LSQ_TRY(gemm_run(g_qkv, b.gemm, b.gemm_bytes, st));
  if (np > 1)
    LSQ_TRY(launch_reduce_rope(parts, np, T, seq, s.H, s.Hkv, s.hd, rope_cs, b.qkv, st));
  else
    LSQ_TRY(launch_rope(b.qkv, T, seq, s.H, s.Hkv, s.hd, rope_cs, st));
  LSQ_TRY(launch_attention_fwd(b.qkv, T, seq, s.H, s.Hkv, s.hd, b.ao, b.lse, st));
  if (down)
    LSQ_TRY(launch_lora_down16(b.ao, s.qd, v.A16_o, T, s.qd, r, nullptr, b.u16_o, b.lscratch,
                               b.lscratch_bytes, st, b.uh_o));
  GemmDesc g_o = nf4_fwd(v.codes[3], v.absmax[3], s.D, s.qd, b.ao, T, v.Bs16_o, b.uh_o, r, x, b.h,
                         s.D);
  g_o.parts_out = &parts;
  g_o.splits_out = &np;
  LSQ_TRY(gemm_run(g_o, b.gemm, b.gemm_bytes, st));
  if (np > 1)
    LSQ_TRY(launch_rmsnorm_fwd_sum(parts, np, x, T, s.D, b.h, v.g2, eps, b.n2, OUT_F16, b.rstd2,
                                   st));
  else
    LSQ_TRY(launch_rmsnorm_fwd(b.h, v.g2, T, s.D, eps, b.n2, OUT_F16, b.rstd2, st));
  if (down)
    LSQ_TRY(launch_lora_down16(b.n2, s.D, v.A16_gu, T, s.D, 2 * r, nullptr, b.u16_gu, b.lscratch,
                               b.lscratch_bytes, st, b.uh_gu));
  LSQ_TRY(gemm_run(nf4_fwd(v.codes[4], v.absmax[4], s.gu_n, s.D, b.n2, T, v.Bs16_gu, b.uh_gu,
                           2 * r, nullptr, b.gu, s.gu_n),
                   b.gemm, b.gemm_bytes, st));
  LSQ_TRY(launch_swiglu_fwd(b.gu, T, s.F, b.m, st));
  if (down)
    LSQ_TRY(launch_lora_down16(b.m, s.F, v.A16_d, T, s.F, r, nullptr, b.u16_d, b.lscratch,
                               b.lscratch_bytes, st, b.uh_d));
  if (x_out)
    LSQ_TRY(gemm_run(nf4_fwd(v.codes[6], v.absmax[6], s.D, s.F, b.m, T, v.Bs16_d, b.uh_d, r, b.h,
                             x_out, s.D),
                     b.gemm, b.gemm_bytes, st));
  return LSQ_OK;
}

}  // namespace

size_t lora16_elems_per_layer(const lsq_cfg* cfg) {
  LayerShapes s;
  if (layer_shapes(cfg, &s) != LSQ_OK) return 0;
  return (size_t)lora16_layout(s).elems;
}

int prepare_lora16(const lsq_cfg* cfg, const float* lora, int n_layers, uint16_t* out,
                   cudaStream_t st) {
  LayerShapes s;
  LSQ_TRY(layer_shapes(cfg, &s));
  lsq_layer_layout L;
  lsq_lora_layout R;
  fill_layout(s, &L, &R);
  const Lora16 o = lora16_layout(s);
  return launch_lora_prepare(lora, R.floats_per_layer, n_layers, out, o.elems,
                             lora16_segs(s, R, o), st);
}

size_t layer_saved_u_bytes(const lsq_cfg* cfg, int64_t T) {
  LayerShapes s;
  if (layer_shapes(cfg, &s) != LSQ_OK || T <= 0) return 0;
  return carve_saved_u(s, T, nullptr, nullptr);
}

size_t layer_ws_bytes(const lsq_cfg* cfg, int64_t T) {
  LayerShapes s;
  if (layer_shapes(cfg, &s) != LSQ_OK || T <= 0) return 0;
  return plan_buffers(s, T, nullptr, nullptr);
}

int layer_fwd_impl(const lsq_cfg* cfg, const void* blob, const float* lora, const float* x_in,
                   int batch, int seq, float* x_out, void* ws, size_t ws_bytes,
                   cudaStream_t st, const float2* rope_cs, const uint16_t* lora16,
                   void* saved_u) {
  LayerShapes s;
  LSQ_TRY(check_layer_args(cfg, blob, lora, x_in, batch, seq, x_out, &s, "decoder_layer_fwd",
                           true));
  const int64_t T = (int64_t)batch * seq;
  const size_t need = plan_buffers(s, T, nullptr, nullptr);
  if (!ws || ws_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "decoder_layer_fwd: workspace %zu < %zu", ws_bytes, need);
  Buffers b;
  plan_buffers(s, T, ws, &b);
  if (saved_u && lora) carve_saved_u(s, T, saved_u, &b);  // u written where the backward finds it
  Views v = views(s, blob, lora);
  LSQ_TRY(attach_lora16(s, lora, lora16, b, &v, st));
  if (!rope_cs) {
    LSQ_TRY(launch_rope_table(seq, s.hd, cfg->rope_theta, b.rope_cs, st));
    rope_cs = b.rope_cs;
  }
  return forward_core(s, v, x_in, batch, seq, rope_cs, cfg->rms_eps, b, x_out, st);
}

int layer_bwd_impl(const lsq_cfg* cfg, const void* blob, const float* lora, const float* x_in,
                   const float* dx_out, const uint16_t* dx_out_bf16, int batch, int seq,
                   float* dx_in, uint16_t* dx_in_bf16, float* lora_grad, int accumulate, void* ws,
                   size_t ws_bytes, cudaStream_t st, const float2* rope_cs,
                   const uint16_t* lora16, const void* saved_u) {
  LayerShapes s;
  LSQ_TRY(check_layer_args(cfg, blob, lora, x_in, batch, seq, dx_in, &s, "decoder_layer_bwd"));
  if (!dx_out || !lora_grad) return set_error(LSQ_ERR_INVALID, "decoder_layer_bwd: null pointer");
  const int64_t T = (int64_t)batch * seq;
  const size_t need = plan_buffers(s, T, nullptr, nullptr);
  if (!ws || ws_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "decoder_layer_bwd: workspace %zu < %zu", ws_bytes, need);
  Buffers b;
  plan_buffers(s, T, ws, &b);
  Views v = views(s, blob, lora);
  LSQ_TRY(attach_lora16(s, lora, lora16, b, &v, st));
  lsq_layer_layout LL;
  lsq_lora_layout RL;
  fill_layout(s, &LL, &RL);
  float* gA_qkv = lora_grad + RL.a_off[0];
  float* gB_qkv = lora_grad + RL.b_off[0];
  float* gA_o = lora_grad + RL.a_off[3];
  float* gB_o = lora_grad + RL.b_off[3];
  float* gA_gu = lora_grad + RL.a_off[4];
  float* gB_gu = lora_grad + RL.b_off[4];
  float* gA_d = lora_grad + RL.a_off[6];
  float* gB_d = lora_grad + RL.b_off[6];
  const int r = s.r;
  const float sc = s.s;
  const int64_t pe3[3] = {s.qd, s.qd + s.kvd, s.qkv_n};
  const int64_t pe2[2] = {s.F, s.gu_n};
  const int64_t pe1[1] = {s.D};

  // recompute the forward from the saved input
  if (!rope_cs) {
    LSQ_TRY(launch_rope_table(seq, s.hd, cfg->rope_theta, b.rope_cs, st));
    rope_cs = b.rope_cs;
  }
  // (the rank-r products u of this layer's forward, when kept, are not recomputed:
  // the same kernels on the same inputs would reproduce them bit for bit)
  if (saved_u) carve_saved_u(s, T, const_cast<void*>(saved_u), &b);
  LSQ_TRY(forward_core(s, v, x_in, batch, seq, rope_cs, cfg->rms_eps, b, nullptr, st,
                       saved_u != nullptr));

  const uint16_t* dout_b = dx_out_bf16;
  if (!dout_b) {
    LSQ_TRY(launch_f32_to_bf16(dx_out, T * s.D, b.dout_b, st));
    dout_b = b.dout_b;
  }
  // down projection
  LSQ_TRY(launch_lora_vproj16(dout_b, T, s.D, v.B16_d, r, nullptr, b.v16_d, b.lscratch,
                              b.lscratch_bytes, st, b.vh_d));
  LSQ_TRY(gemm_run(nf4_dx(v.codes[6], v.absmax[6], s.D, s.F, dout_b, T, v.At16_d, b.vh_d, r, b.dm,
                          1),
                   b.gemm, b.gemm_bytes, st));
  LSQ_TRY(launch_lora_grad_ab16(b.v16_d, b.m, s.F, gA_d, dout_b, b.u16_d, s.D, r, 1, pe1, T, sc,
                                accumulate, gB_d, st));
  // SwiGLU and gate|up
  LSQ_TRY(launch_swiglu_bwd(b.dm, b.gu, T, s.F, b.dgu, st));
  LSQ_TRY(launch_lora_vproj16(b.dgu, T, s.gu_n, v.B16_gu, 2 * r, nullptr, b.v16_gu, b.lscratch,
                              b.lscratch_bytes, st, b.vh_gu));
  // (a product split over K leaves its partials to the RMSNorm backward after it;
  // the rank-r products in between do not use the GEMM workspace)
  const float* parts = nullptr;
  int np = 1;
  GemmDesc g_gu = nf4_dx(v.codes[4], v.absmax[4], s.gu_n, s.D, b.dgu, T, v.At16_gu, b.vh_gu,
                         2 * r, b.dn2, 1);
  g_gu.parts_out = &parts;
  g_gu.splits_out = &np;
  LSQ_TRY(gemm_run(g_gu, b.gemm, b.gemm_bytes, st));
  LSQ_TRY(launch_lora_grad_ab16(b.v16_gu, b.n2, s.D, gA_gu, b.dgu, b.u16_gu, s.gu_n, r, 2, pe2, T,
                                sc, accumulate, gB_gu, st));
  // second RMSNorm + residual
  if (np > 1)
    LSQ_TRY(launch_rmsnorm_bwd_sum(parts, np, b.h, v.g2, b.rstd2, dx_out, T, s.D, b.dh, b.dh_b,
                                   st));
  else
    LSQ_TRY(launch_rmsnorm_bwd(b.dn2, b.h, v.g2, b.rstd2, dx_out, T, s.D, b.dh, b.dh_b, st));
  // o projection
  LSQ_TRY(launch_lora_vproj16(b.dh_b, T, s.D, v.B16_o, r, nullptr, b.v16_o, b.lscratch,
                              b.lscratch_bytes, st, b.vh_o));
  LSQ_TRY(gemm_run(nf4_dx(v.codes[3], v.absmax[3], s.D, s.qd, b.dh_b, T, v.At16_o, b.vh_o, r, b.da,
                          0),
                   b.gemm, b.gemm_bytes, st));
  LSQ_TRY(launch_lora_grad_ab16(b.v16_o, b.ao, s.qd, gA_o, b.dh_b, b.u16_o, s.D, r, 1, pe1, T, sc,
                                accumulate, gB_o, st));
  // attention, RoPE
  LSQ_TRY(launch_attention_bwd(b.qkv, b.ao, b.da, b.lse, T, seq, s.H, s.Hkv, s.hd, b.delta, b.dq,
                               b.dk, b.dv, st));
  LSQ_TRY(launch_rope_grad(b.dq, b.dk, b.dv, T, seq, s.H, s.Hkv, s.hd, rope_cs, b.dqkv, st));
  // q|k|v projections
  LSQ_TRY(launch_lora_vproj16(b.dqkv, T, s.qkv_n, v.B16_qkv, 3 * r, nullptr, b.v16_qkv,
                              b.lscratch, b.lscratch_bytes, st, b.vh_qkv));
  GemmDesc g_qkv = nf4_dx(v.codes[0], v.absmax[0], s.qkv_n, s.D, b.dqkv, T, v.At16_qkv, b.vh_qkv,
                          3 * r, b.dn1, 1);
  g_qkv.parts_out = &parts;
  g_qkv.splits_out = &np;
  LSQ_TRY(gemm_run(g_qkv, b.gemm, b.gemm_bytes, st));
  LSQ_TRY(launch_lora_grad_ab16(b.v16_qkv, b.n1, s.D, gA_qkv, b.dqkv, b.u16_qkv, s.qkv_n, r, 3,
                                pe3, T, sc, accumulate, gB_qkv, st));
  // first RMSNorm + residual
  if (np > 1)
    LSQ_TRY(launch_rmsnorm_bwd_sum(parts, np, x_in, v.g1, b.rstd1, b.dh, T, s.D, dx_in, dx_in_bf16,
                                   st));
  else
    LSQ_TRY(launch_rmsnorm_bwd(b.dn1, x_in, v.g1, b.rstd1, b.dh, T, s.D, dx_in, dx_in_bf16, st));
  return LSQ_OK;
}

}  // namespace lsq

using namespace lsq;

extern "C" int lsq_layer_layout_get(const lsq_cfg* cfg, lsq_layer_layout* out) {
  if (!out) return set_error(LSQ_ERR_INVALID, "lsq_layer_layout_get: null output");
  LayerShapes s;
  LSQ_TRY(layer_shapes(cfg, &s));
  lsq_lora_layout R;
  fill_layout(s, out, &R);
  return LSQ_OK;
}

extern "C" int lsq_lora_layout_get(const lsq_cfg* cfg, lsq_lora_layout* out) {
  if (!out) return set_error(LSQ_ERR_INVALID, "lsq_lora_layout_get: null output");
  LayerShapes s;
  LSQ_TRY(layer_shapes(cfg, &s));
  lsq_layer_layout L;
  fill_layout(s, &L, out);
  return LSQ_OK;
}

extern "C" size_t decoder_layer_workspace_bytes(const lsq_cfg* cfg, int32_t batch, int32_t seq) {
  if (batch <= 0 || seq <= 0) return 0;
  return layer_ws_bytes(cfg, (int64_t)batch * seq);
}

extern "C" int decoder_layer_fwd(const lsq_cfg* cfg, const void* blob, const float* lora,
                                 const float* x_in, int32_t batch, int32_t seq, float* x_out,
                                 void* ws, size_t ws_bytes, void* stream) {
  return layer_fwd_impl(cfg, blob, lora, x_in, batch, seq, x_out, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream));
}

extern "C" int decoder_layer_bwd(const lsq_cfg* cfg, const void* blob, const float* lora,
                                 const float* x_in, const float* dx_out, int32_t batch,
                                 int32_t seq, float* dx_in, float* lora_grad, int32_t accumulate,
                                 void* ws, size_t ws_bytes, void* stream) {
  return layer_bwd_impl(cfg, blob, lora, x_in, dx_out, nullptr, batch, seq, dx_in, nullptr,
                        lora_grad, accumulate, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

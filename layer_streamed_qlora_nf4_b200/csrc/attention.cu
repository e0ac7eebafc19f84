// Causal grouped-query attention, forward and backward, for one layer of the
// Llama-style decoder (the model the Soup layer-streaming tutorial names in
// "維護者的 4GB／8B 成績"): o = softmax(q k^T / sqrt(d), causal) v, with query
// head h reading kv head h / (H / Hkv), positions restarting at 0 per sequence.
//
// Tiles of 64 queries x 64 keys, 4 warps x 16 rows, tensor-core MMAs
// (m16n8k16) with fp32 accumulation and an online (running max / running sum)
// softmax in the exp2 domain.  Precision: q, k, v and o are fp16 (the forward
// activations); the forward and the recomputed scores use fp16 products, with
// the probabilities rounded to fp16 for P V.  The backward's products with a
// gradient operand (dO, dS) are bf16: the fp16 q, k, v fragments are rounded to
// bf16 as they are loaded into registers, and P and dS are rounded to bf16.  The forward saves the row log-sum-exp.  The
// backward recomputes the probabilities from it and is split into a dK/dV
// kernel (one CTA per key block and kv head, summing over that head's query
// heads in a fixed order) and a dQ kernel, so no output is accumulated with
// atomics and every result is deterministic.
#include <math.h>

#include "common.cuh"

namespace lsq {

namespace {

constexpr int kTile = 64;

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 fragment registers -> bf16 (each fp16 value rounded to bf16)
template <int N>
__device__ __forceinline__ void to_bf16(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) r[i] = f16x2_to_bf16x2(r[i]);
}

// Copy `rows` rows (of `D` bf16 each, global row stride ld) into smem rows of
// stride D+8, zero-filling rows >= valid.
template <int D>
__device__ __forceinline__ void load_tile(uint16_t* sm, const uint16_t* g, int64_t ld, int valid) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int i = threadIdx.x; i < kTile * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < valid) v = *reinterpret_cast<const uint4*>(g + (int64_t)r * ld + c * 8);
    *reinterpret_cast<uint4*>(sm + r * (D + 8) + c * 8) = v;
  }
}

// The same with cp.async (16-byte chunks, zero-filled rows >= valid): the copy
// completes at the caller's cp.async wait, so it can overlap the previous tile's math.
template <int D>
__device__ __forceinline__ void load_tile_async(uint16_t* sm, const uint16_t* g, int64_t ld,
                                                int valid) {
  constexpr int CH = D / 8;
  for (int i = threadIdx.x; i < kTile * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    const bool in = r < valid;
    const uint16_t* src = g + (in ? (int64_t)r * ld + c * 8 : 0);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sm + r * (D + 8) + c * 8)),
                 "l"(src), "r"(in ? 16u : 0u)
                 : "memory");
  }
}

// A-operand fragment (16 rows x 16 cols) of a row-major smem tile: rows r0..r0+15, cols c0..
template <int D>
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const uint16_t* sm, int r0, int c0) {
  const int lane = threadIdx.x & 31;
  ldsm_x4(a, smem_u32(sm + (r0 + (lane & 15)) * (D + 8) + c0 + 8 * (lane >> 4)));
}
// B fragments of two n8 tiles where the smem tile rows are the N index and the
// columns the K index (e.g. keys x dims for S = Q K^T): b[0],b[1] -> n rows
// n0..n0+7, b[2],b[3] -> n0+8..n0+15, k cols k0..k0+15.
template <int D>
__device__ __forceinline__ void frag_b_nk(uint32_t (&b)[4], const uint16_t* sm, int n0, int k0) {
  const int lane = threadIdx.x & 31;
  ldsm_x4(b, smem_u32(sm + (n0 + (lane & 7) + 8 * (lane >> 4)) * (D + 8) + k0 + 8 * ((lane >> 3) & 1)));
}
// B fragments of two n8 tiles where the smem tile rows are the K index and the
// columns the N index (e.g. keys x dims for O = P V): k rows k0..k0+15,
// b[0],b[1] -> n cols n0..n0+7, b[2],b[3] -> n0+8..n0+15.
template <int D>
__device__ __forceinline__ void frag_b_kn(uint32_t (&b)[4], const uint16_t* sm, int k0, int n0) {
  const int lane = threadIdx.x & 31;
  ldsm_x4_t(b, smem_u32(sm + (k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * (D + 8) + n0 + 8 * (lane >> 4)));
}

template <int D>
__global__ void __launch_bounds__(128) attn_fwd_kernel(const uint16_t* __restrict__ qkv, int64_t T,
                                                       int seq, int H, int Hkv,
                                                       uint16_t* __restrict__ out,
                                                       float* __restrict__ lse_out, float sl2) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  extern __shared__ __align__(16) uint16_t smem_attn[];
  uint16_t* Qs = smem_attn;
  uint16_t* Kb = Qs + kTile * (D + 8);      // [2] K tiles
  uint16_t* Vb = Kb + 2 * kTile * (D + 8);  // [2] V tiles
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t ld = (int64_t)(H + 2 * Hkv) * D;
  const int64_t tok0 = (int64_t)b * seq;
  const int q0 = qb * kTile;
  load_tile_async<D>(Qs, qkv + (tok0 + q0) * ld + (int64_t)h * D, ld, min(kTile, seq - q0));
  // K/V tile kb goes to buffer kb & 1, one tile ahead of the math
  auto load_kv = [&](int kb) {
    const int k0 = kb * kTile;
    load_tile_async<D>(Kb + (kb & 1) * kTile * (D + 8), qkv + (tok0 + k0) * ld + (int64_t)(H + g) * D,
                       ld, min(kTile, seq - k0));
    load_tile_async<D>(Vb + (kb & 1) * kTile * (D + 8),
                       qkv + (tok0 + k0) * ld + (int64_t)(H + Hkv + g) * D, ld, min(kTile, seq - k0));
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  load_kv(0);

  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const int qrow[2] = {q0 + warp * 16 + gid, q0 + warp * 16 + gid + 8};

  for (int kb = 0; kb <= qb; ++kb) {
    const int k0 = kb * kTile;
    if (kb < qb) {
      load_kv(kb + 1);  // its buffer was last read before the previous iteration's end barrier
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();  // tile kb (and Q) visible to every warp
    const uint16_t* Ks = Kb + (kb & 1) * kTile * (D + 8);
    const uint16_t* Vs = Vb + (kb & 1) * kTile * (D + 8);
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4];
      frag_a<D>(a, Qs, warp * 16, kk * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t bb[4];
        frag_b_nk<D>(bb, Ks, j * 16, kk * 16);
        mma16816_f16(s[2 * j], a, bb[0], bb[1]);
        mma16816_f16(s[2 * j + 1], a, bb[2], bb[3]);
      }
    }
    // scale into the log2 domain, mask, row max
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + 8 * j + 2 * tig + (e & 1);
        const int qr = qrow[e >> 1];
        float v = s[j][e] * sl2;
        if (key > qr || key >= seq) v = -INFINITY;
        s[j][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float corr[2];
#pragma unroll
    for (int rI = 0; rI < 2; ++rI) {
      mx[rI] = fmaxf(mx[rI], __shfl_xor_sync(0xFFFFFFFFu, mx[rI], 1));
      mx[rI] = fmaxf(mx[rI], __shfl_xor_sync(0xFFFFFFFFu, mx[rI], 2));
      const float m_new = fmaxf(m_run[rI], mx[rI]);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      corr[rI] = exp2f(m_run[rI] - m_use);
      m_run[rI] = m_new;
      mx[rI] = m_use;
    }
    float rs[2] = {0.f, 0.f};
    uint32_t pa[4][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = exp2f(s[j][0] - mx[0]), p1 = exp2f(s[j][1] - mx[0]);
      const float p2 = exp2f(s[j][2] - mx[1]), p3 = exp2f(s[j][3] - mx[1]);
      rs[0] += p0 + p1;
      rs[1] += p2 + p3;
      pa[j >> 1][(j & 1) * 2 + 0] = pack_f16x2(p0, p1);
      pa[j >> 1][(j & 1) * 2 + 1] = pack_f16x2(p2, p3);
    }
#pragma unroll
    for (int rI = 0; rI < 2; ++rI) {
      rs[rI] += __shfl_xor_sync(0xFFFFFFFFu, rs[rI], 1);
      rs[rI] += __shfl_xor_sync(0xFFFFFFFFu, rs[rI], 2);
      l_run[rI] = l_run[rI] * corr[rI] + rs[rI];
    }
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= corr[0];
      o[j][1] *= corr[0];
      o[j][2] *= corr[1];
      o[j][3] *= corr[1];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // A fragment of P for keys 16i..16i+15: (row g, k 2t), (row g+8, k 2t), (row g, k 8+2t), (row g+8, k 8+2t)
      const uint32_t a[4] = {pa[i][0], pa[i][1], pa[i][2], pa[i][3]};
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        uint32_t bb[4];
        frag_b_kn<D>(bb, Vs, i * 16, j * 16);
        mma16816_f16(o[2 * j], a, bb[0], bb[1]);
        mma16816_f16(o[2 * j + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();  // every warp is done with buffer kb & 1 before it is refilled
  }
  // finalize
#pragma unroll
  for (int rI = 0; rI < 2; ++rI) {
    const int qr = qrow[rI];
    if (qr >= seq) continue;
    const float inv = 1.f / l_run[rI];
    uint16_t* orow = out + (tok0 + qr) * (int64_t)H * D + (int64_t)h * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const int col = 8 * j + 2 * tig;
      *reinterpret_cast<uint32_t*>(orow + col) =
          pack_f16x2(o[j][2 * rI] * inv, o[j][2 * rI + 1] * inv);
    }
    if (tig == 0)
      lse_out[(int64_t)h * T + tok0 + qr] = (m_run[rI] + log2f(l_run[rI])) * 0.69314718055994531f;
  }
}

// delta[h, t] = sum_d dO[t, h, d] * O[t, h, d]  (O fp16, dO bf16)
template <int D>
__global__ void attn_delta_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                  int64_t T, int H, float* __restrict__ delta) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= T * H) return;
  const int64_t t = wid / H;
  const int h = (int)(wid % H);
  const uint16_t* a = o + t * (int64_t)H * D + (int64_t)h * D;
  const uint16_t* c = dout + t * (int64_t)H * D + (int64_t)h * D;
  float acc = 0.f;
  for (int i = lane * 2; i < D; i += 64) {
    const float2 x = unpack_f16x2(*reinterpret_cast<const uint32_t*>(a + i));
    const float2 y = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(c + i));
    acc += x.x * y.x + x.y * y.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (lane == 0) delta[(int64_t)h * T + t] = acc;
}

// dK, dV contributions of one query head for one key block (written per query
// head; the sum over a kv head's query heads happens later, in a fixed order).
template <int D>
__global__ void __launch_bounds__(128) attn_bwd_dkdv_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, int64_t T, int seq, int H,
    int Hkv, float sl2, float scale, float* __restrict__ dk, float* __restrict__ dv) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  extern __shared__ __align__(16) uint16_t smem_attn[];
  uint16_t* Ks = smem_attn;
  uint16_t* Vs = Ks + kTile * (D + 8);
  uint16_t* Qb = Vs + kTile * (D + 8);       // [2] Q tiles
  uint16_t* dOb = Qb + 2 * kTile * (D + 8);  // [2] dO tiles
  float* lse_b = reinterpret_cast<float*>(dOb + 2 * kTile * (D + 8));  // [2][kTile]
  float* del_b = lse_b + 2 * kTile;                                      // [2][kTile]
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t ld = (int64_t)(H + 2 * Hkv) * D;
  const int64_t ldo = (int64_t)H * D;
  const int64_t tok0 = (int64_t)b * seq;
  const int k0 = kb * kTile;
  load_tile<D>(Ks, qkv + (tok0 + k0) * ld + (int64_t)(H + g) * D, ld, min(kTile, seq - k0));
  load_tile<D>(Vs, qkv + (tok0 + k0) * ld + (int64_t)(H + Hkv + g) * D, ld, min(kTile, seq - k0));
  float dkacc[D / 8][4], dvacc[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) dkacc[j][e] = dvacc[j][e] = 0.f;
  const int krow[2] = {k0 + warp * 16 + gid, k0 + warp * 16 + gid + 8};
  const int nqb = (seq + kTile - 1) / kTile;
  // the Q / dO tiles (and their lse, delta rows) of query block qb go to buffer
  // (qb - kb) & 1, one block ahead of the math
  auto load_q = [&](int qb) {
    const int q0 = qb * kTile, sl = (qb - kb) & 1;
    load_tile_async<D>(Qb + sl * kTile * (D + 8), qkv + (tok0 + q0) * ld + (int64_t)h * D, ld,
                       min(kTile, seq - q0));
    load_tile_async<D>(dOb + sl * kTile * (D + 8), dout + (tok0 + q0) * ldo + (int64_t)h * D, ldo,
                       min(kTile, seq - q0));
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int i = threadIdx.x; i < kTile; i += blockDim.x) {
      const bool ok = q0 + i < seq;
      lse_b[sl * kTile + i] = ok ? lse[(int64_t)h * T + tok0 + q0 + i] * 1.4426950408889634f : 0.f;
      del_b[sl * kTile + i] = ok ? delta[(int64_t)h * T + tok0 + q0 + i] : 0.f;
    }
  };
  load_q(kb);
  {
    for (int qb = kb; qb < nqb; ++qb) {
      const int q0 = qb * kTile;
      if (qb + 1 < nqb) {
        load_q(qb + 1);  // its buffers were last read before the previous iteration's end barrier
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();  // block qb (and K, V) visible to every warp
      const int sl = (qb - kb) & 1;
      const uint16_t* Qs = Qb + sl * kTile * (D + 8);
      const uint16_t* dOs = dOb + sl * kTile * (D + 8);
      const float* lse_s = lse_b + sl * kTile;
      const float* del_s = del_b + sl * kTile;
      // S^T = K Q^T  (16 keys of this warp x 64 queries)
      float st[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) st[j][0] = st[j][1] = st[j][2] = st[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a<D>(a, Ks, warp * 16, kk * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t bb[4];
          frag_b_nk<D>(bb, Qs, j * 16, kk * 16);
          mma16816_f16(st[2 * j], a, bb[0], bb[1]);
          mma16816_f16(st[2 * j + 1], a, bb[2], bb[3]);
        }
      }
      // P^T
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qi = 8 * j + 2 * tig + (e & 1);
          const int q = q0 + qi;
          const int kr = krow[e >> 1];
          st[j][e] = (q < kr || q >= seq || kr >= seq) ? 0.f : exp2f(st[j][e] * sl2 - lse_s[qi]);
        }
      // dV += P^T dO
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t a[4] = {pack_bf16x2(st[2 * i][0], st[2 * i][1]),
                               pack_bf16x2(st[2 * i][2], st[2 * i][3]),
                               pack_bf16x2(st[2 * i + 1][0], st[2 * i + 1][1]),
                               pack_bf16x2(st[2 * i + 1][2], st[2 * i + 1][3])};
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          uint32_t bb[4];
          frag_b_kn<D>(bb, dOs, i * 16, j * 16);
          mma16816(dvacc[2 * j], a, bb[0], bb[1]);
          mma16816(dvacc[2 * j + 1], a, bb[2], bb[3]);
        }
      }
      // dP^T = V dO^T
      float dp[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) dp[j][0] = dp[j][1] = dp[j][2] = dp[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a<D>(a, Vs, warp * 16, kk * 16);
        to_bf16(a);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t bb[4];
          frag_b_nk<D>(bb, dOs, j * 16, kk * 16);
          mma16816(dp[2 * j], a, bb[0], bb[1]);
          mma16816(dp[2 * j + 1], a, bb[2], bb[3]);
        }
      }
      // dS^T = P^T (dP^T - delta), then dK += dS^T Q
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qi = 8 * j + 2 * tig + (e & 1);
          st[j][e] = st[j][e] * (dp[j][e] - del_s[qi]);
        }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t a[4] = {pack_bf16x2(st[2 * i][0], st[2 * i][1]),
                               pack_bf16x2(st[2 * i][2], st[2 * i][3]),
                               pack_bf16x2(st[2 * i + 1][0], st[2 * i + 1][1]),
                               pack_bf16x2(st[2 * i + 1][2], st[2 * i + 1][3])};
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          uint32_t bb[4];
          frag_b_kn<D>(bb, Qs, i * 16, j * 16);
          to_bf16(bb);
          mma16816(dkacc[2 * j], a, bb[0], bb[1]);
          mma16816(dkacc[2 * j + 1], a, bb[2], bb[3]);
        }
      }
      __syncthreads();  // every warp is done with buffer (qb - kb) & 1 before it is refilled
    }
  }
#pragma unroll
  for (int rI = 0; rI < 2; ++rI) {
    const int kr = krow[rI];
    if (kr >= seq) continue;
    float* dkr = dk + (tok0 + kr) * (int64_t)H * D + (int64_t)h * D;
    float* dvr = dv + (tok0 + kr) * (int64_t)H * D + (int64_t)h * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const int col = 8 * j + 2 * tig;
      *reinterpret_cast<float2*>(dkr + col) =
          make_float2(dkacc[j][2 * rI] * scale, dkacc[j][2 * rI + 1] * scale);
      *reinterpret_cast<float2*>(dvr + col) = make_float2(dvacc[j][2 * rI], dvacc[j][2 * rI + 1]);
    }
  }
}

// dQ for one query block of one query head.
template <int D>
__global__ void __launch_bounds__(128) attn_bwd_dq_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, int64_t T, int seq, int H,
    int Hkv, float sl2, float scale, float* __restrict__ dq) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  extern __shared__ __align__(16) uint16_t smem_attn[];
  uint16_t* Qs = smem_attn;
  uint16_t* dOs = Qs + kTile * (D + 8);
  uint16_t* Kb = dOs + kTile * (D + 8);     // [2] K tiles
  uint16_t* Vb = Kb + 2 * kTile * (D + 8);  // [2] V tiles
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t ld = (int64_t)(H + 2 * Hkv) * D;
  const int64_t ldo = (int64_t)H * D;
  const int64_t tok0 = (int64_t)b * seq;
  const int q0 = qb * kTile;
  load_tile<D>(Qs, qkv + (tok0 + q0) * ld + (int64_t)h * D, ld, min(kTile, seq - q0));
  load_tile<D>(dOs, dout + (tok0 + q0) * ldo + (int64_t)h * D, ldo, min(kTile, seq - q0));
  const int qrow[2] = {q0 + warp * 16 + gid, q0 + warp * 16 + gid + 8};
  float lse2[2], del[2];
#pragma unroll
  for (int rI = 0; rI < 2; ++rI) {
    const bool ok = qrow[rI] < seq;
    lse2[rI] = ok ? lse[(int64_t)h * T + tok0 + qrow[rI]] * 1.4426950408889634f : 0.f;
    del[rI] = ok ? delta[(int64_t)h * T + tok0 + qrow[rI]] : 0.f;
  }
  float dqacc[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) dqacc[j][0] = dqacc[j][1] = dqacc[j][2] = dqacc[j][3] = 0.f;
  // K/V tile kb goes to buffer kb & 1, one tile ahead of the math
  auto load_kv = [&](int kb) {
    const int k0 = kb * kTile;
    load_tile_async<D>(Kb + (kb & 1) * kTile * (D + 8), qkv + (tok0 + k0) * ld + (int64_t)(H + g) * D,
                       ld, min(kTile, seq - k0));
    load_tile_async<D>(Vb + (kb & 1) * kTile * (D + 8),
                       qkv + (tok0 + k0) * ld + (int64_t)(H + Hkv + g) * D, ld, min(kTile, seq - k0));
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  load_kv(0);
  for (int kb = 0; kb <= qb; ++kb) {
    const int k0 = kb * kTile;
    if (kb < qb) {
      load_kv(kb + 1);  // its buffer was last read before the previous iteration's end barrier
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();  // tile kb (and Q, dO) visible to every warp
    const uint16_t* Ks = Kb + (kb & 1) * kTile * (D + 8);
    const uint16_t* Vs = Vb + (kb & 1) * kTile * (D + 8);
    float s[8][4], dp[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[j][e] = dp[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4], ad[4];
      frag_a<D>(a, Qs, warp * 16, kk * 16);
      frag_a<D>(ad, dOs, warp * 16, kk * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t bb[4], bv[4];
        frag_b_nk<D>(bb, Ks, j * 16, kk * 16);
        frag_b_nk<D>(bv, Vs, j * 16, kk * 16);
        to_bf16(bv);
        mma16816_f16(s[2 * j], a, bb[0], bb[1]);
        mma16816_f16(s[2 * j + 1], a, bb[2], bb[3]);
        mma16816(dp[2 * j], ad, bv[0], bv[1]);
        mma16816(dp[2 * j + 1], ad, bv[2], bv[3]);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + 8 * j + 2 * tig + (e & 1);
        const int qr = qrow[e >> 1];
        const float p = (key > qr || key >= seq || qr >= seq)
                            ? 0.f
                            : exp2f(s[j][e] * sl2 - lse2[e >> 1]);
        s[j][e] = p * (dp[j][e] - del[e >> 1]);
      }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a[4] = {pack_bf16x2(s[2 * i][0], s[2 * i][1]),
                             pack_bf16x2(s[2 * i][2], s[2 * i][3]),
                             pack_bf16x2(s[2 * i + 1][0], s[2 * i + 1][1]),
                             pack_bf16x2(s[2 * i + 1][2], s[2 * i + 1][3])};
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        uint32_t bb[4];
        frag_b_kn<D>(bb, Ks, i * 16, j * 16);
        to_bf16(bb);
        mma16816(dqacc[2 * j], a, bb[0], bb[1]);
        mma16816(dqacc[2 * j + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();  // every warp is done with buffer kb & 1 before it is refilled
  }
#pragma unroll
  for (int rI = 0; rI < 2; ++rI) {
    const int qr = qrow[rI];
    if (qr >= seq) continue;
    float* dqr = dq + (tok0 + qr) * (int64_t)H * D + (int64_t)h * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const int col = 8 * j + 2 * tig;
      *reinterpret_cast<float2*>(dqr + col) =
          make_float2(dqacc[j][2 * rI] * scale, dqacc[j][2 * rI + 1] * scale);
    }
  }
}

template <int D>
int attn_fwd_t(const uint16_t* qkv, int64_t T, int seq, int H, int Hkv, uint16_t* o, float* lse,
               cudaStream_t st) {
  const size_t smem = 5 * kTile * (D + 8) * sizeof(uint16_t);  // Q + two K + two V tiles
  static bool attr = false;
  if (!attr) {
    LSQ_CUDA(cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem));
    attr = true;
  }
  const int batch = (int)(T / seq);
  dim3 grid((seq + kTile - 1) / kTile, H, batch);
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);
  attn_fwd_kernel<D><<<grid, 128, smem, st>>>(qkv, T, seq, H, Hkv, o, lse, sl2);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

template <int D>
int attn_bwd_t(const uint16_t* qkv, const uint16_t* o, const uint16_t* dout, const float* lse,
               int64_t T, int seq, int H, int Hkv, float* delta, float* dq, float* dk, float* dv,
               cudaStream_t st) {
  const size_t s_kv = 6 * kTile * (D + 8) * sizeof(uint16_t) + 4 * kTile * sizeof(float);
  const size_t s_q = 6 * kTile * (D + 8) * sizeof(uint16_t);
  static bool attr = false;
  if (!attr) {
    LSQ_CUDA(cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_kv));
    LSQ_CUDA(cudaFuncSetAttribute(attn_bwd_dq_kernel<D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_q));
    attr = true;
  }
  const int batch = (int)(T / seq);
  const float scale = 1.f / sqrtf((float)D);
  const float sl2 = 1.4426950408889634f * scale;
  const int64_t nw = T * H;
  attn_delta_kernel<D><<<(unsigned)((nw * 32 + 255) / 256), 256, 0, st>>>(o, dout, T, H, delta);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  dim3 gkv((seq + kTile - 1) / kTile, H, batch);
  attn_bwd_dkdv_kernel<D><<<gkv, 128, s_kv, st>>>(qkv, dout, lse, delta, T, seq, H, Hkv, sl2, scale,
                                                  dk, dv);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  dim3 gq((seq + kTile - 1) / kTile, H, batch);
  attn_bwd_dq_kernel<D><<<gq, 128, s_q, st>>>(qkv, dout, lse, delta, T, seq, H, Hkv, sl2, scale, dq);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

}  // namespace

int launch_attention_fwd(const uint16_t* qkv, int64_t T, int seq, int H, int Hkv, int d,
                         uint16_t* o, float* lse, cudaStream_t st) {
  if (seq <= 0 || T % seq != 0 || H % Hkv != 0)
    return set_error(LSQ_ERR_SHAPE, "attention: bad batch/seq/head shape");
  if (d != 128 && d != 64) return set_error(LSQ_ERR_SHAPE, "attention: head_dim must be 64 or 128");
  const int prof = prof_begin(st);
  LSQ_TRY(d == 128 ? attn_fwd_t<128>(qkv, T, seq, H, Hkv, o, lse, st)
                   : attn_fwd_t<64>(qkv, T, seq, H, Hkv, o, lse, st));
  // causal: 2 GEMMs of d per (query, key<=query) pair and head
  const double pairs = (double)(T / seq) * (double)seq * (seq + 1) / 2.0;
  prof_end(prof, st, "attention_fwd", 4.0 * H * d * pairs,
           2.0 * T * (double)(H + 2 * Hkv) * d + 2.0 * T * H * d);
  return LSQ_OK;
}

int launch_attention_bwd(const uint16_t* qkv, const uint16_t* o, const uint16_t* dout,
                         const float* lse, int64_t T, int seq, int H, int Hkv, int d, float* delta,
                         float* dq, float* dk, float* dv, cudaStream_t st) {
  if (seq <= 0 || T % seq != 0 || H % Hkv != 0)
    return set_error(LSQ_ERR_SHAPE, "attention: bad batch/seq/head shape");
  if (d != 128 && d != 64) return set_error(LSQ_ERR_SHAPE, "attention: head_dim must be 64 or 128");
  const int prof = prof_begin(st);
  LSQ_TRY(d == 128 ? attn_bwd_t<128>(qkv, o, dout, lse, T, seq, H, Hkv, delta, dq, dk, dv, st)
                   : attn_bwd_t<64>(qkv, o, dout, lse, T, seq, H, Hkv, delta, dq, dk, dv, st));
  // five causal GEMMs (S, dP, dV, dK, dQ) = 2.5x the forward's two
  const double pairs = (double)(T / seq) * (double)seq * (seq + 1) / 2.0;
  prof_end(prof, st, "attention_bwd", 10.0 * H * d * pairs,
           2.0 * T * (double)(H + 2 * Hkv) * d + 6.0 * T * H * d + 4.0 * T * (H + 2 * Hkv) * d);
  return LSQ_OK;
}

}  // namespace lsq

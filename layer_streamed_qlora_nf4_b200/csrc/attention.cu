// Causal grouped-query attention, forward and backward, for one layer of the
// Llama-style decoder (the model the Soup layer-streaming tutorial names in
// "維護者的 4GB／8B 成績"): o = softmax(q k^T / sqrt(d), causal) v, with query
// head h reading kv head h / (H / Hkv), positions restarting at 0 per sequence.
//
// Forward: 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM, TMA
// tiles of 128 queries x 128 keys), see attn_fwd_tc_kernel.  Backward: tiles of
// 64 queries x 64 keys, 4 warps x 16 rows, m16n8k16 tensor-core MMAs with fp32
// accumulation.  Both use an online (running max / running sum) softmax in the
// exp2 domain.  Precision: q, k, v and o are fp16 (the forward activations);
// the forward and the recomputed scores use fp16 products, with the
// probabilities rounded to fp16 for P V.  The backward's products with a
// gradient operand (dO, dS) are bf16: the fp16 q, k, v fragments are rounded to
// bf16 as they are loaded into registers, and P and dS are rounded to bf16.  The
// forward saves the row log-sum-exp.  The backward recomputes the probabilities
// from it and is split into a dK/dV kernel (one CTA per key block and kv head,
// summing over that head's query heads in a fixed order) and a dQ kernel, so no
// output is accumulated with atomics and every result is deterministic.
#include <cuda.h>
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

// ------------------------------------------------------------------ forward on tcgen05
// One CTA per (128 queries of one sequence, query head).  Q and the K/V tiles of
// 128 keys arrive by TMA in the 128-byte-swizzle layout; S = Q K^T is computed by
// tcgen05.mma into one of two TMEM buffers (so the next tile's scores overlap
// the softmax of this one); the softmax warps (one query row per thread) read S
// from TMEM, write P = exp2(s - m) as fp16 into shared memory, and O += P V
// accumulates in TMEM (V is the MN-major B operand).  The reference maximum m
// of a row moves only when a tile's maximum exceeds it by more than 2^8 (then O
// and the running sum are rescaled): the result is exact for any reference, and
// P stays below 2^8, well inside fp16.
//   warps 0-7: softmax and epilogue; warp w and w + 4 share TMEM lane quarter
//              w % 4 (query rows 32 (w % 4) ..), w / 4 selects the half of the
//              128 keys (and of O's columns) a thread handles for its row
//   warp 8   : TMA producer (Q once, then K and V into two buffers)
//   warp 9   : TMEM allocation and the MMA issuer (lane 0)
constexpr int kAQ = 128;   // queries per CTA (UMMA M)
constexpr int kAK = 128;   // keys per tile (UMMA N of S, K of P V)
constexpr int kAThreads = 320;
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr float kRescaleLog2 = 8.f;

template <int D>
struct AttnSmem {
  static constexpr int DA = D / 64;                   // 64-element swizzle atoms along d
  static constexpr uint32_t kQ = kAQ * D * 2;         // Q: DA boxes of [128 rows x 64]
  static constexpr uint32_t kKV = kAK * D * 2;        // one K or V tile
  static constexpr uint32_t kP = kAQ * kAK * 2;       // P: 2 atoms of [128 rows x 64 keys]
  static constexpr uint32_t kBytes = 1024 + kQ + 4 * kKV + kP;  // Q, 2 x (K, V), P
};

__device__ __forceinline__ uint8_t* align1024_a(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D>
__global__ void __launch_bounds__(kAThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, int64_t T, int seq, int H,
                       int Hkv, uint16_t* __restrict__ out, float* __restrict__ lse_out, float sl2,
                       int* __restrict__ dev_err) {
  using SM = AttnSmem<D>;
  constexpr int DA = SM::DA;
  extern __shared__ uint8_t attn_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_kv[2], bar_kv_free[2], bar_s[2], bar_s_free[2];
  __shared__ __align__(8) uint64_t bar_p, bar_pv;
  __shared__ __align__(8) uint64_t bar_sm;  // the eight softmax warps meet here
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  __shared__ float xch[2][kAQ];  // the two halves of a row exchange its maximum, then its sum
  volatile int* abort_flag = &abort_sh;
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run

  uint8_t* Qs = align1024_a(attn_raw);
  uint8_t* Ks = Qs + SM::kQ;            // [2] K tiles
  uint8_t* Vs = Ks + 2 * SM::kKV;       // [2] V tiles
  uint8_t* Ps = Vs + 2 * SM::kKV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int q0 = qb * kAQ;                        // first query position of the block
  const int64_t tok0 = (int64_t)b * seq;
  const int kv_end = min(seq, q0 + kAQ);          // keys this block can attend to
  const int n_kv = (kv_end + kAK - 1) / kAK;
  constexpr uint32_t kColS = 0, kColO = 2 * kAK;  // TMEM: S buffers at 0 and 128, O at 256

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar_q), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_kv[i]), 1);
      mbar_init(smem_u32(&bar_kv_free[i]), 1);
      mbar_init(smem_u32(&bar_s[i]), 1);
      mbar_init(smem_u32(&bar_s_free[i]), 8);
    }
    mbar_init(smem_u32(&bar_p), 8);
    mbar_init(smem_u32(&bar_pv), 1);
    mbar_init(smem_u32(&bar_sm), 8);
    abort_sh = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&tmem_sh), 512);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) tma_prefetch_desc(&tm_qkv);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;

  if (warp == kWarpTma) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      pdl_wait();  // q, k, v come from the kernel before
      mbar_arrive_expect_tx(smem_u32(&bar_q), SM::kQ);
      for (int a = 0; a < DA; ++a)
        tma_load_2d(smem_u32(Qs + a * kAQ * 128), &tm_qkv, smem_u32(&bar_q), h * D + 64 * a,
                    (int)(tok0 + q0));
      for (int j = 0; j < n_kv; ++j) {
        const int buf = j & 1;
        if (j >= 2 && !mbar_wait_bounded(smem_u32(&bar_kv_free[buf]), (uint32_t)(((j - 2) >> 1) & 1),
                                         abort_flag, dev_err, DEV_ERR_WAIT_GEMM))
          break;
        const uint32_t fb = smem_u32(&bar_kv[buf]);
        mbar_arrive_expect_tx(fb, 2 * SM::kKV);
        for (int a = 0; a < DA; ++a) {
          tma_load_2d(smem_u32(Ks + buf * SM::kKV + a * kAK * 128), &tm_qkv, fb,
                      (H + g) * D + 64 * a, (int)(tok0 + j * kAK));
          tma_load_2d(smem_u32(Vs + buf * SM::kKV + a * kAK * 128), &tm_qkv, fb,
                      (H + Hkv + g) * D + 64 * a, (int)(tok0 + j * kAK));
        }
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_f16(kAQ, kAK);
      const uint32_t idesc_o = umma_idesc_f16(kAQ, D) | (1u << 16);  // B (V) MN-major
      bool ok = mbar_wait_bounded(smem_u32(&bar_q), 0u, abort_flag, dev_err, DEV_ERR_WAIT_GEMM);
      auto issue_s = [&](int j) -> bool {
        const int buf = j & 1;
        if (!mbar_wait_bounded(smem_u32(&bar_kv[buf]), (uint32_t)((j >> 1) & 1), abort_flag,
                               dev_err, DEV_ERR_WAIT_GEMM))
          return false;
        if (j >= 2 && !mbar_wait_bounded(smem_u32(&bar_s_free[buf]), (uint32_t)(((j - 2) >> 1) & 1),
                                         abort_flag, dev_err, DEV_ERR_WAIT_GEMM))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kAQ * 128 + (kk & 3) * 32);
          const uint64_t ad = umma_desc_k_sw128(smem_u32(Qs) + off);
          const uint64_t bd = umma_desc_k_sw128(smem_u32(Ks + buf * SM::kKV) + off);
          tc_mma_bf16(tmem + kColS + (uint32_t)buf * kAK, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&bar_s[buf]));
        return true;
      };
      ok = ok && issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int buf = j & 1;
        if (j + 1 < n_kv) ok = issue_s(j + 1);
        if (!ok) break;
        // P_j written (and O rescaled if its reference maximum moved)
        ok = mbar_wait_bounded(smem_u32(&bar_p), (uint32_t)(j & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kAK / 16; ++kk) {
          const uint64_t ad = umma_desc_k_sw128(smem_u32(Ps) + (uint32_t)((kk >> 2) * kAQ * 128 +
                                                                          (kk & 3) * 32));
          const uint64_t bd = umma_desc_mn_sw128(smem_u32(Vs + buf * SM::kKV) + (uint32_t)kk * 16 * 128,
                                                 (uint32_t)(kAK * 128), 1024u);
          tc_mma_bf16(tmem + kColO, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&bar_pv));           // P free, O updated
        tc_commit(smem_u32(&bar_kv_free[buf]));  // K_j and V_j read
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax (warps 0-7)
    const int r = (warp & 3) * 32 + lane;  // query row of the block = TMEM lane
    const int hf = warp >> 2;               // half: keys (and O columns) 64 hf ..
    const int q = q0 + r;                   // the row's position in the sequence
    const int kmax = min(q, seq - 1);       // its last key
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    constexpr int KH = kAK / 2, DH = D / 2;  // keys and O columns per half
    float m_ref = -INFINITY, l_run = 0.f;    // l_run: this half's share of the row sum
    bool ok = true;
    // the eight softmax warps meet at a bounded barrier (one arrival per warp),
    // so that an abort in one of them cannot strand the others
    int sm_phase = 0;
    auto sm_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_sm));
      const bool rr = mbar_wait_bounded(smem_u32(&bar_sm), (uint32_t)(sm_phase & 1), abort_flag,
                                        dev_err, DEV_ERR_WAIT_GEMM);
      ++sm_phase;
      return __all_sync(0xFFFFFFFFu, rr);
    };
    for (int j = 0; j < n_kv && ok; ++j) {
      const int buf = j & 1;
      ok = mbar_wait_bounded(smem_u32(&bar_s[buf]), (uint32_t)((j >> 1) & 1), abort_flag, dev_err,
                             DEV_ERR_WAIT_GEMM);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      const int k0 = j * kAK + hf * KH;  // first key of this half
      const bool full = k0 + KH - 1 <= kmax;  // no key of this half is masked for the row
      // this half of the row's scores, all loads in flight at once
      uint32_t sv[KH / 16][16];
#pragma unroll
      for (int c = 0; c < KH / 16; ++c)
        tmem_ld16(trow + kColS + (uint32_t)buf * kAK + (uint32_t)(hf * KH + 16 * c), sv[c]);
      tmem_ld_wait();
      float mt = -INFINITY;
      if (full) {
#pragma unroll
        for (int c = 0; c < KH / 16; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e) mt = fmaxf(mt, __uint_as_float(sv[c][e]));
      } else {
#pragma unroll
        for (int c = 0; c < KH / 16; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            if (k0 + 16 * c + e > kmax) sv[c][e] = __float_as_uint(-INFINITY);
            mt = fmaxf(mt, __uint_as_float(sv[c][e]));
          }
      }
      // the row's maximum over both halves, in the log2 domain
      xch[hf][r] = mt;
      ok = sm_sync();
      mt = fmaxf(mt, xch[hf ^ 1][r]) * sl2;
      ok = sm_sync() && ok;  // xch is free again
      if (!ok) break;
      float corr = 1.f;
      bool moved = false;
      if (j == 0) {
        m_ref = mt;
      } else if (mt > m_ref + kRescaleLog2) {
        corr = exp2f(m_ref - mt);
        m_ref = mt;
        l_run *= corr;
        moved = true;
      }
      // the previous P V has read P and written O
      if (j > 0) {
        ok = mbar_wait_bounded(smem_u32(&bar_pv), (uint32_t)((j - 1) & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xFFFFFFFFu, moved)) {
#pragma unroll 1
        for (int c = 0; c < DH / 16; ++c) {
          uint32_t v[16];
          tmem_ld16(trow + kColO + (uint32_t)(hf * DH + 16 * c), v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
          tmem_st16(trow + kColO + (uint32_t)(hf * DH + 16 * c), v);
        }
        tmem_st_wait();
      }
      // P = exp2(s sl2 - m_ref) in fp16 into this half's 64-key atom of the P
      // tile (masked scores are -inf, so their p is 0), and this half's row sum
      const float nm = -m_ref;
      float rs = 0.f;
      uint8_t* atom = Ps + hf * kAQ * 128;
#pragma unroll
      for (int c = 0; c < KH / 16; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float p0 = exp2f(fmaf(__uint_as_float(sv[c][e]), sl2, nm));
          const float p1 = exp2f(fmaf(__uint_as_float(sv[c][e + 1]), sl2, nm));
          rs += p0 + p1;
          pk[e >> 1] = pack_f16x2(p0, p1);
        }
        *reinterpret_cast<uint4*>(atom + sw128_offset((uint32_t)r, (uint32_t)(2 * c))) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(atom + sw128_offset((uint32_t)r, (uint32_t)(2 * c + 1))) =
            make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      l_run += rs;
      fence_proxy_async_smem();  // P visible to the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bar_s_free[buf]));
        mbar_arrive(smem_u32(&bar_p));
      }
    }
    // ---------------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait_bounded(smem_u32(&bar_pv), (uint32_t)((n_kv - 1) & 1), abort_flag,
                                   dev_err, DEV_ERR_WAIT_GEMM);
    ok = __all_sync(0xFFFFFFFFu, ok);
    // the row sum over both halves (every softmax thread reaches the barrier)
    xch[hf][r] = l_run;
    ok = sm_sync() && ok;
    const float l_row = l_run + xch[hf ^ 1][r];
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l_row;
      const bool live = q < seq;
      uint16_t* orow = out + (tok0 + q) * (int64_t)H * D + (int64_t)h * D + hf * DH;
      uint32_t ov[DH / 16][16];
#pragma unroll
      for (int c = 0; c < DH / 16; ++c) tmem_ld16(trow + kColO + (uint32_t)(hf * DH + 16 * c), ov[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < DH / 16; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2)
          pk[e >> 1] =
              pack_f16x2(__uint_as_float(ov[c][e]) * inv, __uint_as_float(ov[c][e + 1]) * inv);
        if (live) {
          *reinterpret_cast<uint4*>(orow + 16 * c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(orow + 16 * c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (live && hf == 0)
        lse_out[(int64_t)h * T + tok0 + q] = (m_ref + log2f(l_row)) * 0.69314718055994531f;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (abort_sh) settle_ns(2000000);  // let issued copies and MMAs land before freeing TMEM
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  using SM = AttnSmem<D>;
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr[dev]) {
    LSQ_CUDA(cudaFuncSetAttribute(attn_fwd_tc_kernel<D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kBytes));
    attr[dev] = true;
  }
  if (T > INT32_MAX - kAK) return set_error(LSQ_ERR_SHAPE, "attention: too many tokens");
  const int64_t row = (int64_t)(H + 2 * Hkv) * D;  // elements per token of q|k|v
  CUtensorMap tm;
  LSQ_TRY(make_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, qkv, (uint64_t)row, (uint64_t)T,
                       (uint64_t)row, 64, kAQ, CU_TENSOR_MAP_SWIZZLE_128B));
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((seq + kAQ - 1) / kAQ), (unsigned)H, (unsigned)(T / seq));
  cfg.blockDim = dim3(kAThreads);
  cfg.dynamicSmemBytes = SM::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  LSQ_CUDA(::lsq::launched(cudaLaunchKernelEx(&cfg, attn_fwd_tc_kernel<D>, tm, T, seq, H, Hkv, o,
                                              lse, sl2, dev_err)));
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

// Causal grouped-query attention, forward and backward, for one layer of the
// Llama-style decoder (the model the Soup layer-streaming tutorial names in
// "維護者的 4GB／8B 成績"): o = softmax(q k^T / sqrt(d), causal) v, with query
// head h reading kv head h / (H / Hkv), positions restarting at 0 per sequence.
//
// All products run on 5th-generation tensor cores: tcgen05.mma from
// 128-byte-swizzled shared-memory tiles (loaded by TMA) into TMEM accumulators.
// The forward (attn_fwd_tc_kernel) keeps an online (running max / running sum)
// softmax in the exp2 domain and saves the row log-sum-exp.  The backward
// recomputes the probabilities from it in two kernels: dK/dV (one CTA per key
// block and query head; the kv-head sums of the query heads' dk, dv are taken
// later in a fixed order) and dQ (one CTA per query block and head), so no
// output is accumulated with atomics and every result is deterministic.
// Precision: q, k, v and o are fp16 (the forward activations); the forward and
// the recomputed scores use fp16 products, with the probabilities rounded to
// fp16 for P V.  The backward's products with a gradient operand (dO, dS) are
// bf16: v and the q (dK) or k (dQ) tiles they meet are converted to bf16 in
// shared memory, and P and dS are rounded to bf16.
#include <cuda.h>
#include <math.h>

#include "common.cuh"

namespace lsq {

namespace {

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
// ------------------------------------------------------------------ backward on tcgen05
// Both kernels recompute the probabilities from the forward's log-sum-exp,
// p = exp2(s sl2 - lse log2 e), and form ds = p (dp - delta) with
// delta = rowsum(dO o O).  Products with a gradient operand are bf16: V, and the
// copies of Q (dK kernel) or K (dQ kernel) that meet dS, are converted from fp16
// to bf16 in place in shared memory once their fp16 use is over.  P and dS are
// rounded to bf16.
//   warps 0-7: the gradient warps (row = TMEM lane, warp / 4 = which half of the
//              64 columns of a chunk), then the epilogue
//   warp 8   : TMA producer;  warp 9: TMEM allocation and the MMA issuer
constexpr int kBC = 64;  // columns of a chunk (queries for dK/dV, keys for dQ)

// fp16 -> bf16 (nearest even) of a tile in place, 16-byte chunks over the 256 gradient threads
__device__ __forceinline__ void tile_f16_to_bf16(uint8_t* tile, uint32_t bytes, int tid) {
  for (uint32_t o = (uint32_t)tid * 16u; o < bytes; o += 256u * 16u) {
    uint4 v = *reinterpret_cast<uint4*>(tile + o);
    v.x = f16x2_to_bf16x2(v.x);
    v.y = f16x2_to_bf16x2(v.y);
    v.z = f16x2_to_bf16x2(v.z);
    v.w = f16x2_to_bf16x2(v.w);
    *reinterpret_cast<uint4*>(tile + o) = v;
  }
}

template <int D>
struct DkvSmem {
  static constexpr uint32_t kKV = kAK * D * 2;   // K (fp16) or V (bf16): 128 keys
  static constexpr uint32_t kQc = kBC * D * 2;   // a chunk of Q or dO: 64 queries
  static constexpr uint32_t kPc = kAK * kBC * 2; // P^T or dS^T: 128 keys x 64 queries
  static constexpr uint32_t kBytes = 1024 + 2 * kKV + 4 * kQc + 2 * kPc;
};

// dK, dV of 128 keys for one query head: loops over the 64-query chunks at and
// after the key block (causal), accumulating dV += P^T dO and dK += dS^T Q in
// TMEM; writes dk = scale dK and dv per query head.
template <int D>
__global__ void __launch_bounds__(kAThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,   // qkv, boxes of 128 rows
                            const __grid_constant__ CUtensorMap tm_q,    // qkv, boxes of 64 rows
                            const __grid_constant__ CUtensorMap tm_do,   // dO, boxes of 64 rows
                            const float* __restrict__ lse, const float* __restrict__ delta,
                            int64_t T, int seq, int H, int Hkv, float sl2, float scale,
                            float* __restrict__ dk, float* __restrict__ dv, int* __restrict__ dev_err) {
  using SM = DkvSmem<D>;
  constexpr int DA = D / 64;
  extern __shared__ uint8_t dkv_raw[];
  __shared__ __align__(8) uint64_t bar_kv, bar_vconv, bar_q[2], bar_qfree[2], bar_sdp[2],
      bar_tfree[2], bar_ds, bar_pds;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  pdl_trigger();

  uint8_t* Ks = align1024_a(dkv_raw);
  uint8_t* Vs = Ks + SM::kKV;
  uint8_t* Qb = Vs + SM::kKV;       // [2] Q chunks (fp16, then bf16)
  uint8_t* dOb = Qb + 2 * SM::kQc;  // [2] dO chunks (bf16)
  uint8_t* Pt = dOb + 2 * SM::kQc;  // P^T (bf16, K-major over queries)
  uint8_t* dSt = Pt + SM::kPc;      // dS^T
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int k0 = kb * kAK;
  const int64_t tok0 = (int64_t)b * seq;
  const int nc = (seq - k0 + kBC - 1) / kBC;  // query chunks from k0 on
  constexpr uint32_t kColS = 0, kColP = 2 * kBC, kColV = 4 * kBC, kColK = 4 * kBC + 128;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar_kv), 1);
    mbar_init(smem_u32(&bar_vconv), 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_q[i]), 1);
      mbar_init(smem_u32(&bar_qfree[i]), 1);
      mbar_init(smem_u32(&bar_sdp[i]), 1);
      mbar_init(smem_u32(&bar_tfree[i]), 8);
    }
    mbar_init(smem_u32(&bar_ds), 8);
    mbar_init(smem_u32(&bar_pds), 1);
    abort_sh = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&tmem_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;

  if (warp == kWarpTma) {
    if (lane == 0) {
      pdl_wait();
      mbar_arrive_expect_tx(smem_u32(&bar_kv), 2 * SM::kKV);
      for (int a = 0; a < DA; ++a) {
        tma_load_2d(smem_u32(Ks + a * kAK * 128), &tm_kv, smem_u32(&bar_kv), (H + g) * D + 64 * a,
                    (int)(tok0 + k0));
        tma_load_2d(smem_u32(Vs + a * kAK * 128), &tm_kv, smem_u32(&bar_kv),
                    (H + Hkv + g) * D + 64 * a, (int)(tok0 + k0));
      }
      for (int c = 0; c < nc; ++c) {
        const int qb = c & 1;
        if (c >= 2 && !mbar_wait_bounded(smem_u32(&bar_qfree[qb]), (uint32_t)(((c - 2) >> 1) & 1),
                                         abort_flag, dev_err, DEV_ERR_WAIT_GEMM))
          break;
        const int row = (int)(tok0 + k0 + c * kBC);
        const uint32_t fb = smem_u32(&bar_q[qb]);
        mbar_arrive_expect_tx(fb, 2 * SM::kQc);
        for (int a = 0; a < DA; ++a) {
          tma_load_2d(smem_u32(Qb + qb * SM::kQc + a * kBC * 128), &tm_q, fb, h * D + 64 * a, row);
          tma_load_2d(smem_u32(dOb + qb * SM::kQc + a * kBC * 128), &tm_do, fb, h * D + 64 * a, row);
        }
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      const uint32_t id_s = umma_idesc_f16(kAK, kBC);            // S^T = K Q^T (fp16)
      const uint32_t id_dp = umma_idesc_bf16(kAK, kBC);          // dP^T = V dO^T (bf16)
      const uint32_t id_acc = umma_idesc_bf16(kAK, D) | (1u << 16);  // dV, dK: B MN-major
      bool ok = mbar_wait_bounded(smem_u32(&bar_kv), 0u, abort_flag, dev_err, DEV_ERR_WAIT_GEMM) &&
                mbar_wait_bounded(smem_u32(&bar_vconv), 0u, abort_flag, dev_err, DEV_ERR_WAIT_GEMM);
      auto issue_sdp = [&](int c) -> bool {
        const int qb = c & 1;
        if (!mbar_wait_bounded(smem_u32(&bar_q[qb]), (uint32_t)((c >> 1) & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM))
          return false;
        if (c >= 2 && !mbar_wait_bounded(smem_u32(&bar_tfree[qb]), (uint32_t)(((c - 2) >> 1) & 1),
                                         abort_flag, dev_err, DEV_ERR_WAIT_GEMM))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (uint32_t)((kk >> 2) * kAK * 128 + (kk & 3) * 32);
          const uint32_t kq = (uint32_t)((kk >> 2) * kBC * 128 + (kk & 3) * 32);
          tc_mma_bf16(tmem + kColS + (uint32_t)qb * kBC, umma_desc_k_sw128(smem_u32(Ks) + ka),
                      umma_desc_k_sw128(smem_u32(Qb + qb * SM::kQc) + kq), id_s, kk > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + kColP + (uint32_t)qb * kBC, umma_desc_k_sw128(smem_u32(Vs) + ka),
                      umma_desc_k_sw128(smem_u32(dOb + qb * SM::kQc) + kq), id_dp, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&bar_sdp[qb]));
        return true;
      };
      ok = ok && issue_sdp(0);
      for (int c = 0; c < nc && ok; ++c) {
        const int qb = c & 1;
        if (c + 1 < nc) ok = issue_sdp(c + 1);
        if (!ok) break;
        ok = mbar_wait_bounded(smem_u32(&bar_ds), (uint32_t)(c & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBC / 16; ++kk) {
          const uint32_t pa = (uint32_t)(kk * 32);
          const uint32_t bo = (uint32_t)kk * 16 * 128;
          const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
          tc_mma_bf16(tmem + kColV, umma_desc_k_sw128(smem_u32(Pt) + pa),
                      umma_desc_mn_sw128(smem_u32(dOb + qb * SM::kQc) + bo, kBC * 128, 1024u), id_acc,
                      acc);
          tc_mma_bf16(tmem + kColK, umma_desc_k_sw128(smem_u32(dSt) + pa),
                      umma_desc_mn_sw128(smem_u32(Qb + qb * SM::kQc) + bo, kBC * 128, 1024u), id_acc,
                      acc);
        }
        tc_commit(smem_u32(&bar_pds));       // P^T, dS^T read; dK, dV updated
        tc_commit(smem_u32(&bar_qfree[qb]));  // the Q and dO chunk read
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- gradient warps
    const int tid = threadIdx.x;               // 0..255
    const int r = (warp & 3) * 32 + lane;      // key row of the block = TMEM lane
    const int hf = warp >> 2;                  // queries 32 hf .. of each chunk
    const int kpos = k0 + r;
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    pdl_wait();  // delta comes from the kernel before
    bool ok = mbar_wait_bounded(smem_u32(&bar_kv), 0u, abort_flag, dev_err, DEV_ERR_WAIT_GEMM);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) {
      tile_f16_to_bf16(Vs, SM::kKV, tid);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_vconv));
    }
    // lse (log2 units) and delta of the warp's 32 queries of a chunk: lane i holds
    // query i's, fetched one chunk ahead, and the lanes read them by shuffle
    auto fetch = [&](int c, float* l2v, float* dlv) {
      const int qq = min(k0 + c * kBC + 32 * hf + lane, seq - 1);
      *l2v = __ldg(lse + (int64_t)h * T + tok0 + qq) * 1.4426950408889634f;
      *dlv = __ldg(delta + (int64_t)h * T + tok0 + qq);
    };
    float l2_own = 0.f, dl_own = 0.f;
    if (nc > 0) fetch(0, &l2_own, &dl_own);
    for (int c = 0; c < nc && ok; ++c) {
      const int qb = c & 1;
      const int q0 = k0 + c * kBC + 32 * hf;  // this thread's first query
      float l2_next = 0.f, dl_next = 0.f;
      if (c + 1 < nc) fetch(c + 1, &l2_next, &dl_next);
      ok = mbar_wait_bounded(smem_u32(&bar_sdp[qb]), (uint32_t)((c >> 1) & 1), abort_flag, dev_err,
                             DEV_ERR_WAIT_GEMM);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][16], pv[2][16];
      tmem_ld16(trow + kColS + (uint32_t)(qb * kBC + 32 * hf), sv[0]);
      tmem_ld16(trow + kColS + (uint32_t)(qb * kBC + 32 * hf + 16), sv[1]);
      tmem_ld16(trow + kColP + (uint32_t)(qb * kBC + 32 * hf), pv[0]);
      tmem_ld16(trow + kColP + (uint32_t)(qb * kBC + 32 * hf + 16), pv[1]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_tfree[qb]));
      uint32_t ppk[16], dpk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float p[2], d[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int qq = q0 + e + u;
          const bool live = kpos <= qq && qq < seq && kpos < seq;
          const float s = __uint_as_float(sv[(e + u) >> 4][(e + u) & 15]);
          const float dp = __uint_as_float(pv[(e + u) >> 4][(e + u) & 15]);
          const float l2 = __shfl_sync(0xFFFFFFFFu, l2_own, e + u);
          const float dl = __shfl_sync(0xFFFFFFFFu, dl_own, e + u);
          p[u] = live ? exp2f(fmaf(s, sl2, -l2)) : 0.f;
          d[u] = p[u] * (dp - dl);
        }
        ppk[e >> 1] = pack_bf16x2(p[0], p[1]);
        dpk[e >> 1] = pack_bf16x2(d[0], d[1]);
      }
      // S^T of this chunk is done with Q (its commit covered it): Q becomes dK's bf16
      // operand, while the previous chunk's dV, dK products may still run
      tile_f16_to_bf16(Qb + qb * SM::kQc, SM::kQc, tid);
      // the previous chunk's dV, dK products have read P^T and dS^T
      if (c > 0) {
        ok = mbar_wait_bounded(smem_u32(&bar_pds), (uint32_t)((c - 1) & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t off = sw128_offset((uint32_t)r, (uint32_t)(hf * 4 + cc));
        *reinterpret_cast<uint4*>(Pt + off) =
            make_uint4(ppk[4 * cc], ppk[4 * cc + 1], ppk[4 * cc + 2], ppk[4 * cc + 3]);
        *reinterpret_cast<uint4*>(dSt + off) =
            make_uint4(dpk[4 * cc], dpk[4 * cc + 1], dpk[4 * cc + 2], dpk[4 * cc + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_ds));
      l2_own = l2_next;
      dl_own = dl_next;
    }
    // ---------------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait_bounded(smem_u32(&bar_pds), (uint32_t)((nc - 1) & 1), abort_flag,
                                   dev_err, DEV_ERR_WAIT_GEMM);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) {
      tc_fence_after();
      const bool live = kpos < seq;
      const int64_t o = (tok0 + kpos) * (int64_t)H * D + (int64_t)h * D + hf * (D / 2);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t kv[16], vv[16];
        tmem_ld16(trow + kColK + (uint32_t)(hf * (D / 2) + 16 * c), kv);
        tmem_ld16(trow + kColV + (uint32_t)(hf * (D / 2) + 16 * c), vv);
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            *reinterpret_cast<float4*>(dk + o + 16 * c + e) =
                make_float4(__uint_as_float(kv[e]) * scale, __uint_as_float(kv[e + 1]) * scale,
                            __uint_as_float(kv[e + 2]) * scale, __uint_as_float(kv[e + 3]) * scale);
            *reinterpret_cast<float4*>(dv + o + 16 * c + e) =
                make_float4(__uint_as_float(vv[e]), __uint_as_float(vv[e + 1]),
                            __uint_as_float(vv[e + 2]), __uint_as_float(vv[e + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (abort_sh) settle_ns(2000000);
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
struct DqSmem {
  static constexpr uint32_t kQ = kAQ * D * 2;    // Q (fp16) or dO (bf16): 128 queries
  static constexpr uint32_t kKc = kBC * D * 2;   // a chunk of K or V: 64 keys
  static constexpr uint32_t kSc = kAQ * kBC * 2; // dS: 128 queries x 64 keys
  static constexpr uint32_t kBytes = 1024 + 2 * kQ + 4 * kKc + kSc;
};

// dQ of 128 queries for one query head: loops over the 64-key chunks up to the
// queries (causal), accumulating dQ += dS K in TMEM; writes dq = scale dQ.
template <int D>
__global__ void __launch_bounds__(kAThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q,    // qkv, boxes of 128 rows
                          const __grid_constant__ CUtensorMap tm_kv,   // qkv, boxes of 64 rows
                          const __grid_constant__ CUtensorMap tm_do,   // dO, boxes of 128 rows
                          const float* __restrict__ lse, const float* __restrict__ delta,
                          int64_t T, int seq, int H, int Hkv, float sl2, float scale,
                          float* __restrict__ dq, int* __restrict__ dev_err) {
  using SM = DqSmem<D>;
  constexpr int DA = D / 64;
  extern __shared__ uint8_t dq_raw[];
  __shared__ __align__(8) uint64_t bar_qd, bar_kv[2], bar_vconv[2], bar_kvfree[2], bar_sdp[2],
      bar_tfree[2], bar_ds, bar_dsfree;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  pdl_trigger();

  uint8_t* Qs = align1024_a(dq_raw);
  uint8_t* dOs = Qs + SM::kQ;
  uint8_t* Kb = dOs + SM::kQ;       // [2] K chunks (fp16, then bf16)
  uint8_t* Vb = Kb + 2 * SM::kKc;   // [2] V chunks (bf16)
  uint8_t* dSs = Vb + 2 * SM::kKc;  // dS (bf16, K-major over keys)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qbk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int q0 = qbk * kAQ;
  const int64_t tok0 = (int64_t)b * seq;
  const int nc = (min(seq, q0 + kAQ) + kBC - 1) / kBC;  // key chunks up to the block's last query
  constexpr uint32_t kColS = 0, kColP = 2 * kBC, kColQ = 4 * kBC;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar_qd), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_kv[i]), 1);
      mbar_init(smem_u32(&bar_vconv[i]), 8);
      mbar_init(smem_u32(&bar_kvfree[i]), 1);
      mbar_init(smem_u32(&bar_sdp[i]), 1);
      mbar_init(smem_u32(&bar_tfree[i]), 8);
    }
    mbar_init(smem_u32(&bar_ds), 8);
    mbar_init(smem_u32(&bar_dsfree), 1);
    abort_sh = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&tmem_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;

  if (warp == kWarpTma) {
    if (lane == 0) {
      pdl_wait();
      mbar_arrive_expect_tx(smem_u32(&bar_qd), 2 * SM::kQ);
      for (int a = 0; a < DA; ++a) {
        tma_load_2d(smem_u32(Qs + a * kAQ * 128), &tm_q, smem_u32(&bar_qd), h * D + 64 * a,
                    (int)(tok0 + q0));
        tma_load_2d(smem_u32(dOs + a * kAQ * 128), &tm_do, smem_u32(&bar_qd), h * D + 64 * a,
                    (int)(tok0 + q0));
      }
      for (int c = 0; c < nc; ++c) {
        const int kb = c & 1;
        if (c >= 2 && !mbar_wait_bounded(smem_u32(&bar_kvfree[kb]), (uint32_t)(((c - 2) >> 1) & 1),
                                         abort_flag, dev_err, DEV_ERR_WAIT_GEMM))
          break;
        const int row = (int)(tok0 + c * kBC);
        const uint32_t fb = smem_u32(&bar_kv[kb]);
        mbar_arrive_expect_tx(fb, 2 * SM::kKc);
        for (int a = 0; a < DA; ++a) {
          tma_load_2d(smem_u32(Kb + kb * SM::kKc + a * kBC * 128), &tm_kv, fb, (H + g) * D + 64 * a,
                      row);
          tma_load_2d(smem_u32(Vb + kb * SM::kKc + a * kBC * 128), &tm_kv, fb,
                      (H + Hkv + g) * D + 64 * a, row);
        }
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      const uint32_t id_s = umma_idesc_f16(kAQ, kBC);            // S = Q K^T (fp16)
      const uint32_t id_dp = umma_idesc_bf16(kAQ, kBC);          // dP = dO V^T (bf16)
      const uint32_t id_acc = umma_idesc_bf16(kAQ, D) | (1u << 16);  // dQ += dS K: B MN-major
      bool ok = mbar_wait_bounded(smem_u32(&bar_qd), 0u, abort_flag, dev_err, DEV_ERR_WAIT_GEMM);
      auto issue_sdp = [&](int c) -> bool {
        const int kb = c & 1;
        if (!mbar_wait_bounded(smem_u32(&bar_kv[kb]), (uint32_t)((c >> 1) & 1), abort_flag,
                               dev_err, DEV_ERR_WAIT_GEMM) ||
            !mbar_wait_bounded(smem_u32(&bar_vconv[kb]), (uint32_t)((c >> 1) & 1), abort_flag,
                               dev_err, DEV_ERR_WAIT_GEMM))
          return false;
        if (c >= 2 && !mbar_wait_bounded(smem_u32(&bar_tfree[kb]), (uint32_t)(((c - 2) >> 1) & 1),
                                         abort_flag, dev_err, DEV_ERR_WAIT_GEMM))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qa = (uint32_t)((kk >> 2) * kAQ * 128 + (kk & 3) * 32);
          const uint32_t ka = (uint32_t)((kk >> 2) * kBC * 128 + (kk & 3) * 32);
          tc_mma_bf16(tmem + kColS + (uint32_t)kb * kBC, umma_desc_k_sw128(smem_u32(Qs) + qa),
                      umma_desc_k_sw128(smem_u32(Kb + kb * SM::kKc) + ka), id_s, kk > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + kColP + (uint32_t)kb * kBC, umma_desc_k_sw128(smem_u32(dOs) + qa),
                      umma_desc_k_sw128(smem_u32(Vb + kb * SM::kKc) + ka), id_dp, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&bar_sdp[kb]));
        return true;
      };
      ok = ok && issue_sdp(0);
      for (int c = 0; c < nc && ok; ++c) {
        const int kb = c & 1;
        if (c + 1 < nc) ok = issue_sdp(c + 1);
        if (!ok) break;
        ok = mbar_wait_bounded(smem_u32(&bar_ds), (uint32_t)(c & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBC / 16; ++kk)
          tc_mma_bf16(tmem + kColQ, umma_desc_k_sw128(smem_u32(dSs) + (uint32_t)(kk * 32)),
                      umma_desc_mn_sw128(smem_u32(Kb + kb * SM::kKc) + (uint32_t)kk * 16 * 128,
                                         kBC * 128, 1024u),
                      id_acc, (c > 0 || kk > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bar_dsfree));     // dS read; dQ updated
        tc_commit(smem_u32(&bar_kvfree[kb]));  // the K and V chunk read
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- gradient warps
    const int tid = threadIdx.x;
    const int r = (warp & 3) * 32 + lane;  // query row of the block = TMEM lane
    const int hf = warp >> 2;              // keys 32 hf .. of each chunk
    const int q = q0 + r;
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    pdl_wait();  // delta comes from the kernels before
    const int qq = min(q, seq - 1);
    const float l2 = __ldg(lse + (int64_t)h * T + tok0 + qq) * 1.4426950408889634f;
    const float dl = __ldg(delta + (int64_t)h * T + tok0 + qq);
    bool ok = true;
    // V of chunk c becomes bf16 (dP's operand) as soon as it lands
    auto convert_v = [&](int c) -> bool {
      const int kb = c & 1;
      bool w = mbar_wait_bounded(smem_u32(&bar_kv[kb]), (uint32_t)((c >> 1) & 1), abort_flag,
                                 dev_err, DEV_ERR_WAIT_GEMM);
      w = __all_sync(0xFFFFFFFFu, w);
      if (!w) return false;
      tile_f16_to_bf16(Vb + kb * SM::kKc, SM::kKc, tid);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_vconv[kb]));
      return true;
    };
    ok = convert_v(0);
    for (int c = 0; c < nc && ok; ++c) {
      const int kb = c & 1;
      if (c + 1 < nc && !convert_v(c + 1)) { ok = false; break; }
      ok = mbar_wait_bounded(smem_u32(&bar_sdp[kb]), (uint32_t)((c >> 1) & 1), abort_flag, dev_err,
                             DEV_ERR_WAIT_GEMM);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][16], pv[2][16];
      tmem_ld16(trow + kColS + (uint32_t)(kb * kBC + 32 * hf), sv[0]);
      tmem_ld16(trow + kColS + (uint32_t)(kb * kBC + 32 * hf + 16), sv[1]);
      tmem_ld16(trow + kColP + (uint32_t)(kb * kBC + 32 * hf), pv[0]);
      tmem_ld16(trow + kColP + (uint32_t)(kb * kBC + 32 * hf + 16), pv[1]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_tfree[kb]));
      const int kfirst = c * kBC + 32 * hf;  // this thread's first key
      uint32_t dpk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float d[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int key = kfirst + e + u;
          const bool live = key <= q && key < seq && q < seq;
          const float s = __uint_as_float(sv[(e + u) >> 4][(e + u) & 15]);
          const float dp = __uint_as_float(pv[(e + u) >> 4][(e + u) & 15]);
          const float p = live ? exp2f(fmaf(s, sl2, -l2)) : 0.f;
          d[u] = p * (dp - dl);
        }
        dpk[e >> 1] = pack_bf16x2(d[0], d[1]);
      }
      // S of this chunk is done with K (its commit covered it): K becomes dQ's bf16
      // operand, while the previous chunk's dQ product may still run
      tile_f16_to_bf16(Kb + kb * SM::kKc, SM::kKc, tid);
      // the previous chunk's dQ product has read dS
      if (c > 0) {
        ok = mbar_wait_bounded(smem_u32(&bar_dsfree), (uint32_t)((c - 1) & 1), abort_flag, dev_err,
                               DEV_ERR_WAIT_GEMM);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        *reinterpret_cast<uint4*>(dSs + sw128_offset((uint32_t)r, (uint32_t)(hf * 4 + cc))) =
            make_uint4(dpk[4 * cc], dpk[4 * cc + 1], dpk[4 * cc + 2], dpk[4 * cc + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_ds));
    }
    if (ok) ok = mbar_wait_bounded(smem_u32(&bar_dsfree), (uint32_t)((nc - 1) & 1), abort_flag,
                                   dev_err, DEV_ERR_WAIT_GEMM);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) {
      tc_fence_after();
      const bool live = q < seq;
      const int64_t o = (tok0 + q) * (int64_t)H * D + (int64_t)h * D + hf * (D / 2);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[16];
        tmem_ld16(trow + kColQ + (uint32_t)(hf * (D / 2) + 16 * c), v);
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(dq + o + 16 * c + e) =
                make_float4(__uint_as_float(v[e]) * scale, __uint_as_float(v[e + 1]) * scale,
                            __uint_as_float(v[e + 2]) * scale, __uint_as_float(v[e + 3]) * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (abort_sh) settle_ns(2000000);
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr[dev]) {
    LSQ_CUDA(cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)DkvSmem<D>::kBytes));
    LSQ_CUDA(cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)DqSmem<D>::kBytes));
    attr[dev] = true;
  }
  if (T > INT32_MAX - kAK) return set_error(LSQ_ERR_SHAPE, "attention: too many tokens");
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  const int batch = (int)(T / seq);
  const float scale = 1.f / sqrtf((float)D);
  const float sl2 = 1.4426950408889634f * scale;
  const int64_t nw = T * H;
  attn_delta_kernel<D><<<(unsigned)((nw * 32 + 255) / 256), 256, 0, st>>>(o, dout, T, H, delta);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  const int64_t row = (int64_t)(H + 2 * Hkv) * D;  // elements per token of q|k|v
  CUtensorMap tm_qkv128, tm_qkv64, tm_do128, tm_do64;
  LSQ_TRY(make_tmap_2d(&tm_qkv128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, qkv, (uint64_t)row,
                       (uint64_t)T, (uint64_t)row, 64, kAK, CU_TENSOR_MAP_SWIZZLE_128B));
  LSQ_TRY(make_tmap_2d(&tm_qkv64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, qkv, (uint64_t)row,
                       (uint64_t)T, (uint64_t)row, 64, kBC, CU_TENSOR_MAP_SWIZZLE_128B));
  LSQ_TRY(make_tmap_2d(&tm_do128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dout, (uint64_t)H * D,
                       (uint64_t)T, (uint64_t)H * D, 64, kAQ, CU_TENSOR_MAP_SWIZZLE_128B));
  LSQ_TRY(make_tmap_2d(&tm_do64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dout, (uint64_t)H * D,
                       (uint64_t)T, (uint64_t)H * D, 64, kBC, CU_TENSOR_MAP_SWIZZLE_128B));
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((seq + kAK - 1) / kAK), (unsigned)H, (unsigned)batch);
  cfg.blockDim = dim3(kAThreads);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cfg.dynamicSmemBytes = DkvSmem<D>::kBytes;
  LSQ_CUDA(::lsq::launched(cudaLaunchKernelEx(&cfg, attn_bwd_dkdv_tc_kernel<D>, tm_qkv128, tm_qkv64,
                                              tm_do64, lse, (const float*)delta, T, seq, H, Hkv,
                                              sl2, scale, dk, dv, dev_err)));
  cfg.gridDim = dim3((unsigned)((seq + kAQ - 1) / kAQ), (unsigned)H, (unsigned)batch);
  cfg.dynamicSmemBytes = DqSmem<D>::kBytes;
  LSQ_CUDA(::lsq::launched(cudaLaunchKernelEx(&cfg, attn_bwd_dq_tc_kernel<D>, tm_qkv128, tm_qkv64,
                                              tm_do128, lse, (const float*)delta, T, seq, H, Hkv,
                                              sl2, scale, dq, dev_err)));
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

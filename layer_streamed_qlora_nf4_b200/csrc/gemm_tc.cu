// Tensor-core GEMM with the NF4 dequantisation fused into the operand load and
// the LoRA up-projection fused as an extra K range ("slab"), for sm_100a.
//
// What it computes (per call): out[t, m] = sum_c Wop[m, c] act[t, c]
//                                         + sum_j la[m, j] lb[t, j] (+ residual)
// Forward of a frozen NF4 linear with LoRA (Soup layer-streaming tutorial,
// "四段資料路徑" part 1): Wop = deq(W), act = x, la = s*B, lb = u = x A^T.
// Its input gradient (part 3 and FAQ 4, W is re-read in backward):
// Wop = deq(W)^T, act = dY, la = s*A^T, lb = v = dY B.
// Operand precision: the forward multiplies fp16 operands (the dequantised
// weight rounded once to fp16, fp16 activations, the LoRA slab in fp16); the
// input gradient multiplies bf16 operands (gradients need bf16's exponent
// range); both accumulate in fp32 in TMEM.
//
// Design for B200 (one CTA per SM, 384 threads, warp-specialised):
//   warp 0    : TMA producer for the activation tile (128-byte swizzle), the LoRA
//               slab's operands (la into the weight stage, lb into the activation
//               stage) and, in the bf16-weight modes, the weight tile itself:
//               K-major for W_BF16_N and W_BF16C_N (converted to fp16 in place by
//               the operand warps), as two MN-major 64-feature atoms for W_BF16_T
//               (read by the MMA as an MN-major A)
//   warp 1    : allocates TMEM, one elected thread issues tcgen05.mma
//               (M = 128 output features x N = up to 256 tokens x K = 16),
//               accumulators in TMEM (up to 2 x 256 fp32 columns)
//   warp 2    : TMA producer for the packed NF4 codes into a staging ring (as deep
//               as the shared memory left after the operand stages allows)
//   warps 4-11: operand stage - expand the staged codes to fp16 / bf16
//               (level[code] * absmax in fp32, then round to nearest) straight into the
//               UMMA canonical K-major 128-byte-swizzle layout, fence the async
//               proxy, arrive.  Two warps per SM sub-partition.  Then the epilogue:
//               each warp reads its TMEM lane quarter (32 features) for every third
//               32-token chunk and writes it with its own TMA stores, with no
//               barrier between warps.
// The output tile is 128 features x all tokens of the CTA (up to 512), so each
// weight element is dequantised once per token tile.  Small problems use a
// fixed-order split over K with an fp32 partial buffer, summed in slice order by a
// reduce kernel or by the kernel that consumes the product: results are
// deterministic and independent of scheduling.
// Every mbarrier wait is bounded (1 s) and aborts the CTA with a device status
// bit instead of hanging.
// Launch: programmatic dependent launch, so that the set-up (barriers, TMEM) and
// the first weight stages - the frozen weight does not depend on the kernel
// before - overlap that kernel's last wave; the activation and slab loads and the
// epilogue wait for it (pdl_wait).
#include <cuda.h>

#include <cstdlib>
#include <mutex>

#include "common.cuh"

namespace lsq {

__device__ int g_lsq_dev_status;

#ifdef LSQ_GEMM_STAMPS
// Diagnostic build only (-DLSQ_GEMM_STAMPS): per-CTA globaltimer stamps of the
// kernel's phases for the most recent launch, read by lsq_debug_gemm_stamps.
// Slots: 0 entry, 1 set-up done, 2 first stage ready (MMA issuer), 3 last MMA
// issued, 4 accumulator ready (epilogue warp 4), 5 epilogue stores done, 6 exit,
// 7 summed issuer wait on operand-ready barriers (ns).
constexpr int kStampCtas = 1024;
__device__ unsigned long long g_gemm_stamps[kStampCtas][8];
#define LSQ_STAMP(slot, v)                                                         \
  do {                                                                             \
    const int _c = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (_c < kStampCtas) g_gemm_stamps[_c][slot] = (v);                            \
  } while (0)
#else
#define LSQ_STAMP(slot, v) \
  do {                     \
  } while (0)
#endif

#ifdef LSQ_GEMM_KTL
// Diagnostic build only (-DLSQ_GEMM_KTL): a per-k-tile timeline (globaltimer) of
// every role of the first two CTAs (one pair) of the most recent launch, read by
// lsq_debug_gemm_ktl.  Rows: 0 warp 0 saw the stage empty, 1 warp 0 issued its
// loads, 2 warp 2 issued the code load, 3 operand warp 4 may fill the stage (code
// slot full, stage empty), 4 its expansion is done and fenced, 5 it arrived,
// 6 the issuer saw the stage full (even CTA) or the forwarder arrived (odd CTA),
// 7 the issuer committed the stage's MMAs.
constexpr int kKtlTiles = 256;
__device__ unsigned long long g_gemm_ktl[2][8][kKtlTiles];
#define LSQ_KTL(row, it)                                                           \
  do {                                                                             \
    const int _c = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (_c < 2 && (it) < kKtlTiles) g_gemm_ktl[_c][row][it] = globaltimer_ns();    \
  } while (0)
#else
#define LSQ_KTL(row, it) \
  do {                   \
  } while (0)
#endif

namespace {

constexpr int kThreads = 384;   // 4 control warps + 8 operand/epilogue warps
constexpr int kOpWarps = 8;
constexpr int kOpThreads = kOpWarps * 32;
constexpr int kBM = 128;        // output features per CTA (UMMA M)
constexpr int kBK = 64;         // contraction per stage = one SW128 atom = one NF4 block
constexpr int kWStageBytes = kBM * kBK * 2;  // 16 KB bf16 operand tile
constexpr int kMaxStages = 4;
constexpr int kMaxRing = 8;
constexpr uint32_t kSmemBudget = 227 * 1024;
constexpr int kAmDepth = 8;  // absmax prefetch ring: 8 k-tiles x 256 floats
constexpr uint32_t kAmRingBytes = kAmDepth * 256 * 4 * 2;  // absmax (or 8-bit words) + scales
constexpr uint32_t kDynSmemLimit = kSmemBudget - 2048;  // the kernel's dynamic shared memory cap
// the epilogue's staging: 12 warps x four 4 KB slots, after the 1 KB alignment pad
constexpr uint32_t kEpilogueBytes = 1024u + 12u * 16384u;
static_assert(W_NF4_N == LSQ_GEMM_NF4_FWD && W_NF4_T == LSQ_GEMM_NF4_DX &&
                  W_BF16_N == LSQ_GEMM_BF16_FWD && W_BF16_T == LSQ_GEMM_BF16_DX &&
                  W_BF16C_N == LSQ_GEMM_BF16_AS_F16_FWD,
              "operand modes match the public constants");

struct KParams {
  int M, T, Kc;
  int bn, nacc, stages, ring_stages;
  int kt_total, kt_per_split, splits;
  uint32_t ring_bytes, alloc_cols;
  const float* absmax;
  const uint8_t* am_q;  // 8-bit absmax mode when non-null
  const float* am_s;
  int w_rows, w_cols;
  int slab_w;
  void* out;
  int out_f32;
  long long ldo;
  const float* residual;
  long long ldr;
  float* partial;
  int* dev_err;
  float levels[16];
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int WMODE, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                   const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_out,
                   const __grid_constant__ CUtensorMap tm_res,
                   const __grid_constant__ CUtensorMap tm_la,
                   const __grid_constant__ CUtensorMap tm_lb, const __grid_constant__ KParams p) {
  extern __shared__ uint8_t dsm_raw[];
  __shared__ __align__(8) uint64_t bar_full[kMaxStages];
  __shared__ __align__(8) uint64_t bar_empty[kMaxStages];
  __shared__ __align__(8) uint64_t bar_cfull[kMaxRing];
  __shared__ __align__(8) uint64_t bar_cempty[kMaxRing];
  __shared__ __align__(8) uint64_t bar_acc;
  __shared__ __align__(8) uint64_t bar_opd[kMaxStages];  // PAIR, odd CTA: its operand warps done
  __shared__ __align__(8) uint64_t bar_wland[kMaxStages];  // W_BF16C_N: this CTA's bf16 tile landed
  __shared__ __align__(8) uint64_t bar_res[kThreads / 32];  // per warp: residual tile landed
  __shared__ __align__(8) uint64_t bar_grp;            // the operand warps
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float lv_sh[16];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &abort_sh;
  if (threadIdx.x == 0) LSQ_STAMP(0, globaltimer_ns());
  constexpr bool F16 = wmode_f16(WMODE);  // fp16 operands (forward) or bf16 (input gradient)
  auto pack2 = [](float lo, float hi) -> uint32_t {
    return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
  };

  const int BT = p.nacc * p.bn;
  const uint32_t acc_stride = (p.nacc > 1) ? 256u : 0u;  // TMEM column of accumulator 1
  // With PAIR, the CTA pair (cluster of 2) computes a 256-feature tile: this CTA
  // dequantises its own 128 features (half of A) and loads half of each
  // accumulator's tokens (half of B); the even CTA issues cta_group::2 MMAs.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int hb = PAIR ? p.bn / 2 : p.bn;  // tokens of each accumulator held here
  const uint32_t xs_bytes = (uint32_t)(p.nacc * hb) * 128u;
  uint8_t* dsm = align1024(dsm_raw);
  uint8_t* xs0 = dsm;
  uint8_t* ws0 = xs0 + (size_t)p.stages * xs_bytes;
  uint8_t* rg0 = ws0 + (size_t)p.stages * kWStageBytes;
  float* am_ring = reinterpret_cast<float*>(rg0 + (size_t)p.ring_stages * p.ring_bytes);  // [kAmDepth][256]
  float* sc_ring = am_ring + kAmDepth * 256;  // 8-bit mode: the scale of each fetched absmax

  // Tile order: CTAs start in launch order (x fastest), and consecutive feature
  // units (CTA pairs, or CTAs) are given a group of up to 8 token tiles each, so
  // that the tiles running together share a few weight and activation tiles in L2.
  int m_tile = blockIdx.x, t_tile = blockIdx.y;
  if (gridDim.y > 1) {
    constexpr int kG = 8;
    const int units = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
    const int lin = (int)blockIdx.y * units + (PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x);
    const int full = (int)gridDim.y / kG * kG;  // token tiles in complete groups
    int unit;
    if (lin < full * units) {
      const int g = lin / (kG * units), r = lin % (kG * units);
      unit = r / kG;
      t_tile = g * kG + r % kG;
    } else {
      const int r = lin - full * units, rest = (int)gridDim.y - full;
      unit = r / rest;
      t_tile = full + r % rest;
    }
    m_tile = PAIR ? 2 * unit + (int)(blockIdx.x & 1u) : unit;
  }
  const int m0 = m_tile * kBM;
  const int t0 = t_tile * BT;
  const int split = blockIdx.z;
  const int kt_begin = split * p.kt_per_split;
  const int kt_end = min(p.kt_total, kt_begin + p.kt_per_split);
  const int n_main = max(0, kt_end - kt_begin);
  const int n_slab = (split == 0 && p.slab_w > 0) ? (p.slab_w + 63) / 64 : 0;
  const int n_iter = n_main + n_slab;
  const int S = p.stages, CS = p.ring_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // producer + this CTA's operand warps (+ one forwarded arrival from the odd CTA)
      mbar_init(smem_u32(&bar_full[s]), 1 + kOpWarps + (PAIR ? 1 : 0));
      mbar_init(smem_u32(&bar_opd[s]), kOpWarps);
      mbar_init(smem_u32(&bar_wland[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);            // tcgen05.commit
    }
    for (int c = 0; c < CS; ++c) {
      mbar_init(smem_u32(&bar_cfull[c]), 1);
      mbar_init(smem_u32(&bar_cempty[c]), kOpWarps);
    }
    mbar_init(smem_u32(&bar_acc), 1);
    for (int w = 0; w < kThreads / 32; ++w) mbar_init(smem_u32(&bar_res[w]), 1);
    mbar_init(smem_u32(&bar_grp), kOpWarps);
    abort_sh = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (threadIdx.x < 16) lv_sh[threadIdx.x] = p.levels[threadIdx.x];
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(&tmem_base_sh), p.alloc_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&tmem_base_sh), p.alloc_cols);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_out);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  if (threadIdx.x == 0) LSQ_STAMP(1, globaltimer_ns());

  if (warp == 0) {
    // ---------------------------------------------------------- activation TMA producer
    // The whole warp walks the loop (so it reaches the final barrier converged);
    // lane 0 issues.  The activations come from the kernel before: wait for it.
    pdl_wait();
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % S;
      const uint32_t ph = (uint32_t)(it / S) & 1u;
      bool ok = mbar_wait_bounded(smem_u32(&bar_empty[s]), ph ^ 1u, abort_flag, p.dev_err,
                                  DEV_ERR_WAIT_GEMM);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint32_t fb = smem_u32(&bar_full[s]);
      if (lane == 0) LSQ_KTL(0, it);
      if (lane == 0) {
        if (it < n_main) {
          const int kt = kt_begin + it;
          constexpr bool kWTma = WMODE == W_BF16_N || WMODE == W_BF16_T;  // W by TMA here
          const uint32_t bytes = xs_bytes + (kWTma ? (uint32_t)kWStageBytes : 0u);
          if (PAIR) {
            // both CTAs' bytes complete on the even CTA's barrier
            const uint32_t fl = mapa_shared(fb, 0);
            if (leader) mbar_arrive_expect_tx(fb, 2 * bytes);
            for (int a = 0; a < p.nacc; ++a)
              tma_load_2d_pair(smem_u32(xs0 + (size_t)s * xs_bytes + (size_t)a * hb * 128), &tm_act,
                               fl, kt * kBK, t0 + a * p.bn + (int)rank * hb);
            if (WMODE == W_BF16_N)
              tma_load_2d_pair(smem_u32(ws0 + (size_t)s * kWStageBytes), &tm_w, fl, kt * kBK, m0);
            if (WMODE == W_BF16_T)  // [64 contraction rows x 64 features], twice
              for (int h2 = 0; h2 < 2; ++h2)
                tma_load_2d_pair(smem_u32(ws0 + (size_t)s * kWStageBytes + h2 * (kWStageBytes / 2)),
                                 &tm_w, fl, m0 + 64 * h2, kt * kBK);
            if (WMODE == W_BF16C_N) {  // converted in place by this CTA's operand warps
              const uint32_t wl = smem_u32(&bar_wland[s]);
              mbar_arrive_expect_tx(wl, (uint32_t)kWStageBytes);
              tma_load_2d(smem_u32(ws0 + (size_t)s * kWStageBytes), &tm_w, wl, kt * kBK, m0);
            }
          } else {
            mbar_arrive_expect_tx(fb, bytes);
            for (int a = 0; a < p.nacc; ++a)
              tma_load_2d(smem_u32(xs0 + (size_t)s * xs_bytes + (size_t)a * p.bn * 128), &tm_act,
                          fb, kt * kBK, t0 + a * p.bn);
            if (WMODE == W_BF16_N)
              tma_load_2d(smem_u32(ws0 + (size_t)s * kWStageBytes), &tm_w, fb, kt * kBK, m0);
            if (WMODE == W_BF16_T)
              for (int h2 = 0; h2 < 2; ++h2)
                tma_load_2d(smem_u32(ws0 + (size_t)s * kWStageBytes + h2 * (kWStageBytes / 2)),
                            &tm_w, fb, m0 + 64 * h2, kt * kBK);
            if (WMODE == W_BF16C_N) {
              const uint32_t wl = smem_u32(&bar_wland[s]);
              mbar_arrive_expect_tx(wl, (uint32_t)kWStageBytes);
              tma_load_2d(smem_u32(ws0 + (size_t)s * kWStageBytes), &tm_w, wl, kt * kBK, m0);
            }
          }
        } else if (p.slab_w > 0) {
          // LoRA slab: s B (or s A^T) into the weight stage, u (or v) into the
          // activation stage, 64 slab columns at a time (beyond slab_w: zeros)
          const int j0 = (it - n_main) * 64;
          const uint32_t bytes = xs_bytes + (uint32_t)kWStageBytes;
          if (PAIR) {
            const uint32_t fl = mapa_shared(fb, 0);
            if (leader) mbar_arrive_expect_tx(fb, 2 * bytes);
            for (int a = 0; a < p.nacc; ++a)
              tma_load_2d_pair(smem_u32(xs0 + (size_t)s * xs_bytes + (size_t)a * hb * 128), &tm_lb,
                               fl, j0, t0 + a * p.bn + (int)rank * hb);
            tma_load_2d_pair(smem_u32(ws0 + (size_t)s * kWStageBytes), &tm_la, fl, j0, m0);
          } else {
            mbar_arrive_expect_tx(fb, bytes);
            for (int a = 0; a < p.nacc; ++a)
              tma_load_2d(smem_u32(xs0 + (size_t)s * xs_bytes + (size_t)a * p.bn * 128), &tm_lb,
                          fb, j0, t0 + a * p.bn);
            tma_load_2d(smem_u32(ws0 + (size_t)s * kWStageBytes), &tm_la, fb, j0, m0);
          }
        } else if (!PAIR || leader) {
          mbar_arrive(fb);
        }
        LSQ_KTL(1, it);
      }
      __syncwarp();
    }
  } else if (warp == 1 && (!PAIR || leader)) {
    // ---------------------------------------------------------- MMA issuer (lane 0)
    const uint32_t idesc = F16 ? umma_idesc_f16(PAIR ? 2 * kBM : kBM, p.bn)
                               : umma_idesc_bf16(PAIR ? 2 * kBM : kBM, p.bn);
    // W_BF16_T: the weight tile is MN-major (two 64-feature atoms of 64 contraction
    // rows, 8 KB apart); the LoRA slab's A is K-major in every mode
    constexpr bool kAMn = WMODE == W_BF16_T;
    const uint32_t idesc_mn = idesc | (1u << 15);
#ifdef LSQ_GEMM_STAMPS
    unsigned long long waited = 0;
#endif
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % S;
      const uint32_t ph = (uint32_t)(it / S) & 1u;
#ifdef LSQ_GEMM_STAMPS
      const unsigned long long w0 = globaltimer_ns();
#endif
      bool ok = PAIR ? mbar_wait_bounded_cluster(smem_u32(&bar_full[s]), ph, abort_flag, p.dev_err,
                                                 DEV_ERR_WAIT_GEMM)
                     : mbar_wait_bounded(smem_u32(&bar_full[s]), ph, abort_flag, p.dev_err,
                                         DEV_ERR_WAIT_GEMM);
#ifdef LSQ_GEMM_STAMPS
      const unsigned long long w1 = globaltimer_ns();
      waited += w1 - w0;
      if (it == 0 && lane == 0) LSQ_STAMP(2, w1);
#endif
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      if (lane == 0) LSQ_KTL(6, it);
      if (lane == 0) {
        int nk = 4;
        if (it >= n_main) nk = min(4, (p.slab_w - (it - n_main) * 64) / 16);
        const uint32_t wa = smem_u32(ws0 + (size_t)s * kWStageBytes);
        const uint32_t xa = smem_u32(xs0 + (size_t)s * xs_bytes);
        const bool a_mn = kAMn && it < n_main;
        const uint32_t id = a_mn ? idesc_mn : idesc;
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t ad =
              a_mn ? umma_desc_mn_sw128(wa + (uint32_t)kk * 16 * 128, (uint32_t)kWStageBytes / 2, 1024u)
                   : umma_desc_k_sw128(wa + kk * 32);
          for (int a = 0; a < p.nacc; ++a) {
            const uint64_t bd = umma_desc_k_sw128(xa + (uint32_t)(a * hb * 128) + kk * 32);
            if (PAIR)
              tc_mma_bf16_pair(tmem + (uint32_t)a * acc_stride, ad, bd, id,
                               (it > 0 || kk > 0) ? 1u : 0u);
            else
              tc_mma_bf16(tmem + (uint32_t)a * acc_stride, ad, bd, id,
                          (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (PAIR)
          tc_commit_pair(smem_u32(&bar_empty[s]));
        else
          tc_commit(smem_u32(&bar_empty[s]));
        LSQ_KTL(7, it);
      }
      __syncwarp();
    }
    if (lane == 0) {
      if (PAIR)
        tc_commit_pair(smem_u32(&bar_acc));
      else
        tc_commit(smem_u32(&bar_acc));
#ifdef LSQ_GEMM_STAMPS
      LSQ_STAMP(3, globaltimer_ns());
      LSQ_STAMP(7, waited);
#endif
    }
    __syncwarp();
  } else if (PAIR && warp == 1) {
    // ---------------------------------------------------------- odd CTA: operand forwarder
    // Once this CTA's eight operand warps have filled stage s, one arrival
    // (release, cluster scope) on the even CTA's operand-ready barrier.
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % S;
      const uint32_t ph = (uint32_t)(it / S) & 1u;
      bool ok = mbar_wait_bounded(smem_u32(&bar_opd[s]), ph, abort_flag, p.dev_err,
                                  DEV_ERR_WAIT_GEMM);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bar_full[s]), 0));
      if (lane == 0) LSQ_KTL(6, it);
      __syncwarp();
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------- staging-ring TMA producer
    if (WMODE == W_NF4_N || WMODE == W_NF4_T) {
      for (int it = 0; it < n_main; ++it) {
        const int c = it % CS;
        const uint32_t ph = (uint32_t)(it / CS) & 1u;
        bool ok = mbar_wait_bounded(smem_u32(&bar_cempty[c]), ph ^ 1u, abort_flag, p.dev_err,
                                    DEV_ERR_WAIT_GEMM);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
        if (lane == 0) {
          const int kt = kt_begin + it;
          const uint32_t cb = smem_u32(&bar_cfull[c]);
          const uint32_t dst = smem_u32(rg0 + (size_t)c * p.ring_bytes);
          mbar_arrive_expect_tx(cb, p.ring_bytes);
          if (WMODE == W_NF4_N) tma_load_2d(dst, &tm_w, cb, kt * 32, m0);       // [128 rows][32 B]
          if (WMODE == W_NF4_T) tma_load_2d(dst, &tm_w, cb, m0 / 2, kt * kBK);  // [64 rows][64 B]
          if (WMODE == W_BF16_T) tma_load_2d(dst, &tm_w, cb, m0, kt * kBK);     // [64][128 bf16]
          if (WMODE == W_BF16C_N) tma_load_2d(dst, &tm_w, cb, kt * kBK, m0);    // [128][64 bf16] SW128
          LSQ_KTL(2, it);
        }
        __syncwarp();
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- operand stage (8 warps)
    const int tid = threadIdx.x - 128;  // 0..255
    const int ow = warp - 4;            // 0..7
    const int nblk = p.w_cols / 64;
    // Bounded barrier among the operand warps (an mbarrier with one arrival per
    // warp), so that an abort in one warp cannot strand the others.
    int grp_phase = 0;
    auto grp_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_grp));
      const bool r = mbar_wait_bounded(smem_u32(&bar_grp), (uint32_t)(grp_phase & 1), abort_flag,
                                       p.dev_err, DEV_ERR_WAIT_GEMM);
      ++grp_phase;
      return __all_sync(0xFFFFFFFFu, r);
    };
    // absmax for k-tile `it` lands in slot it % kAmDepth of a shared ring, copied
    // with cp.async kAmDepth - 1 k-tiles ahead.  NF4_N: thread tid fetches the
    // absmax of its own row m0 + (tid & 127), block kt.  NF4_T: threads 0..127
    // fetch the tile's 64 rows x 2 blocks together (row kt*64 + tid/2, block
    // m0/64 + tid%2).  With an 8-bit absmax the slot receives the aligned 32-bit
    // word holding the code, and the scale ring the run's fp32 scale; the user
    // of the value extracts the byte and multiplies (absmax_value below).
    const bool q8 = p.am_q != nullptr;
    auto issue_am = [&](int it) {
      if (it < n_main && (WMODE == W_NF4_N || (WMODE == W_NF4_T && tid < 128))) {
        const int kt = kt_begin + it;
        float* dst = am_ring + (it % kAmDepth) * 256 + tid;
        size_t b = 0;
        bool in;
        if (WMODE == W_NF4_N) {
          const int m = m0 + (tid & 127);
          in = m < p.w_rows;
          b = in ? (size_t)m * nblk + kt : 0;
        } else {
          const int n = kt * kBK + (tid >> 1);
          const int bcol = (m0 >> 6) + (tid & 1);
          in = n < p.w_rows && bcol < nblk;
          b = in ? (size_t)n * nblk + bcol : 0;
        }
        if (q8) {
          cp_async4(smem_u32(dst), p.am_q + (b & ~size_t(3)), in ? 4u : 0u);
          cp_async4(smem_u32(sc_ring + (it % kAmDepth) * 256 + tid), p.am_s + (b >> 8),
                    in ? 4u : 0u);
        } else {
          cp_async4(smem_u32(dst), p.absmax + b, in ? 4u : 0u);
        }
      }
      cp_async_commit();  // one group per k-tile (possibly empty) keeps the counting uniform
    };
#pragma unroll 1
    for (int i = 0; i < kAmDepth - 1; ++i) issue_am(i);
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int s = it % S;
      const uint32_t ph = (uint32_t)(it / S) & 1u;
      uint8_t* wst = ws0 + (size_t)s * kWStageBytes;
      cp_async_wait<kAmDepth - 2>();  // this thread's copies for k-tile `it` have landed
      if (WMODE == W_NF4_T) {
        // every thread's copies visible to all, and the slot of k-tile it - 1 free
        if (!grp_sync()) { ok = false; break; }
      }
      issue_am(it + kAmDepth - 1);
      if (it < n_main) {
        if (WMODE == W_BF16_N || WMODE == W_BF16_T) {
          ok = mbar_wait_bounded(smem_u32(&bar_empty[s]), ph ^ 1u, abort_flag, p.dev_err,
                                 DEV_ERR_WAIT_GEMM);
          ok = __all_sync(0xFFFFFFFFu, ok);
        } else if (WMODE == W_BF16C_N) {
          // the bf16 [128 x 64] tile landed in the stage, already in the 128-byte-swizzle
          // layout the MMA reads (its load was issued once the stage was free): convert
          // each 16-byte chunk to fp16 in place.  A weight beyond the fp16 range latches
          // the non-finite status bit.
          ok = mbar_wait_bounded(smem_u32(&bar_wland[s]), ph, abort_flag, p.dev_err,
                                 DEV_ERR_WAIT_GEMM);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (ok) {
            bool big = false;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int off = (tid + q * kOpThreads) * 16;
              const uint4 v = *reinterpret_cast<const uint4*>(wst + off);
              const uint32_t in[4] = {v.x, v.y, v.z, v.w};
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = unpack_bf16x2(in[e]);
                big |= !(fabsf(f.x) <= kF16Max) || !(fabsf(f.y) <= kF16Max);
                o[e] = pack_f16x2(f.x, f.y);
              }
              *reinterpret_cast<uint4*>(wst + off) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            if (__any_sync(0xFFFFFFFFu, big) && lane == 0) atomicOr(p.dev_err, DEV_ERR_NONFINITE);
            fence_proxy_async_smem();
            __syncwarp();
          }
        } else {
          const int c = it % CS;
          const uint32_t cph = (uint32_t)(it / CS) & 1u;
          const uint8_t* ring = rg0 + (size_t)c * p.ring_bytes;
          const float* amc = am_ring + (it % kAmDepth) * 256;
          const float* scc = sc_ring + (it % kAmDepth) * 256;
          // absmax of ring entry e, fetched for block b of W
          auto absmax_value = [&](int e, size_t b) -> float {
            if (!q8) return amc[e];
            const uint32_t w = __float_as_uint(amc[e]);
            return (float)((w >> (8u * (uint32_t)(b & 3))) & 0xFFu) * scc[e];
          };
          ok = mbar_wait_bounded(smem_u32(&bar_cfull[c]), cph, abort_flag, p.dev_err,
                                 DEV_ERR_WAIT_GEMM) &&
               mbar_wait_bounded(smem_u32(&bar_empty[s]), ph ^ 1u, abort_flag, p.dev_err,
                                 DEV_ERR_WAIT_GEMM);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (ok && warp == 4 && lane == 0) LSQ_KTL(3, it);
          if (ok) {
            if (WMODE == W_NF4_N) {
              // thread: row r, half h of its 64 codes (chunks 4h .. 4h+3)
              const int r = tid & 127, h = tid >> 7;
              const int kt = kt_begin + it;
              const float am = absmax_value(tid, (size_t)(m0 + r) * nblk + kt);
              const uint4 cw = *reinterpret_cast<const uint4*>(ring + r * 32 + h * 16);
              const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t w = words[q];
                uint32_t o[4];
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  const uint32_t byte = (w >> (8 * b)) & 0xFFu;
                  o[b] = pack2(lv_sh[byte >> 4] * am, lv_sh[byte & 15u] * am);
                }
                *reinterpret_cast<uint4*>(wst + sw128_offset(r, 4 * h + q)) =
                    make_uint4(o[0], o[1], o[2], o[3]);
              }
            } else if (WMODE == W_NF4_T) {
              // The [64 n x 128 m] tile is 8 x 16 blocks of 8 x 8.  Warp ow stores the
              // blocks of n-block ow, four consecutive m-blocks per stmatrix: lane t
              // dequantises (n = 8 ow + t/4, m = 32 mq + 8j + 2(t%4) + {0,1}) for
              // j = 0..3 - the fragment layout - from one 16-byte code read, and the
              // transposing store puts 8 consecutive n of one m into each 16-byte
              // chunk of the K-major tile.
              const int nb = ow;
              const int n = nb * 8 + (lane >> 2);
#pragma unroll
              for (int mq = 0; mq < 4; ++mq) {
                const uint4 seg = *reinterpret_cast<const uint4*>(ring + n * 64 + mq * 16);
                const float am = absmax_value(
                    n * 2 + (mq >> 1),
                    (size_t)((kt_begin + it) * kBK + n) * nblk + (m0 >> 6) + (mq >> 1));
                const uint32_t words[4] = {seg.x, seg.y, seg.z, seg.w};
                uint32_t regs[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const uint32_t byte = (words[j] >> (8 * (lane & 3))) & 0xFFu;
                  regs[j] = pack2(lv_sh[byte >> 4] * am, lv_sh[byte & 15u] * am);
                }
                const int m = mq * 32 + (lane >> 3) * 8 + (lane & 7);
                stmatrix_x4_trans(smem_u32(wst + sw128_offset(m, nb)), regs);
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (warp == 4 && lane == 0) LSQ_KTL(4, it);
            if (lane == 0) mbar_arrive(smem_u32(&bar_cempty[c]));
          }
        }
      } else {
        // LoRA slab (by TMA, issued by warp 0): the stage only has to be free before
        // this warp arrives
        ok = mbar_wait_bounded(smem_u32(&bar_empty[s]), ph ^ 1u, abort_flag, p.dev_err,
                               DEV_ERR_WAIT_GEMM);
        ok = __all_sync(0xFFFFFFFFu, ok);
      }
      if (ok && lane == 0)
        mbar_arrive(smem_u32(PAIR && !leader ? &bar_opd[s] : &bar_full[s]));
      if (ok && warp == 4 && lane == 0) LSQ_KTL(5, it);
    }

  }

  // ------------------------------------------------------------ epilogue (all 12 warps)
  // Every warp joins once the accumulator is complete: warp w reads TMEM lane
  // quarter w % 4 (32 features) and takes every third 32-token chunk of that
  // quarter (w / 4 selects which); it stages a chunk in one of four private
  // shared-memory slots of the drained pipeline and writes it with TMA stores of
  // [16 tokens x 32 features] boxes, so no warp waits for another.  Residual
  // tiles arrive by TMA into the slot, the next chunk's while this one stores.
  {
    pdl_wait();  // the residual and the output buffers belong to the kernels before
    bool acc_ok = mbar_wait_bounded(smem_u32(&bar_acc), 0u, abort_flag, p.dev_err,
                                    DEV_ERR_WAIT_GEMM);
    acc_ok = __all_sync(0xFFFFFFFFu, acc_ok && (*abort_flag == 0));
    if (warp == 4 && lane == 0) LSQ_STAMP(4, globaltimer_ns());
    if (acc_ok) {
      tc_fence_after();
      const int qtr = warp & 3;          // TMEM lane quarter = features 32 qtr .. +31
      const int part = warp >> 2;        // chunks q with q % 3 == part
      const uint32_t tbase = tmem + ((uint32_t)(qtr * 32) << 16);
      const bool partial = p.splits > 1;
      const bool f32 = partial || p.out_f32;
      const int es = f32 ? 4 : 2;
      const bool res = !partial && p.residual != nullptr;  // fp32, with an fp32 output
      bool big = false;  // an fp16 output beyond the fp16 range
      const uint32_t sub_bytes = 16u * 32u * (uint32_t)es;   // one [16 x 32] box
      // 4 slots of <= 4 KB: a slot is written again only after the store of the chunk
      // four back has read it, so stores stay in flight while the next chunks drain
      uint8_t* myslots = dsm + (size_t)warp * 16384;
      const uint32_t rbar = smem_u32(&bar_res[warp]);
      const int mcol = m0 + qtr * 32;
      // this warp's chunks (at most 6: 2 accumulators x 8 chunks / 3)
      int ma[8], mc[8], nm = 0;
      {
        int q = 0;
        for (int a = 0; a < p.nacc; ++a)
          for (int c0 = 0; c0 < p.bn; c0 += 32, ++q) {
            if (t0 + a * p.bn + c0 >= p.T) break;
            if (q % 3 == part && nm < 8) {
              ma[nm] = a;
              mc[nm] = c0;
              ++nm;
            }
          }
      }
      auto issue_res = [&](int i) {  // lane 0: residual of my chunk i into slot i & 3
        const int tb = t0 + ma[i] * p.bn + mc[i];
        const int nsub = (p.bn - mc[i] >= 32) ? 2 : 1;
        uint8_t* slot = myslots + (i & 3) * (2 * sub_bytes);
        mbar_arrive_expect_tx(rbar, (uint32_t)nsub * sub_bytes);
        for (int sb = 0; sb < nsub; ++sb)
          tma_load_2d(smem_u32(slot + sb * sub_bytes), &tm_res, rbar, mcol, tb + 16 * sb);
      };
      if (res && nm > 0 && lane == 0) issue_res(0);
      for (int i = 0; i < nm && acc_ok; ++i) {
        const int a = ma[i], c0 = mc[i];
        const int tb = t0 + a * p.bn + c0;
        const int nsub = (p.bn - c0 >= 32) ? 2 : 1;   // 16-token sub-chunks
        uint8_t* slot = myslots + (i & 3) * (2 * sub_bytes);
        if (res) {
          acc_ok = mbar_wait_bounded(rbar, (uint32_t)(i & 1), abort_flag, p.dev_err,
                                     DEV_ERR_WAIT_GEMM);
          acc_ok = __all_sync(0xFFFFFFFFu, acc_ok);
          if (!acc_ok) break;
        } else {
          if (i >= 4 && lane == 0) bulk_wait_read<3>();  // the store that used this slot has read it
          __syncwarp();
        }
        uint32_t rg[2][16];
        tmem_ld16(tbase + (uint32_t)a * acc_stride + (uint32_t)c0, rg[0]);
        if (nsub == 2) tmem_ld16(tbase + (uint32_t)a * acc_stride + (uint32_t)c0 + 16, rg[1]);
        tmem_ld_wait();
        for (int sb = 0; sb < nsub; ++sb) {
          uint8_t* base = slot + sb * sub_bytes;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float v = __uint_as_float(rg[sb][j]);
            if (f32) {
              float* d = reinterpret_cast<float*>(base + (j * 32 + lane) * 4);
              if (res) v += *d;
              *d = v;
            } else if (F16) {
              big |= !(fabsf(v) <= kF16Max);
              *reinterpret_cast<uint16_t*>(base + (j * 32 + lane) * 2) = float_to_f16_bits(v);
            } else {
              *reinterpret_cast<uint16_t*>(base + (j * 32 + lane) * 2) = float_to_bf16_bits(v);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int sb = 0; sb < nsub; ++sb) {
            if (tb + 16 * sb >= p.T) break;
            if (partial)
              tma_store_3d(&tm_out, smem_u32(slot + sb * sub_bytes), mcol, tb + 16 * sb, split);
            else
              tma_store_2d(&tm_out, smem_u32(slot + sb * sub_bytes), mcol, tb + 16 * sb);
          }
          bulk_commit();
          if (res && i + 1 < nm) {
            bulk_wait_read<3>();  // chunk i - 3's store has read slot (i + 1) & 3
            issue_res(i + 1);
          }
        }
        __syncwarp();
      }
      if (lane == 0) bulk_wait_all();
      if (warp == 4 && lane == 0) LSQ_STAMP(5, globaltimer_ns());
      if (__any_sync(0xFFFFFFFFu, big) && lane == 0) atomicOr(p.dev_err, DEV_ERR_NONFINITE);
      __syncwarp();
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (abort_sh) settle_ns(2000000);  // let issued copies and MMAs land before freeing TMEM
  // The even CTA's MMAs read the odd CTA's shared memory and write its TMEM:
  // neither leaves (or frees TMEM) before both are here.
  if (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, p.alloc_cols);
    else
      tmem_dealloc(tmem, p.alloc_cols);
  }
  if (threadIdx.x == 0) LSQ_STAMP(6, globaltimer_ns());
}

// ------------------------------------------------------------------ host side
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(f);
  });
  return fn;
}

int make_tmap(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base,
              uint64_t inner, uint64_t rows, uint64_t row_stride_elems, uint32_t box_inner,
              uint32_t box_rows, CUtensorMapSwizzle sw) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return set_error(LSQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_elems * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(LSQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): inner=%llu rows=%llu",
                     (int)r, (unsigned long long)inner, (unsigned long long)rows);
  return LSQ_OK;
}

struct Plan {
  int bn, nacc, t_tiles, m_tiles, kt_total, kt_per_split, splits, stages, ring_stages;
  bool pair;  // CTA pairs with cta_group::2 MMAs (M = 256 per pair)
  uint32_t ring_bytes, smem_bytes, alloc_cols;
  uint32_t xs_bytes;  // activation bytes of one stage, per CTA
  size_t partial_bytes;
};

int g_num_sms = 0;

// CTA pairs are used unless LSQ_GEMM_PAIR=0 is set in the environment (which
// selects the one-CTA kernel, e.g. to compare the two).
bool pair_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LSQ_GEMM_PAIR");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

// The launch plan for `sms` SMs; allow_pair = false asks for one-CTA tiles.
Plan make_plan(const GemmDesc& d, int sms, bool allow_pair) {
  Plan pl{};
  const int64_t T = d.T;
  pl.m_tiles = (int)((d.M + kBM - 1) / kBM);
  pl.pair = allow_pair && pl.m_tiles >= 2;
  const int64_t gran = pl.pair ? 32 : 16;  // a pair splits each accumulator's tokens in two
  if (T <= 256) {
    pl.nacc = 1;
    pl.bn = (int)((T + gran - 1) / gran * gran);
  } else {
    pl.nacc = 2;
    const int64_t half = (std::min<int64_t>(T, 512) + 1) / 2;
    pl.bn = (int)std::min<int64_t>(256, (half + gran - 1) / gran * gran);
  }
  if (pl.pair) pl.m_tiles = (pl.m_tiles + 1) / 2 * 2;
  const int BT = pl.nacc * pl.bn;
  pl.t_tiles = (int)((T + BT - 1) / BT);
  pl.kt_total = (int)((d.Kc + kBK - 1) / kBK);
  const int base = pl.m_tiles * pl.t_tiles;
  int splits = 1;
  if (d.force_splits > 0) {
    splits = d.force_splits;
  } else if (base < sms) {
    splits = std::max(1, std::min(sms / base, pl.kt_total / 4));
    splits = std::min(splits, 16);
  }
  splits = std::max(1, std::min(splits, pl.kt_total));
  pl.kt_per_split = (pl.kt_total + splits - 1) / splits;
  pl.splits = (pl.kt_total + pl.kt_per_split - 1) / pl.kt_per_split;
  pl.partial_bytes = pl.splits > 1 ? (size_t)pl.splits * (size_t)T * (size_t)d.M * 4 : 0;
  const bool w_tma = d.wmode == W_BF16_N || d.wmode == W_BF16_T || d.wmode == W_BF16C_N;
  pl.ring_bytes = w_tma ? 0 : 4096;
  const uint32_t xs = (uint32_t)(pl.pair ? BT / 2 : BT) * 128;
  pl.xs_bytes = xs;
  int ring = w_tma ? 0 : kMaxRing;
  int stages = kMaxStages;
  auto total = [&](int st, int rs) {
    return 1024u + (uint32_t)st * (xs + kWStageBytes) + (uint32_t)rs * pl.ring_bytes +
           kAmRingBytes;
  };
  // Operand stages before codes-ring depth: at 512 tokens per tile, 4 stages with a
  // 3-deep ring run the transposed (input-gradient) NF4 product 4-7% faster than
  // 3 stages with an 8-deep ring, and the forward product as fast.
  while (ring > 2 && total(stages, ring) > kSmemBudget - 4096) --ring;
  while (stages > 2 && total(stages, ring) > kSmemBudget - 4096) --stages;
  pl.stages = stages;
  pl.ring_stages = std::max(ring, 1);
  pl.smem_bytes = std::max(total(stages, ring), kEpilogueBytes);
  uint32_t cols = 32;
  while (cols < (uint32_t)pl.bn) cols <<= 1;
  pl.alloc_cols = (pl.nacc > 1) ? 512u : cols;
  return pl;
}

template <int WMODE, bool PAIR>
int launch_mode(const GemmDesc& d, const Plan& pl, float* partial, cudaStream_t st) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    LSQ_CUDA(cudaFuncSetAttribute(tc_gemm_kernel<WMODE, PAIR>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kDynSmemLimit));
    attr_done[dev] = true;
  }
  constexpr bool F16 = wmode_f16(WMODE);
  const CUtensorMapDataType dt16 =
      F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tm_act, tm_w;
  LSQ_TRY(make_tmap(&tm_act, dt16, 2, d.act, (uint64_t)d.Kc,
                    (uint64_t)d.T, (uint64_t)d.act_ld, kBK, (uint32_t)(PAIR ? pl.bn / 2 : pl.bn),
                    CU_TENSOR_MAP_SWIZZLE_128B));
  if (WMODE == W_NF4_N)
    LSQ_TRY(make_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d.w, (uint64_t)d.w_cols / 2,
                      (uint64_t)d.w_rows, (uint64_t)d.w_cols / 2, 32, kBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE));
  if (WMODE == W_NF4_T)
    LSQ_TRY(make_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d.w, (uint64_t)d.w_cols / 2,
                      (uint64_t)d.w_rows, (uint64_t)d.w_cols / 2, 64, 64,
                      CU_TENSOR_MAP_SWIZZLE_NONE));
  if (WMODE == W_BF16_N || WMODE == W_BF16C_N)
    LSQ_TRY(make_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.w, (uint64_t)d.w_cols,
                      (uint64_t)d.w_rows, (uint64_t)d.w_cols, kBK, kBM,
                      CU_TENSOR_MAP_SWIZZLE_128B));
  if (WMODE == W_BF16_T)  // [64 contraction rows x 64 features] atoms, 128-byte swizzle
    LSQ_TRY(make_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.w, (uint64_t)d.w_cols,
                      (uint64_t)d.w_rows, (uint64_t)d.w_cols, 64, kBK,
                      CU_TENSOR_MAP_SWIZZLE_128B));
  CUtensorMap tm_out, tm_res;
  if (partial) {
    PFN_encodeTiled enc = get_encode();
    if (!enc) return set_error(LSQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)d.M, (cuuint64_t)d.T, (cuuint64_t)pl.splits};
    cuuint64_t strides[2] = {(cuuint64_t)d.M * 4, (cuuint64_t)d.M * (cuuint64_t)d.T * 4};
    cuuint32_t box[3] = {32, 16, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&tm_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, partial, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return set_error(LSQ_ERR_CUDA, "cuTensorMapEncodeTiled (partials) failed (%d)", (int)r);
  } else if (d.out_f32) {
    LSQ_TRY(make_tmap(&tm_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d.out, (uint64_t)d.M,
                      (uint64_t)d.T, (uint64_t)d.ldo, 32, 16, CU_TENSOR_MAP_SWIZZLE_NONE));
  } else {
    LSQ_TRY(make_tmap(&tm_out, dt16, 2, d.out, (uint64_t)d.M, (uint64_t)d.T, (uint64_t)d.ldo, 32,
                      16, CU_TENSOR_MAP_SWIZZLE_NONE));
  }
  if (d.residual && !partial)
    LSQ_TRY(make_tmap(&tm_res, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d.residual, (uint64_t)d.M,
                      (uint64_t)d.T, (uint64_t)d.ldr, 32, 16, CU_TENSOR_MAP_SWIZZLE_NONE));
  else
    tm_res = tm_out;  // unused
  CUtensorMap tm_la = tm_out, tm_lb = tm_out;  // unused without a slab
  if (d.slab_w > 0) {
    LSQ_TRY(make_tmap(&tm_la, dt16, 2, d.la16, (uint64_t)d.slab_w, (uint64_t)d.M,
                      (uint64_t)d.la16_ld, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B));
    LSQ_TRY(make_tmap(&tm_lb, dt16, 2, d.lb16, (uint64_t)d.slab_w, (uint64_t)d.T,
                      (uint64_t)d.lb16_ld, kBK, (uint32_t)(PAIR ? pl.bn / 2 : pl.bn),
                      CU_TENSOR_MAP_SWIZZLE_128B));
  }
  KParams p{};
  p.M = (int)d.M;
  p.T = (int)d.T;
  p.Kc = (int)d.Kc;
  p.bn = pl.bn;
  p.nacc = pl.nacc;
  p.stages = pl.stages;
  p.ring_stages = pl.ring_stages;
  p.kt_total = pl.kt_total;
  p.kt_per_split = pl.kt_per_split;
  p.splits = pl.splits;
  p.ring_bytes = pl.ring_bytes;
  p.alloc_cols = pl.alloc_cols;
  p.absmax = d.absmax;
  p.am_q = d.absmax_q;
  p.am_s = d.absmax_s;
  p.w_rows = (int)d.w_rows;
  p.w_cols = (int)d.w_cols;
  p.slab_w = d.slab_w;
  p.out = d.out;
  p.out_f32 = d.out_f32;
  p.ldo = d.ldo;
  p.residual = d.residual;
  p.ldr = d.ldr;
  p.partial = partial;
  p.dev_err = device_status_ptr();
  const float* lv = nf4_levels();
  for (int i = 0; i < 16; ++i) p.levels[i] = lv[i];
  if (!p.dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.m_tiles, pl.t_tiles, pl.splits);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  LSQ_CUDA(::lsq::launched(
      cudaLaunchKernelEx(&cfg, tc_gemm_kernel<WMODE, PAIR>, tm_act, tm_w, tm_out, tm_res, tm_la,
                         tm_lb, p)));
  return LSQ_OK;
}

}  // namespace

int make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base,
                 uint64_t inner, uint64_t rows, uint64_t row_stride_elems, uint32_t box_inner,
                 uint32_t box_rows, CUtensorMapSwizzle sw) {
  return make_tmap(m, dt, elem_bytes, base, inner, rows, row_stride_elems, box_inner, box_rows, sw);
}

int gemm_num_sms() {
  if (g_num_sms == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_num_sms = n > 0 ? n : 148;
  }
  return g_num_sms;
}

int* device_status_ptr() {
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_lsq_dev_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(a);
  }
  return ptrs[dev];
}

#ifdef LSQ_GEMM_KTL
}  // namespace lsq
// Diagnostic build only: copies the per-k-tile timeline of the last launch
// (2 CTAs x 8 rows x 256 k-tiles) to host.
extern "C" int lsq_debug_gemm_ktl(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, lsq::g_gemm_ktl, sizeof(lsq::g_gemm_ktl)) == cudaSuccess ? 0
                                                                                             : 3;
}
namespace lsq {
#endif

#ifdef LSQ_GEMM_STAMPS
}  // namespace lsq
// Diagnostic build only: copies the stamps of the last launch (kStampCtas x 8) to host.
extern "C" int lsq_debug_gemm_stamps(unsigned long long* out) {
  return cudaMemcpyFromSymbol(out, lsq::g_gemm_stamps, sizeof(lsq::g_gemm_stamps)) == cudaSuccess
             ? 0 : 3;
}
namespace lsq {
#endif

size_t gemm_workspace_bytes(const GemmDesc& d) {
  if (d.M <= 0 || d.T <= 0 || d.Kc <= 0) return 0;
  return make_plan(d, gemm_num_sms(), pair_enabled()).partial_bytes;
}

int gemm_run(const GemmDesc& d, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (d.M <= 0 || d.T <= 0 || d.Kc <= 0) return set_error(LSQ_ERR_SHAPE, "gemm: empty problem");
  if (!d.w || !d.act || !d.out) return set_error(LSQ_ERR_INVALID, "gemm: null operand");
  if ((d.wmode == W_NF4_N || d.wmode == W_NF4_T) && !d.absmax && !(d.absmax_q && d.absmax_s))
    return set_error(LSQ_ERR_INVALID, "gemm: null absmax");
  if (d.w_cols % 64 != 0 && (d.wmode == W_NF4_N || d.wmode == W_NF4_T))
    return set_error(LSQ_ERR_SHAPE, "gemm: NF4 weight columns must be a multiple of 64");
  if (d.act_ld % 8 != 0 || d.w_cols % 8 != 0)
    return set_error(LSQ_ERR_SHAPE, "gemm: row strides must be multiples of 16 bytes");
  if (d.slab_w % 16 != 0 || d.slab_w < 0)
    return set_error(LSQ_ERR_SHAPE, "gemm: LoRA slab width must be a multiple of 16");
  if (d.slab_w > 0 && (!d.la16 || !d.lb16))
    return set_error(LSQ_ERR_INVALID, "gemm: null LoRA slab");
  if (d.slab_w > 0 && (d.la16_ld % 8 != 0 || d.lb16_ld % 8 != 0 || d.la16_ld < d.slab_w ||
                       d.lb16_ld < d.slab_w))
    return set_error(LSQ_ERR_SHAPE, "gemm: 16-bit LoRA slab operands need row strides >= the "
                                    "slab width, multiples of 8");
  if (d.residual && !d.out_f32) return set_error(LSQ_ERR_INVALID, "gemm: residual needs an fp32 output");
  if (d.ldo % 8 != 0 || (d.residual && d.ldr % 8 != 0))
    return set_error(LSQ_ERR_SHAPE, "gemm: output strides must be multiples of 16 bytes");
  if (d.M > INT32_MAX || d.T > INT32_MAX || d.Kc > INT32_MAX)
    return set_error(LSQ_ERR_SHAPE, "gemm: dimension too large");
  Plan pl = make_plan(d, gemm_num_sms(), pair_enabled());
  float* partial = nullptr;
  if (pl.splits > 1) {
    if (!ws || ws_bytes < pl.partial_bytes)
      return set_error(LSQ_ERR_WORKSPACE, "gemm: split-K workspace %zu < %zu", ws_bytes,
                       pl.partial_bytes);
    partial = static_cast<float*>(ws);
  }
  const int prof = prof_begin(st);
  switch (d.wmode) {
    case W_NF4_N:
      LSQ_TRY((pl.pair ? launch_mode<W_NF4_N, true>(d, pl, partial, st)
                       : launch_mode<W_NF4_N, false>(d, pl, partial, st)));
      break;
    case W_NF4_T:
      LSQ_TRY((pl.pair ? launch_mode<W_NF4_T, true>(d, pl, partial, st)
                       : launch_mode<W_NF4_T, false>(d, pl, partial, st)));
      break;
    case W_BF16_N:
      LSQ_TRY((pl.pair ? launch_mode<W_BF16_N, true>(d, pl, partial, st)
                       : launch_mode<W_BF16_N, false>(d, pl, partial, st)));
      break;
    case W_BF16_T:
      LSQ_TRY((pl.pair ? launch_mode<W_BF16_T, true>(d, pl, partial, st)
                       : launch_mode<W_BF16_T, false>(d, pl, partial, st)));
      break;
    case W_BF16C_N:
      LSQ_TRY((pl.pair ? launch_mode<W_BF16C_N, true>(d, pl, partial, st)
                       : launch_mode<W_BF16C_N, false>(d, pl, partial, st)));
      break;
    default: return set_error(LSQ_ERR_INVALID, "gemm: bad operand mode");
  }
  if (d.splits_out) *d.splits_out = pl.splits;
  if (d.parts_out) *d.parts_out = pl.splits > 1 ? partial : nullptr;
  if (pl.splits > 1 && !d.parts_out)
    LSQ_TRY(launch_splitk_reduce(partial, pl.splits, d.T, d.M, d.out,
                                 d.out_f32 ? OUT_F32 : (wmode_f16(d.wmode) ? OUT_F16 : OUT_BF16),
                                 d.ldo, d.residual, d.ldr, st));
  if (prof >= 0) {
    // algorithmic work: the contraction plus the LoRA slab; minimum DRAM traffic:
    // the weight once, the activation once, the output (and residual) once
    const double M = (double)d.M, T = (double)d.T, K = (double)d.Kc;
    const double flops = 2.0 * M * T * (K + d.slab_w);
    const bool nf4 = d.wmode == W_NF4_N || d.wmode == W_NF4_T;
    const double am_bytes = d.absmax_q ? 1.0 / 64.0 + 4.0 / (64.0 * 256.0) : 4.0 / 64.0;
    const double wbytes = nf4 ? M * K * (0.5 + am_bytes) : 2.0 * M * K;
    const double bytes = wbytes + 2.0 * T * K + T * M * (d.out_f32 ? 4.0 : 2.0) +
                         (d.residual ? 4.0 * T * M : 0.0);
    static const char* names[5] = {"gemm_nf4_fwd", "gemm_nf4_dx", "gemm_bf16_fwd",
                                   "gemm_bf16_dx", "gemm_bf16_fwd"};
    prof_end(prof, st, d.prof_name ? d.prof_name : names[d.wmode], flops, bytes);
  }
  return LSQ_OK;
}

}  // namespace lsq

extern "C" int lsq_gemm_plan_get(int32_t mode, int64_t M, int64_t T, int64_t Kc, int32_t num_sms,
                                 int32_t allow_pair, lsq_gemm_plan* out) {
  using namespace lsq;
  if (!out) return set_error(LSQ_ERR_INVALID, "lsq_gemm_plan_get: null output");
  if (mode < W_NF4_N || mode > W_BF16C_N)
    return set_error(LSQ_ERR_INVALID, "lsq_gemm_plan_get: bad operand mode %d", (int)mode);
  if (M <= 0 || T <= 0 || Kc <= 0 || num_sms <= 0 || M > INT32_MAX || T > INT32_MAX ||
      Kc > INT32_MAX)
    return set_error(LSQ_ERR_SHAPE, "lsq_gemm_plan_get: bad size");
  GemmDesc d;
  d.wmode = mode;
  d.M = M;
  d.T = T;
  d.Kc = Kc;
  const Plan pl = make_plan(d, num_sms, allow_pair != 0);
  lsq_gemm_plan o{};
  o.pair = pl.pair ? 1 : 0;
  o.bn = pl.bn;
  o.nacc = pl.nacc;
  o.m_tiles = pl.m_tiles;
  o.t_tiles = pl.t_tiles;
  o.splits = pl.splits;
  o.kt_total = pl.kt_total;
  o.kt_per_split = pl.kt_per_split;
  o.stages = pl.stages;
  o.ring_stages = pl.ring_stages;
  o.x_stage_bytes = (int32_t)pl.xs_bytes;
  o.w_stage_bytes = kWStageBytes;
  o.ring_bytes = (int32_t)pl.ring_bytes;
  o.absmax_ring_bytes = (int32_t)kAmRingBytes;
  o.smem_bytes = (int32_t)pl.smem_bytes;
  o.smem_limit = (int32_t)kDynSmemLimit;
  o.epilogue_bytes = (int32_t)kEpilogueBytes;
  o.tmem_cols = (int32_t)pl.alloc_cols;
  o.partial_bytes = (int64_t)pl.partial_bytes;
  *out = o;
  return LSQ_OK;
}

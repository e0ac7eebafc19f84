// LoRA rank-r products around the fused NF4 GEMM, on 5th-generation tensor cores.
//
// For y = x W^T + s (x A^T) B^T (Soup layer-streaming tutorial, "四段資料路徑"
// part 1) and its backward (part 3): u = x A^T (forward), v = dY B, and the
// trainable gradients dA = s v^T x, dB = s dY^T u.  All four are "tall x
// skinny" products C[m, n] = sum_k A(m, k) B(n, k) with n spanning the rank
// (r to 3 r columns, up to 192) and m and k the long dimensions.
//
// One kernel serves all four: a CTA owns 128 rows of C and up to 256 columns
// (all of them for ranks up to 256), over one slice of the reduction.  A (the activation or gradient, 128 x 64 per
// stage) and B (the rank-side operand, n_pad x 64) arrive by TMA in the
// 128-byte-swizzle layout; one thread issues tcgen05.mma (M = 128, N = n_pad,
// K = 16) into a TMEM accumulator; the four warps read it back in the epilogue.
// A is K-major for u and v (x, dY read along their rows) and MN-major for dA and
// dB (x, dY read along their columns, the reduction running over tokens).  B is
// always K-major: the products that feed dA and dB store their 16-bit result
// transposed (u16, v16: [R][ld] with ld = T rounded up to 8), and the B operand
// of v is stored transposed too ([R][N]), so the rank is never the swizzled
// dimension.  Operand types follow the activations: u = x A^T multiplies fp16;
// v, dA and dB multiply bf16 (each has a gradient operand, which needs bf16's
// range); dA's fp16 activation is converted to bf16 in shared memory as each
// stage lands.  Accumulation is fp32 (the tutorial's part 1: the LoRA A/B
// matrices are computed at a higher precision than the NF4 storage).  When a
// product is split along its reduction (into 2, 4 or 8 slices), the slices of a
// tile run as one thread-block cluster: each copies its accumulator into its
// shared memory, and after a cluster barrier each sums its share of the tile's
// rows over the slices, in slice order, through distributed shared memory.  No
// partials leave the SMs, no second kernel runs, and the results are
// deterministic (no atomics).
#include <cuda.h>
#include <stdlib.h>

#include "common.cuh"

namespace lsq {

namespace {

constexpr int kSM = 128;       // rows of C per CTA (UMMA M)
constexpr int kSK = 64;        // reduction per stage: one 128-byte swizzle atom of 16-bit values
constexpr int kSThreads = 128;
constexpr int kSMs = 148;
constexpr int kSMaxN = 256;    // columns per CTA (one MMA's N); wider products tile the columns
constexpr uint32_t kSAStage = kSM * kSK * 2;  // 16 KB

struct SkinnyArgs {
  int64_t M, N, K;     // C is M x N, reduction over K
  int splits;          // slices of the reduction = CTAs of a cluster (1, 2, 4 or 8); slice
                       // z takes the stages [z kt / splits, (z + 1) kt / splits) of kt
  // unsplit: dst[m * c_m + n * c_n] = alpha * C[m, n] (+ dst if accumulate)
  float* dst;
  int64_t c_m, c_n;
  float alpha;
  int accumulate;
  // Output options (applied where the result is written): c16 (nullable) also receives the result rounded to bf16,
  // c16[m * c16_m + n * c16_n], for the product that consumes it; with part_r >
  // 0 the rows are split into parts ending at part_end[], and row m of part p
  // keeps only columns [p part_r, (p + 1) part_r), written to column n - p part_r.
  uint16_t* c16;
  int64_t c16_m, c16_n;
  // h16 (nullable): the result rounded to fp16 (h16_f16) or bf16 at
  // h16[m * h16_m + n * h16_n] - the LoRA slab operand of the fused GEMM
  uint16_t* h16;
  int64_t h16_m, h16_n;
  int h16_f16;
  int part_r, n_parts;
  int64_t part_end[4];
};

// Writes one result element of row m, column n (see SkinnyArgs).
__device__ __forceinline__ void store_result(const SkinnyArgs& a, int64_t m, int64_t n, float v) {
  int64_t col = n;
  if (a.part_r > 0) {
    int p = 0;
    while (p + 1 < a.n_parts && m >= a.part_end[p]) ++p;
    col = n - (int64_t)p * a.part_r;
    if (col < 0 || col >= a.part_r) return;
  }
  if (a.dst) {
    float* d = a.dst + m * a.c_m + col * a.c_n;
    *d = (a.accumulate ? *d : 0.f) + a.alpha * v;
  }
  if (a.c16) a.c16[m * a.c16_m + n * a.c16_n] = float_to_bf16_bits(v);
  if (a.h16)
    a.h16[m * a.h16_m + n * a.h16_n] = a.h16_f16 ? float_to_f16_bits(v) : float_to_bf16_bits(v);
}

__device__ __forceinline__ uint8_t* align1024_s(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// A_MN: A is MN-major (its m index contiguous in memory).  One launch may carry two
// products of the same width and reduction (the dA and dB of a projection group):
// the first tiles1 row tiles (grid.x) are the first product's (tm_a, tm_b, a0), the
// rest the second's (tm_a2, tm_b2, a1).  Bit i of conv_mask: product i's A is stored
// fp16 and converted to bf16 in shared memory before the MMA reads it.
//   warp 0: TMA producer (lane 0);  warp 1: TMEM and the MMA issuer (lane 0);
//   warps 2-3: the conversion; all four: the epilogue (TMEM lane quarter = warp)
template <bool A_MN>
__global__ void __launch_bounds__(kSThreads, 1)
    tc_skinny_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_a2,
                     const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ SkinnyArgs a0,
                     const __grid_constant__ SkinnyArgs a1, int tiles1, int conv_mask,
                     uint32_t idesc, int n_pad, int stages, uint32_t tmem_cols, int* dev_err) {
  extern __shared__ uint8_t sk_raw[];
  constexpr int kMaxSt = 4;
  __shared__ __align__(8) uint64_t bar_full[kMaxSt], bar_conv[kMaxSt], bar_empty[kMaxSt], bar_acc;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  volatile int* abort_flag = &abort_sh;
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t b_bytes = (uint32_t)n_pad * 128u;
  uint8_t* st0 = align1024_s(sk_raw);
  const uint32_t st_bytes = kSAStage + ((b_bytes + 1023u) & ~1023u);
  const bool second = (int)blockIdx.x >= tiles1;
  const SkinnyArgs& a = second ? a1 : a0;
  const CUtensorMap* tma = second ? &tm_a2 : &tm_a;
  const CUtensorMap* tmb = second ? &tm_b2 : &tm_b;
  const bool CONV = ((conv_mask >> (second ? 1 : 0)) & 1) != 0;
  const int64_t m0 = (int64_t)((int)blockIdx.x - (second ? tiles1 : 0)) * kSM;
  const int kt_total = (int)((a.K + kSK - 1) / kSK);
  const int kt_begin = (int)((int64_t)blockIdx.z * kt_total / a.splits);
  const int n_it = (int)((int64_t)(blockIdx.z + 1) * kt_total / a.splits) - kt_begin;
  const int S = stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_conv[s]), 2);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    mbar_init(smem_u32(&bar_acc), 1);
    abort_sh = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_sh), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();  // both operands come from the kernels before
      for (int it = 0; it < n_it; ++it) {
        const int s = it % S;
        if (!mbar_wait_bounded(smem_u32(&bar_empty[s]), (uint32_t)((it / S) & 1) ^ 1u, abort_flag,
                               dev_err, DEV_ERR_WAIT_GEMM))
          break;
        const int k0 = (kt_begin + it) * kSK;
        uint8_t* sa = st0 + (size_t)s * st_bytes;
        const uint32_t fb = smem_u32(&bar_full[s]);
        mbar_arrive_expect_tx(fb, kSAStage + b_bytes);
        if (A_MN) {  // two [64 k x 64 m] boxes, 64 m apart
          tma_load_2d(smem_u32(sa), tma, fb, (int)m0, k0);
          tma_load_2d(smem_u32(sa + kSAStage / 2), tma, fb, (int)m0 + 64, k0);
        } else {     // one [128 m x 64 k] box
          tma_load_2d(smem_u32(sa), tma, fb, k0, (int)m0);
        }
        tma_load_2d(smem_u32(sa + kSAStage), tmb, fb, k0, (int)blockIdx.y * n_pad);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int s = it % S;
        const uint32_t ph = (uint32_t)((it / S) & 1);
        if (!mbar_wait_bounded(smem_u32(CONV ? &bar_conv[s] : &bar_full[s]), ph, abort_flag,
                               dev_err, DEV_ERR_WAIT_GEMM))
          break;
        tc_fence_after();
        const uint32_t sa = smem_u32(st0 + (size_t)s * st_bytes);
#pragma unroll
        for (int kk = 0; kk < kSK / 16; ++kk) {
          const uint64_t ad = A_MN ? umma_desc_mn_sw128(sa + (uint32_t)kk * 16 * 128, kSAStage / 2, 1024u)
                                   : umma_desc_k_sw128(sa + (uint32_t)kk * 32);
          const uint64_t bd = umma_desc_k_sw128(sa + kSAStage + (uint32_t)kk * 32);
          tc_mma_bf16(tmem, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&bar_empty[s]));
      }
      tc_commit(smem_u32(&bar_acc));
    }
    __syncwarp();
  } else if (CONV) {
    // warps 2-3: each landed A stage from fp16 to bf16, in place
    const int tid = threadIdx.x - 64;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % S;
      bool ok = mbar_wait_bounded(smem_u32(&bar_full[s]), (uint32_t)((it / S) & 1), abort_flag,
                                  dev_err, DEV_ERR_WAIT_GEMM);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      uint8_t* sa = st0 + (size_t)s * st_bytes;
      for (uint32_t o = (uint32_t)tid * 16u; o < kSAStage; o += 64u * 16u) {
        uint4 v = *reinterpret_cast<uint4*>(sa + o);
        v.x = f16x2_to_bf16x2(v.x);
        v.y = f16x2_to_bf16x2(v.y);
        v.z = f16x2_to_bf16x2(v.z);
        v.w = f16x2_to_bf16x2(v.w);
        *reinterpret_cast<uint4*>(sa + o) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_conv[s]));
    }
  }

  // ------------------------------------------------------------------ epilogue
  const int Z = a.splits;
  bool ok = mbar_wait_bounded(smem_u32(&bar_acc), 0u, abort_flag, dev_err, DEV_ERR_WAIT_GEMM);
  ok = __all_sync(0xFFFFFFFFu, ok);
  tc_fence_after();
  const int64_t nc = (int64_t)blockIdx.y * n_pad;  // first column of this CTA
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  if (Z == 1) {
    if (ok) {
      const int64_t m = m0 + warp * 32 + lane;  // this thread's row (its TMEM lane)
      for (int n0 = 0; n0 < n_pad; n0 += 16) {
        uint32_t v[16];
        tmem_ld16(trow + (uint32_t)n0, v);
        tmem_ld_wait();
        if (m >= a.M) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (nc + n0 + j < a.N) store_result(a, m, nc + n0 + j, __uint_as_float(v[j]));
      }
    }
  } else {
    // The accumulator into this CTA's shared memory (the drained pipeline),
    // [128 rows][n_pad + 4] fp32 ...
    float* red = reinterpret_cast<float*>(st0);
    const int ldr = n_pad + 4;
    if (ok) {
      const int row = warp * 32 + lane;
      for (int n0 = 0; n0 < n_pad; n0 += 16) {
        uint32_t v[16];
        tmem_ld16(trow + (uint32_t)n0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4*>(red + row * ldr + n0 + j) =
              make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                          __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
      }
    }
    // ... then every slice of the tile sums its share of the rows over all
    // slices, in slice order, through distributed shared memory.
    cluster_sync_all();
    const int cr = (int)cluster_ctarank();  // = this CTA's slice
    const int rows = kSM / Z, n4 = n_pad / 4;
    if (ok && !abort_sh) {
      for (int e = threadIdx.x; e < rows * n4; e += kSThreads) {
        const int row = cr * rows + e / n4, c4 = e % n4;
        const int64_t m = m0 + row;
        if (m >= a.M) continue;
        const uint32_t off = smem_u32(red + row * ldr + 4 * c4);
        float4 acc = ld_shared_cluster_f4(mapa_shared(off, 0));
        for (int q = 1; q < Z; ++q) {
          const float4 v = ld_shared_cluster_f4(mapa_shared(off, (uint32_t)q));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        const float r4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (nc + 4 * c4 + j < a.N) store_result(a, m, nc + 4 * c4 + j, r4[j]);
      }
    }
    cluster_sync_all();  // no CTA leaves while another reads its shared memory
  }
  tc_fence_before();
  __syncthreads();
  if (abort_sh) settle_ns(2000000);  // let issued copies and MMAs land before freeing TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// out[i * ld_out + j] = fp16 of in[i * ld_in + j] for j < cols, 0 for cols <= j < ld_out
__global__ void to_f16_rows_kernel(const float* __restrict__ in, int64_t rows, int64_t cols,
                                   int64_t ld_in, uint16_t* __restrict__ out, int64_t ld_out) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t n_el = rows * ld_out;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / ld_out, j = i % ld_out;
    out[i] = float_to_f16_bits(j < cols ? in[r * ld_in + j] : 0.f);
  }
}

// out[j * rows + i] = bf16 of in[i * cols + j]: an [rows x cols] matrix transposed
__global__ void to_bf16_transposed_kernel(const float* __restrict__ in, int64_t rows,
                                          int64_t cols, uint16_t* __restrict__ out) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t n_el = rows * cols;
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < n_el;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = o / rows, i = o % rows;
    out[o] = float_to_bf16_bits(in[i * cols + j]);
  }
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }
// columns per CTA: the product's width rounded up to 16, at most 256
int npad_for(int64_t N) { return (int)std::min<int64_t>(kSMaxN, (N + 15) / 16 * 16); }

// Stages and CTAs per SM: four stages for every width; the widest tiles (n_pad up
// to 256, up to 48 KB a stage) run one CTA per SM, those up to 64 columns (24 KB a
// stage) two.  (Up to eight stages were measured: no faster, since the dA product
// is then paced by its in-place conversion.)
size_t stage_bytes(int n_pad) { return kSAStage + ((size_t)n_pad * 128 + 1023) / 1024 * 1024; }
int stages_for(int) { return 4; }
size_t smem_for(int n_pad) { return 1024 + (size_t)stages_for(n_pad) * stage_bytes(n_pad); }
int ctas_per_sm(int n_pad) { return smem_for(n_pad) <= 110 * 1024 ? 2 : 1; }

// Splits of the reduction (a cluster of 2, 4 or 8 CTAs per tile) on `sms` SMs: only
// where the product's own tiles leave at least half of the resident CTA slots
// empty, up to filling them, each slice at least two stages long.
int splits_for(int64_t M, int64_t N, int64_t K, int sms) {
  if (K <= 0 || M <= 0 || N <= 0) return 1;
  const int64_t tiles = (M + kSM - 1) / kSM * ((N + kSMaxN - 1) / kSMaxN);
  const int64_t slots = (int64_t)sms * ctas_per_sm(npad_for(N));
  if (tiles * 2 > slots) return 1;
  const int64_t kt = (K + kSK - 1) / kSK;
  const int64_t cap = std::min<int64_t>(8, std::min<int64_t>(slots / tiles, kt / 2));
  int z = 1;
  while (z * 2 <= cap) z *= 2;
  return z;
}

// One launch of one product (second == nullptr) or of two products of the same
// width and reduction length (dA and dB of a projection group) side by side.
template <bool A_MN>
int launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const SkinnyArgs& a, bool conv,
              const CUtensorMap* ta2, const CUtensorMap* tb2, const SkinnyArgs* a2, bool conv2,
              int tiles1, uint32_t idesc, int n_pad, dim3 grid, cudaStream_t st) {
  const size_t smem = smem_for(n_pad);
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr[dev]) {
    LSQ_CUDA(cudaFuncSetAttribute(tc_skinny_kernel<A_MN>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_for(kSMaxN)));
    attr[dev] = true;
  }
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  uint32_t cols = 32;
  while (cols < (uint32_t)n_pad) cols <<= 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;  // the slices of a tile
  at[1].val.clusterDim.x = 1;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = (unsigned)a.splits;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const int mask = (conv ? 1 : 0) | ((a2 ? conv2 : conv) ? 2 : 0);
  LSQ_CUDA(::lsq::launched(cudaLaunchKernelEx(
      &cfg, tc_skinny_kernel<A_MN>, ta, tb, ta2 ? *ta2 : ta, tb2 ? *tb2 : tb, a, a2 ? *a2 : a,
      a2 ? tiles1 : (int)grid.x, mask, idesc, n_pad, stages_for(n_pad), cols, dev_err)));
  return LSQ_OK;
}

// The operands of one product, as 2-D row-major 16-bit tensors.
struct Operand {
  const uint16_t* p;
  int64_t inner, rows, ld;  // elements per row, rows, row stride (elements)
  bool f16;
};

int tmaps_for(bool a_mn, const Operand& A, const Operand& B, int n_pad, CUtensorMap* ta,
              CUtensorMap* tb) {
  const CUtensorMapDataType dta = A.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapDataType dtb = B.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  LSQ_TRY(make_tmap_2d(ta, dta, 2, A.p, (uint64_t)A.inner, (uint64_t)A.rows, (uint64_t)A.ld, 64,
                       a_mn ? 64 : kSM, CU_TENSOR_MAP_SWIZZLE_128B));
  LSQ_TRY(make_tmap_2d(tb, dtb, 2, B.p, (uint64_t)B.inner, (uint64_t)B.rows, (uint64_t)B.ld, 64,
                       (uint32_t)n_pad, CU_TENSOR_MAP_SWIZZLE_128B));
  return LSQ_OK;
}

// C = A B^T over K (A: M x K, K-major unless A_MN; B: N x K, K-major), written as
// a prescribes (dst, alpha, accumulate, c16, parts).  CONV: A is fp16 and meets a
// bf16 B.
template <bool A_MN, bool CONV>
int run(SkinnyArgs a, const Operand& A, const Operand& B, bool f16, cudaStream_t st) {
  if (a.M <= 0 || a.N <= 0) return LSQ_OK;
  if (a.K <= 0) return set_error(LSQ_ERR_SHAPE, "lora product: empty reduction");
  const int n_pad = npad_for(a.N);
  const int z = splits_for(a.M, a.N, a.K, gemm_num_sms());  // slices of >= two stages
  a.splits = z;
  CUtensorMap ta, tb;
  LSQ_TRY(tmaps_for(A_MN, A, B, n_pad, &ta, &tb));
  uint32_t idesc = f16 ? umma_idesc_f16(kSM, n_pad) : umma_idesc_bf16(kSM, n_pad);
  if (A_MN) idesc |= 1u << 15;  // A MN-major
  const dim3 grid((unsigned)((a.M + kSM - 1) / kSM), (unsigned)((a.N + n_pad - 1) / n_pad),
                  (unsigned)z);
  return launch_tc<A_MN>(ta, tb, a, CONV, nullptr, nullptr, nullptr, false, 0, idesc, n_pad,
                         grid, st);
}

// Two token-reduction products (MN-major A, bf16) of the same width N and
// reduction K in one launch: the first's row tiles, then the second's.  The
// reduction is split for their tiles together.
int run_pair_mn(SkinnyArgs a, const Operand& A, bool conv, SkinnyArgs b, const Operand& Ab,
                bool conv_b, const Operand& B, const Operand& Bb, cudaStream_t st) {
  if (a.N <= 0 || a.N != b.N || a.K != b.K) return set_error(LSQ_ERR_SHAPE, "lora pair: widths");
  if (a.K <= 0) return set_error(LSQ_ERR_SHAPE, "lora product: empty reduction");
  const int n_pad = npad_for(a.N);
  const int64_t t1 = (a.M + kSM - 1) / kSM, t2 = (b.M + kSM - 1) / kSM;
  const int z = splits_for((t1 + t2) * kSM, a.N, a.K, gemm_num_sms());
  a.splits = b.splits = z;
  CUtensorMap ta, tb, ta2, tb2;
  LSQ_TRY(tmaps_for(true, A, B, n_pad, &ta, &tb));
  LSQ_TRY(tmaps_for(true, Ab, Bb, n_pad, &ta2, &tb2));
  const uint32_t idesc = umma_idesc_bf16(kSM, n_pad) | (1u << 15);  // A MN-major
  const dim3 grid((unsigned)(t1 + t2), (unsigned)((a.N + n_pad - 1) / n_pad), (unsigned)z);
  return launch_tc<true>(ta, tb, a, conv, &ta2, &tb2, &b, conv_b, (int)t1, idesc, n_pad, grid,
                         st);
}

int check_ranks(int64_t R) {
  if (R < 1)
    return set_error(LSQ_ERR_SHAPE, "lora: rank-r products need at least one column (got %lld)",
                     (long long)R);
  if (R % 8 != 0)
    return set_error(LSQ_ERR_SHAPE, "lora: product widths must be multiples of 8 (got %lld)",
                     (long long)R);
  return LSQ_OK;
}

SkinnyArgs out_args(float* dst, int64_t c_m, int64_t c_n, float alpha, int accumulate,
                    uint16_t* c16, int64_t c16_m, int64_t c16_n) {
  SkinnyArgs a{};
  a.dst = dst;
  a.c_m = c_m;
  a.c_n = c_n;
  a.alpha = alpha;
  a.accumulate = accumulate;
  a.c16 = c16;
  a.c16_m = c16_m;
  a.c16_n = c16_n;
  return a;
}

// 16-bit copies of fp32 LoRA operands, at the start of the scratch.
struct Split {
  uint16_t* q;
  float* rest;
  size_t rest_bytes;
};
int split_scratch(float* scratch, size_t bytes, size_t q_elems, Split* out, const char* who) {
  const size_t qb = align256(q_elems * 2);
  if (!scratch || bytes < qb)
    return set_error(LSQ_ERR_WORKSPACE, "%s: scratch %zu < %zu", who, bytes, qb);
  out->q = reinterpret_cast<uint16_t*>(scratch);
  out->rest = reinterpret_cast<float*>(reinterpret_cast<char*>(scratch) + qb);
  out->rest_bytes = bytes - qb;
  return LSQ_OK;
}

unsigned grid_for_elems(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > kSMs * 8) g = kSMs * 8;
  return (unsigned)std::max<int64_t>(1, g);
}

}  // namespace

int64_t lora16_ld(int64_t T) { return (T + 7) / 8 * 8; }

size_t lora_scratch_bytes(int64_t T, int64_t K, int R) {
  // The 16-bit copy of an fp32 LoRA operand (R x K elements, the fp32-operand
  // forms); the split products need none (their slices meet in shared memory).
  (void)T;
  return align256((size_t)std::max(R, 8) * std::max<int64_t>(K, 1) * 2);
}

int launch_lora_down16(const uint16_t* x, int64_t ldx, const uint16_t* A16, int64_t T, int64_t K,
                       int R, float* u, uint16_t* u16, float* scratch, size_t scratch_bytes,
                       cudaStream_t st, uint16_t* uh) {
  LSQ_TRY(check_ranks(R));
  if (K % 8 != 0 || ldx % 8 != 0) return set_error(LSQ_ERR_SHAPE, "lora_down: K %% 8 != 0");
  // C[t, j] = sum_k x[t, k] A[j, k]   (fp16 operands); u16 transposed [R][ld]; uh fp16 [T][R]
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(u, R, 1, 1.f, 0, u16, 1, lora16_ld(T));
  a.h16 = uh;
  a.h16_m = R;
  a.h16_n = 1;
  a.h16_f16 = 1;
  a.M = T; a.N = R; a.K = K;
  const Operand A{x, K, T, ldx, true}, B{A16, K, R, K, true};
  LSQ_TRY((run<false, false>(a, A, B, true, st)));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r_u", 2.0 * T * R * K, 2.0 * T * K + 2.0 * R * K);
  return LSQ_OK;
}

int launch_lora_vproj16(const uint16_t* dy, int64_t T, int64_t N, const uint16_t* Bs, int R,
                        float* v, uint16_t* v16, float* scratch, size_t scratch_bytes,
                        cudaStream_t st, uint16_t* vh) {
  LSQ_TRY(check_ranks(R));
  if (N % 8 != 0) return set_error(LSQ_ERR_SHAPE, "lora_vproj: N %% 8 != 0");
  // C[t, c] = sum_n dy[t, n] Bs^T[c, n]   (bf16 operands); v16 transposed [R][ld]; vh bf16 [T][R]
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(v, R, 1, 1.f, 0, v16, 1, lora16_ld(T));
  a.h16 = vh;
  a.h16_m = R;
  a.h16_n = 1;
  a.h16_f16 = 0;
  a.M = T; a.N = R; a.K = N;
  const Operand A{dy, N, T, N, false}, B{Bs, N, R, N, false};
  LSQ_TRY((run<false, false>(a, A, B, false, st)));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r_v", 2.0 * T * R * N, 2.0 * T * N + 2.0 * R * N);
  return LSQ_OK;
}

int launch_lora_grad_ab16(const uint16_t* v16, const uint16_t* x, int64_t K, float* dA,
                          const uint16_t* dy, const uint16_t* u16, int64_t N, int r, int n_parts,
                          const int64_t* part_end, int64_t T, float s, int accumulate, float* dB,
                          cudaStream_t st) {
  const int R = n_parts * r;
  LSQ_TRY(check_ranks(R));
  if (n_parts < 1 || n_parts > 4) return set_error(LSQ_ERR_SHAPE, "lora_grad_ab: 1..4 parts");
  if (K % 8 != 0 || N % 8 != 0) return set_error(LSQ_ERR_SHAPE, "lora_grad_ab: K, N %% 8 != 0");
  if (T <= 0) return LSQ_OK;
  // dA: C[k, j] = sum_t x[t, k] v[t, j], dA[j, k] (+)= s C[k, j] (x converted from fp16 to
  // bf16 as it lands); dB: C[n, c] = sum_t dy[t, n] u[t, c], dB[n, j] (+)= s C[n, part(n) r +
  // j], each row keeping its own part's columns; one launch
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(dA, 1, K, s, accumulate, nullptr, 0, 0);
  a.M = K; a.N = R; a.K = T;
  SkinnyArgs b = out_args(dB, r, 1, s, accumulate, nullptr, 0, 0);
  b.M = N; b.N = R; b.K = T;
  if (n_parts > 1) {
    b.part_r = r;
    b.n_parts = n_parts;
    for (int q = 0; q < n_parts; ++q) b.part_end[q] = part_end[q];
  }
  const Operand Aa{x, K, T, K, true}, Ba{v16, T, R, lora16_ld(T), false};
  const Operand Ab{dy, N, T, N, false}, Bb{u16, T, R, lora16_ld(T), false};
  LSQ_TRY(run_pair_mn(a, Aa, true, b, Ab, false, Ba, Bb, st));
  if (prof >= 0)
    prof_end(prof, st, "lora_rank_r_dAdB", 2.0 * T * R * (K + N),
             2.0 * T * K + 2.0 * T * N + 4.0 * T * R);
  return LSQ_OK;
}

// fp32-operand forms (one part), used by the single-linear entry points: the LoRA
// operand is rounded once into the start of the scratch, then the product runs.
int launch_lora_down(const uint16_t* x, int64_t ldx, const float* A, int64_t T, int64_t K, int R,
                     float* u, uint16_t* u16, float* scratch, size_t scratch_bytes,
                     cudaStream_t st, uint16_t* uh) {
  LSQ_TRY(check_ranks(R));
  Split sp;
  LSQ_TRY(split_scratch(scratch, scratch_bytes, (size_t)R * K, &sp, "lora_down"));
  to_f16_rows_kernel<<<grid_for_elems((int64_t)R * K), 256, 0, st>>>(A, R, K, K, sp.q, K);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return launch_lora_down16(x, ldx, sp.q, T, K, R, u, u16, sp.rest, sp.rest_bytes, st, uh);
}

int launch_lora_vproj(const uint16_t* dy, int64_t T, int64_t N, const float* B, int r, float* v,
                      uint16_t* v16, float* scratch, size_t scratch_bytes, cudaStream_t st,
                      uint16_t* vh) {
  LSQ_TRY(check_ranks(r));
  Split sp;
  LSQ_TRY(split_scratch(scratch, scratch_bytes, (size_t)N * r, &sp, "lora_vproj"));
  to_bf16_transposed_kernel<<<grid_for_elems((int64_t)N * r), 256, 0, st>>>(B, N, r, sp.q);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return launch_lora_vproj16(dy, T, N, sp.q, r, v, v16, sp.rest, sp.rest_bytes, st, vh);
}

// One layer's LoRA operands in their product types (see internal.h).
__global__ void lora_prepare_kernel(const float* __restrict__ lora, int64_t lora_stride,
                                    uint16_t* __restrict__ out, int64_t out_stride,
                                    const LoraPrepSegs segs) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int layer = blockIdx.y;
  const float* src = lora + (int64_t)layer * lora_stride;
  uint16_t* dst = out + (int64_t)layer * out_stride;
  for (int b = 0; b < segs.n; ++b) {
    const LoraPrepSeg& g = segs.seg[b];
    const int64_t n_el = g.rows * g.ld_out;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el;
         i += (int64_t)gridDim.x * blockDim.x) {
      if (g.kind == 0) {  // A: fp16 copy, [rows][cols]
        const int64_t row = i / g.ld_out, col = i % g.ld_out;
        dst[g.dst_off + i] = float_to_f16_bits(src[g.src_off + row * g.cols + col]);
      } else if (g.kind == 1) {  // B: bf16 block-diagonal stack, transposed: [n_parts r][rows]
        const int64_t j = i / g.rows, row = i % g.rows;
        int p = 0;
        while (p + 1 < g.n_parts && row >= g.part_end[p]) ++p;
        const int64_t jj = j - (int64_t)p * g.cols;
        const float v = (jj >= 0 && jj < g.cols) ? src[g.src_off + row * g.cols + jj] : 0.f;
        dst[g.dst_off + i] = float_to_bf16_bits(v);
      } else if (g.kind == 2) {  // scale * B, fp16 block-diagonal stack: [rows][n_parts r]
        const int64_t row = i / g.ld_out, j = i % g.ld_out;
        int p = 0;
        while (p + 1 < g.n_parts && row >= g.part_end[p]) ++p;
        const int64_t jj = j - (int64_t)p * g.cols;
        const float v = (jj >= 0 && jj < g.cols) ? g.scale * src[g.src_off + row * g.cols + jj]
                                                 : 0.f;
        dst[g.dst_off + i] = float_to_f16_bits(v);
      } else {  // scale * A^T, bf16: A [ld_out][rows] -> [rows][ld_out]
        const int64_t row = i / g.ld_out, j = i % g.ld_out;
        dst[g.dst_off + i] = float_to_bf16_bits(g.scale * src[g.src_off + j * g.rows + row]);
      }
    }
  }
}

int launch_lora_prepare(const float* lora, int64_t lora_stride, int n_layers, uint16_t* out,
                        int64_t out_stride, const LoraPrepSegs& segs, cudaStream_t st) {
  if (n_layers <= 0) return LSQ_OK;
  int64_t most = 0;
  for (int b = 0; b < segs.n; ++b) most = std::max(most, segs.seg[b].rows * segs.seg[b].ld_out);
  // about 32 resident CTAs' worth of threads per SM over all layers
  const int64_t cap = std::max<int64_t>(1, (int64_t)kSMs * 32 / n_layers);
  unsigned gx = (unsigned)std::max<int64_t>(1, std::min<int64_t>((most + 255) / 256, cap));
  lora_prepare_kernel<<<dim3(gx, (unsigned)n_layers), 256, 0, st>>>(lora, lora_stride, out,
                                                                    out_stride, segs);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

}  // namespace lsq

extern "C" int lsq_lora_plan_get(int64_t M, int64_t N, int64_t K, int32_t num_sms,
                                 lsq_lora_plan* out) {
  using namespace lsq;
  if (!out) return set_error(LSQ_ERR_INVALID, "lsq_lora_plan_get: null output");
  if (M <= 0 || N <= 0 || K <= 0 || num_sms <= 0)
    return set_error(LSQ_ERR_SHAPE, "lsq_lora_plan_get: bad size");
  const int n_pad = npad_for(N);
  const int z = splits_for(M, N, K, num_sms);
  lsq_lora_plan o{};
  o.n_pad = n_pad;
  o.row_tiles = (int32_t)((M + kSM - 1) / kSM);
  o.col_tiles = (int32_t)((N + n_pad - 1) / n_pad);
  o.splits = z;
  o.kt_total = (int32_t)((K + kSK - 1) / kSK);
  o.stages = stages_for(n_pad);
  o.stage_bytes = (int32_t)stage_bytes(n_pad);
  o.smem_bytes = (int32_t)smem_for(n_pad);
  o.smem_limit = (int32_t)smem_for(kSMaxN);
  o.ctas_per_sm = ctas_per_sm(n_pad);
  uint32_t cols = 32;
  while (cols < (uint32_t)n_pad) cols <<= 1;
  o.tmem_cols = (int32_t)cols;
  o.reduce_bytes = z > 1 ? kSM * (n_pad + 4) * 4 : 0;
  *out = o;
  return LSQ_OK;
}

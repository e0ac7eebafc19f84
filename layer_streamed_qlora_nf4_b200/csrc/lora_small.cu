// LoRA rank-r products around the fused NF4 GEMM (tensor cores, mma.sync).
//
// For y = x W^T + s (x A^T) B^T (Soup layer-streaming tutorial, "四段資料路徑"
// part 1) and its backward (part 3): u = x A^T (forward), v = dY B, and the
// trainable gradients dA = s v^T x, dB = s dY^T u.  All four are "tall x
// skinny" products: C[m, n] = sum_k P(m, k) Q(k, n) with n spanning r to 3 r
// columns (one tile of up to 192 columns, more tiles beyond), P a bf16
// activation and Q an fp32 LoRA tensor.
//
// One kernel serves all four.  A CTA owns 128 rows x BN columns of C over one
// slice of the reduction.  Q is first rounded once to a 16-bit type (nearest
// even) into scratch, rows padded to a multiple of 8 elements with zeros;
// accumulation is fp32 (the tutorial's part 1: the LoRA A/B matrices are
// computed at a higher precision than the NF4 storage).  Operand types follow
// the activations: u = x A^T multiplies fp16 (x is an fp16 forward activation,
// A is rounded to fp16); v, dA and dB multiply bf16 (each has a gradient
// operand, which needs bf16's range; dA's fp16 activation is rounded to bf16
// as it moves from shared memory into registers).  Both operands then stream through a ring of 4 to 6
// cp.async stages (16-byte chunks along whichever index is contiguous in
// memory; ldmatrix, transposing where needed, gives the MMA fragments), so
// that each SM keeps enough bytes in flight to run these HBM-bound products
// near the memory roofline.  When a product is split along its reduction, the
// slices are summed by a second kernel in a fixed order, so results are
// deterministic (no atomics); an unsplit product writes its result directly.
#include <stdlib.h>

#include "common.cuh"

namespace lsq {

namespace {

constexpr int kBM = 128;  // rows of C per CTA
constexpr int kBK = 32;   // reduction elements per stage
constexpr int kThreads = 256;
constexpr int kSMs = 148;

struct SkinnyArgs {
  const uint16_t* P;   // bf16: P(m, k) = P[m * p_m + k * p_k]
  int64_t p_m, p_k;
  const uint16_t* Q;   // bf16: Q(k, n) = Q[k * q_k + n * q_n]; rows padded to 8 elements
  int64_t q_k, q_n;
  int64_t M, N, K;     // C is M x N, reduction over K
  int64_t k_per_split;
  float* part;         // [splits][M][N] when split
  // unsplit: dst[m * c_m + n * c_n] = alpha * C[m, n] (+ dst if accumulate)
  float* dst;
  int64_t c_m, c_n;
  float alpha;
  int accumulate;
  int direct;
  // Output options (applied where the result is written: the direct epilogue or
  // the slice sum): c16 (nullable) also receives the result rounded to bf16,
  // c16[m * c16_ld + n], for the product that consumes it; with part_r > 0 the
  // rows are split into parts ending at part_end[], and row m of part p keeps
  // only columns [p part_r, (p + 1) part_r), written to column n - p part_r.
  uint16_t* c16;
  int64_t c16_ld;
  int part_r, n_parts;
  int64_t part_end[4];
};

// Writes one result element of row m, column n (see SkinnyArgs); false if dropped.
__device__ __forceinline__ void store_result(const SkinnyArgs& a, int64_t m, int64_t n, float v) {
  int64_t col = n;
  if (a.part_r > 0) {
    int p = 0;
    while (p + 1 < a.n_parts && m >= a.part_end[p]) ++p;
    col = n - (int64_t)p * a.part_r;
    if (col < 0 || col >= a.part_r) return;
  }
  float* d = a.dst + m * a.c_m + col * a.c_n;
  *d = (a.accumulate ? *d : 0.f) + a.alpha * v;
  if (a.c16) a.c16[m * a.c16_ld + n] = float_to_bf16_bits(v);
}

__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Operand precision of a product: PM_BF16 both operands bf16; PM_F16 both fp16;
// PM_P16 P stored fp16 and rounded to bf16 in registers, Q bf16.
enum { PM_BF16 = 0, PM_F16 = 1, PM_P16 = 2 };
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Shared-memory tiles per stage (bf16, rows padded by 8 elements so that the
// eight 16-byte rows an ldmatrix reads fall in distinct banks):
//   P_RED: P as [kBM m][kBK + 8]   else P as [kBK k][kBM + 8]
//   Q_RED: Q as [BN n][kBK + 8]    else Q as [kBK k][BN + 8]
// Stages and CTAs per SM: BN 64 -> 4 stages, 3 CTAs (61 KB each); BN 128 -> 4
// stages, 2 CTAs (82 KB); BN 192 -> 6 stages, 1 CTA (154 KB).
template <bool P_RED, bool Q_RED, int BN>
struct Tile {
  static constexpr int kStages = BN > 128 ? 6 : 4;
  static constexpr int kMinBlocks = BN <= 64 ? 3 : BN <= 128 ? 2 : 1;
  static constexpr int kPE = P_RED ? kBM * (kBK + 8) : kBK * (kBM + 8);
  static constexpr int kQE = Q_RED ? BN * (kBK + 8) : kBK * (BN + 8);
  static constexpr size_t kSmem = (size_t)kStages * (kPE + kQE) * 2;
};

// P_RED: the reduction index is the contiguous one in P (else the row index m is).
// Q_RED: the reduction index is the contiguous one in Q (else the column n is).
template <bool P_RED, bool Q_RED, int BN, int PM>
__global__ void __launch_bounds__(kThreads, (Tile<P_RED, Q_RED, BN>::kMinBlocks))
    skinny_kernel(const SkinnyArgs a) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  using TL = Tile<P_RED, Q_RED, BN>;
  constexpr int S = TL::kStages, PE = TL::kPE, QE = TL::kQE;
  extern __shared__ __align__(16) uint16_t sk_smem[];
  uint16_t* Ps = sk_smem;        // [S][PE]
  uint16_t* Qs = Ps + S * PE;    // [S][QE]
  constexpr int WN = BN / 2;     // columns per warp (warps: 4 along m x 2 along n)
  constexpr int NF = WN / 8;     // n8 fragments per warp
  constexpr int QC = BN * kBK / 8 / kThreads;  // 16-byte chunks of Q per thread per stage
  static_assert(QC >= 1 && (BN * kBK / 8) % kThreads == 0, "Q tile split");
  static_assert(NF % 2 == 0, "B fragments are loaded in pairs");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp & 3, wn = warp >> 2;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int64_t n0 = (int64_t)blockIdx.y * BN;
  const int64_t k_begin = (int64_t)blockIdx.z * a.k_per_split;
  const int64_t k_end = min(a.K, k_begin + a.k_per_split);
  const int64_t n_it = k_end > k_begin ? (k_end - k_begin + kBK - 1) / kBK : 0;

  float acc[2][NF][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < NF; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  // One stage: 512 chunks of P (two per thread) and BN * 4 chunks of Q.  Chunks
  // outside the product (or this CTA's slice of the reduction) are zero-filled.
  auto load_stage = [&](int slot, int64_t kb) {
    uint16_t* pd = Ps + slot * PE;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + i * kThreads;
      if (P_RED) {  // row m, 4 chunks of k per row
        const int mm = c >> 2, kc = (c & 3) * 8;
        const int64_t m = m0 + mm, k = kb + kc;
        const bool in = m < a.M && k < k_end;
        cp_async16(smem_u32(pd + mm * (kBK + 8) + kc), a.P + (in ? m * a.p_m + k : 0),
                   in ? 16u : 0u);
      } else {      // row k, 16 chunks of m per row
        const int kk = c >> 4, mc = (c & 15) * 8;
        const int64_t m = m0 + mc, k = kb + kk;
        const bool in = m < a.M && k < k_end;
        cp_async16(smem_u32(pd + kk * (kBM + 8) + mc), a.P + (in ? k * a.p_k + m : 0),
                   in ? 16u : 0u);
      }
    }
    uint16_t* qd = Qs + slot * QE;
#pragma unroll
    for (int i = 0; i < QC; ++i) {
      const int c = tid + i * kThreads;
      if (Q_RED) {  // row n, 4 chunks of k per row
        const int nn = c >> 2, kc = (c & 3) * 8;
        const int64_t n = n0 + nn, k = kb + kc;
        const bool in = n < a.N && k < k_end;
        cp_async16(smem_u32(qd + nn * (kBK + 8) + kc), a.Q + (in ? n * a.q_n + k : 0),
                   in ? 16u : 0u);
      } else {      // row k, BN / 8 chunks of n per row (the padded row ends on a chunk)
        const int kk = c / (BN / 8), nc = (c % (BN / 8)) * 8;
        const int64_t n = n0 + nc, k = kb + kk;
        const bool in = n < a.N && k < k_end;
        cp_async16(smem_u32(qd + kk * (BN + 8) + nc), a.Q + (in ? k * a.q_k + n : 0),
                   in ? 16u : 0u);
      }
    }
  };

  // Ring: stage j lives in slot j % S; S - 1 stages are in flight ahead of the math.
#pragma unroll
  for (int j = 0; j < S - 1; ++j) {
    if (j < n_it) load_stage(j, k_begin + (int64_t)j * kBK);
    cp_async_commit();
  }
  for (int64_t it = 0; it < n_it; ++it) {
    cp_async_wait<S - 2>();  // stage it has landed (this thread's chunks)
    __syncthreads();         // ... every thread's, and slot (it - 1) % S is free again
    {
      const int64_t nx = it + S - 1;
      if (nx < n_it) load_stage((int)(nx % S), k_begin + nx * kBK);
      cp_async_commit();
    }
    const int slot = (int)(it % S);
    const uint16_t* ps = Ps + slot * PE;
    const uint16_t* qs = Qs + slot * QE;
#pragma unroll
    for (int k16 = 0; k16 < kBK; k16 += 16) {
      uint32_t af[2][4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const int r0 = wm * 32 + mi * 16;
        if (P_RED) {
          ldsm4(af[mi], smem_u32(ps + (r0 + (lane & 15)) * (kBK + 8) + k16 + 8 * (lane >> 4)));
        } else {
          const int i = lane >> 3, j = lane & 7;
          ldsm4_t(af[mi], smem_u32(ps + (k16 + j + 8 * (i >> 1)) * (kBM + 8) + r0 + 8 * (i & 1)));
        }
        if (PM == PM_P16) {
#pragma unroll
          for (int e = 0; e < 4; ++e) af[mi][e] = f16x2_to_bf16x2(af[mi][e]);
        }
      }
#pragma unroll
      for (int nj = 0; nj < NF; nj += 2) {
        // matrices: (n block nj, k 0-7), (nj, k 8-15), (nj + 1, k 0-7), (nj + 1, k 8-15)
        const int i = lane >> 3, j = lane & 7;
        uint32_t bh[4];
        if (Q_RED) {
          const int nr = wn * WN + (nj + (i >> 1)) * 8 + j;
          ldsm4(bh, smem_u32(qs + nr * (kBK + 8) + k16 + 8 * (i & 1)));
        } else {
          const int kr = k16 + 8 * (i & 1) + j;
          ldsm4_t(bh, smem_u32(qs + kr * (BN + 8) + wn * WN + (nj + (i >> 1)) * 8));
        }
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          if (PM == PM_F16) {
            mma_f16(acc[mi][nj], af[mi], bh[0], bh[1]);
            mma_f16(acc[mi][nj + 1], af[mi], bh[2], bh[3]);
          } else {
            mma_bf16(acc[mi][nj], af[mi], bh[0], bh[1]);
            mma_bf16(acc[mi][nj + 1], af[mi], bh[2], bh[3]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();  // only empty groups can remain; leave none behind

#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
    for (int nj = 0; nj < NF; ++nj) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t m = m0 + wm * 32 + mi * 16 + (lane >> 2) + 8 * h;
        const int64_t n = n0 + wn * WN + nj * 8 + 2 * (lane & 3);
        if (m >= a.M) continue;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (n + e >= a.N) continue;
          const float v = acc[mi][nj][2 * h + e];
          if (a.direct) {
            store_result(a, m, n + e, v);
          } else {
            a.part[((size_t)blockIdx.z * a.M + m) * a.N + n + e] = v;
          }
        }
      }
    }
  }
}

// sum_z part[z][m][n] in z order, written as SkinnyArgs a prescribes (store_result)
__global__ void split_sum_kernel(const float* __restrict__ part, int splits, const SkinnyArgs a) {
  const int64_t M = a.M, N = a.N;
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t n_el = M * N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    // unrolled so that several slices' loads are in flight; the adds stay in z order
#pragma unroll 8
    for (int z = 0; z < splits; ++z) s += part[(size_t)z * n_el + i];
    store_result(a, i / N, i % N, s);
  }
}

// out[i * ld_out + j] = bf16 or fp16 (F16) of in[i * ld_in + j] for j < cols, 0 for
// cols <= j < ld_out
template <bool F16>
__global__ void to_16_rows_kernel(const float* __restrict__ in, int64_t rows, int64_t cols,
                                  int64_t ld_in, uint16_t* __restrict__ out, int64_t ld_out) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t n_el = rows * ld_out;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / ld_out, j = i % ld_out;
    const float v = j < cols ? in[r * ld_in + j] : 0.f;
    out[i] = F16 ? float_to_f16_bits(v) : float_to_bf16_bits(v);
  }
}

int64_t pad8(int64_t n) { return (n + 7) / 8 * 8; }
size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// Column tile.  Default 64 for every product: 3 CTAs per SM, and a product
// wider than 64 columns runs several column tiles, which read the same
// activation rows (the second and third time mostly from L2).  LSQ_LORA_BN=128
// or 192 selects one tile of up to that many columns instead (fewer activation
// reads, 2 or 1 CTAs per SM).
int bn_limit() {
  static const int v = [] {
    const char* e = getenv("LSQ_LORA_BN");
    const int x = e ? atoi(e) : 64;
    return (x == 128 || x == 192) ? x : 64;
  }();
  return v;
}
int bn_for(int64_t N) {
  const int lim = bn_limit();
  return (N <= 64 || lim == 64) ? 64 : (N <= 128 || lim == 128) ? 128 : 192;
}
int ctas_per_sm(int bn) { return bn <= 64 ? 3 : bn <= 128 ? 2 : 1; }

// Splits of the reduction: only where the product's own tiles leave at least
// half of the resident CTA slots (148 SMs x CTAs per SM) empty, up to filling
// them, each slice at least four stages long (the partials cost a round trip
// through HBM, so a grid that already fills the GPU is not split).
int splits_for(int64_t M, int64_t N, int64_t K) {
  if (K <= 0 || M <= 0 || N <= 0) return 1;
  const int bn = bn_for(N);
  const int64_t xy = ((M + kBM - 1) / kBM) * ((N + bn - 1) / bn);
  int64_t z = (int64_t)kSMs * ctas_per_sm(bn) / xy;
  const int64_t zmax = std::max<int64_t>(1, K / (4 * kBK));
  z = std::max<int64_t>(1, std::min<int64_t>(z, std::min<int64_t>(zmax, 64)));
  const int64_t kps = ((K + z - 1) / z + kBK - 1) / kBK * kBK;
  return (int)((K + kps - 1) / kps);
}

template <bool P_RED, bool Q_RED, int BN, int PM>
int launch_bn(const SkinnyArgs& a, dim3 grid, cudaStream_t st) {
  constexpr size_t smem = Tile<P_RED, Q_RED, BN>::kSmem;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    LSQ_CUDA(cudaFuncSetAttribute(skinny_kernel<P_RED, Q_RED, BN, PM>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr_done[dev] = true;
  }
  skinny_kernel<P_RED, Q_RED, BN, PM><<<grid, kThreads, smem, st>>>(a);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

int convert_rows(const float* in, int64_t rows, int64_t cols, int64_t ld_in, uint16_t* out,
                 int64_t ld_out, cudaStream_t st, bool f16 = false) {
  int64_t g = (rows * ld_out + 255) / 256;
  if (g > kSMs * 8) g = kSMs * 8;
  if (g < 1) return LSQ_OK;
  if (f16)
    to_16_rows_kernel<true><<<(unsigned)g, 256, 0, st>>>(in, rows, cols, ld_in, out, ld_out);
  else
    to_16_rows_kernel<false><<<(unsigned)g, 256, 0, st>>>(in, rows, cols, ld_in, out, ld_out);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

// C = P Q over K, written as a prescribes (dst, alpha, accumulate, c16, parts);
// scratch holds the fixed-order partials when the product is split.
template <bool P_RED, bool Q_RED, int PM>
int run(SkinnyArgs a, float* scratch, size_t scratch_bytes, cudaStream_t st) {
  if (a.M <= 0 || a.N <= 0) return LSQ_OK;
  const int z = splits_for(a.M, a.N, a.K);
  const size_t need = z > 1 ? (size_t)z * a.M * a.N * sizeof(float) : 0;
  if (need && (!scratch || scratch_bytes < need))
    return set_error(LSQ_ERR_WORKSPACE, "lora product: scratch %zu < %zu", scratch_bytes, need);
  a.k_per_split = a.K > 0 ? ((a.K + z - 1) / z + kBK - 1) / kBK * kBK : kBK;
  a.direct = z == 1;
  a.part = z > 1 ? scratch : nullptr;
  const int bn = bn_for(a.N);
  dim3 grid((unsigned)((a.M + kBM - 1) / kBM), (unsigned)((a.N + bn - 1) / bn), (unsigned)z);
  switch (bn) {
    case 64: LSQ_TRY((launch_bn<P_RED, Q_RED, 64, PM>(a, grid, st))); break;
    case 128: LSQ_TRY((launch_bn<P_RED, Q_RED, 128, PM>(a, grid, st))); break;
    default: LSQ_TRY((launch_bn<P_RED, Q_RED, 192, PM>(a, grid, st))); break;
  }
  if (z == 1) return LSQ_OK;
  int64_t g = (a.M * a.N + 255) / 256;
  if (g > kSMs * 8) g = kSMs * 8;
  split_sum_kernel<<<(unsigned)g, 256, 0, st>>>(a.part, z, a);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
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
                    uint16_t* c16, int64_t c16_ld) {
  SkinnyArgs a{};
  a.dst = dst;
  a.c_m = c_m;
  a.c_n = c_n;
  a.alpha = alpha;
  a.accumulate = accumulate;
  a.c16 = c16;
  a.c16_ld = c16_ld;
  return a;
}

// 16-bit copies of fp32 LoRA operands, at the start of the scratch; returns the
// scratch left for the partials.
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

}  // namespace

size_t lora_scratch_bytes(int64_t T, int64_t K, int R) {
  // An upper bound over every product a caller sizing by (T, K, R) can make:
  // any width R' <= R, a reduction or a part of up to K elements:
  //   u = x A^T, v      M = T, N = R', reduction <= K, Q = A [R'][K] or B [<= K][R']
  //   dA, dB            M <= K, N = R', reduction T,   Q = v or u [T][R']
  // The first needs z(T, R', K) slices at most (splits grow with the reduction);
  // the second z * M <= min(64, T / (4 kBK)) K, and z * M <= slots * kBM as well,
  // since z <= slots / (M / kBM tiles).  The 16-bit copy of an fp32 operand comes first.
  size_t best = 0;
  for (int rr = 1; rr <= R; ++rr) {
    const int64_t q1 = K * pad8(rr);
    const int z1 = splits_for(T, rr, K);
    best = std::max(best, align256((size_t)q1 * 2) +
                              (z1 > 1 ? (size_t)z1 * T * rr * sizeof(float) : 0));
    const int64_t q2 = T * pad8(rr);
    const int64_t zcap = std::max<int64_t>(1, std::min<int64_t>(64, T / (4 * kBK)));
    const int64_t zm = std::min<int64_t>(zcap * K, (int64_t)kSMs * ctas_per_sm(bn_for(rr)) * kBM);
    best = std::max(best, align256((size_t)q2 * 2) +
                              (zcap > 1 ? (size_t)zm * rr * sizeof(float) : 0));
  }
  return best;
}

int launch_lora_down16(const uint16_t* x, int64_t ldx, const uint16_t* A16, int64_t T, int64_t K,
                       int R, float* u, uint16_t* u16, float* scratch, size_t scratch_bytes,
                       cudaStream_t st) {
  LSQ_TRY(check_ranks(R));
  if (K % 8 != 0) return set_error(LSQ_ERR_SHAPE, "lora_down: K %% 8 != 0");
  // C[t, j] = sum_k x[t, k] A[j, k]   (fp16 operands)
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(u, R, 1, 1.f, 0, u16, R);
  a.P = x; a.p_m = ldx; a.p_k = 1;
  a.Q = A16; a.q_k = 1; a.q_n = K;
  a.M = T; a.N = R; a.K = K;
  LSQ_TRY((run<true, true, PM_F16>(a, scratch, scratch_bytes, st)));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r_u", 2.0 * T * R * K, 2.0 * T * K + 2.0 * R * K);
  return LSQ_OK;
}

int launch_lora_vproj16(const uint16_t* dy, int64_t T, int64_t N, const uint16_t* Bs, int R,
                        float* v, uint16_t* v16, float* scratch, size_t scratch_bytes,
                        cudaStream_t st) {
  LSQ_TRY(check_ranks(R));
  // C[t, c] = sum_n dy[t, n] Bs[n, c]   (bf16 operands; Bs block-diagonal over the parts)
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(v, R, 1, 1.f, 0, v16, R);
  a.P = dy; a.p_m = N; a.p_k = 1;
  a.Q = Bs; a.q_k = R; a.q_n = 1;
  a.M = T; a.N = R; a.K = N;
  LSQ_TRY((run<true, false, PM_BF16>(a, scratch, scratch_bytes, st)));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r_v", 2.0 * T * R * N, 2.0 * T * N + 2.0 * R * N);
  return LSQ_OK;
}

int launch_lora_grad_a16(const uint16_t* v16, const uint16_t* x, int64_t T, int64_t K, int R,
                         float s, int accumulate, float* dA, float* scratch, size_t scratch_bytes,
                         cudaStream_t st) {
  LSQ_TRY(check_ranks(R));
  // C[k, j] = sum_t x[t, k] v[t, j];  dA[j, k] (+)= s C[k, j]   (x rounded from fp16 to bf16)
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(dA, 1, K, s, accumulate, nullptr, 0);
  a.P = x; a.p_m = 1; a.p_k = K;
  a.Q = v16; a.q_k = R; a.q_n = 1;
  a.M = K; a.N = R; a.K = T;
  LSQ_TRY((run<false, false, PM_P16>(a, scratch, scratch_bytes, st)));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r_dA", 2.0 * T * R * K, 2.0 * T * K + 2.0 * T * R);
  return LSQ_OK;
}

int launch_lora_grad_b16(const uint16_t* dy, const uint16_t* u16, int64_t T, int64_t N, int r,
                         int n_parts, const int64_t* part_end, float s, int accumulate, float* dB,
                         float* scratch, size_t scratch_bytes, cudaStream_t st) {
  const int R = n_parts * r;
  LSQ_TRY(check_ranks(R));
  if (n_parts < 1 || n_parts > 4) return set_error(LSQ_ERR_SHAPE, "lora_grad_b: 1..4 parts");
  // C[n, c] = sum_t dy[t, n] u[t, c];  dB[n, j] (+)= s C[n, part(n) r + j]: one product over
  // all parts, each row keeping its own part's columns
  const int prof = prof_begin(st);
  SkinnyArgs a = out_args(dB, r, 1, s, accumulate, nullptr, 0);
  a.P = dy; a.p_m = 1; a.p_k = N;
  a.Q = u16; a.q_k = R; a.q_n = 1;
  a.M = N; a.N = R; a.K = T;
  if (n_parts > 1) {
    a.part_r = r;
    a.n_parts = n_parts;
    for (int p = 0; p < n_parts; ++p) a.part_end[p] = part_end[p];
  }
  LSQ_TRY((run<false, false, PM_BF16>(a, scratch, scratch_bytes, st)));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r_dB", 2.0 * T * R * N, 2.0 * T * N + 2.0 * T * R);
  return LSQ_OK;
}

// fp32-operand forms (one part), used by the single-linear entry points: the LoRA
// operand is rounded once into the start of the scratch, then the product runs.
int launch_lora_down(const uint16_t* x, int64_t ldx, const float* A, int64_t T, int64_t K, int R,
                     float* u, uint16_t* u16, float* scratch, size_t scratch_bytes,
                     cudaStream_t st) {
  LSQ_TRY(check_ranks(R));
  Split sp;
  LSQ_TRY(split_scratch(scratch, scratch_bytes, (size_t)R * K, &sp, "lora_down"));
  LSQ_TRY(convert_rows(A, R, K, K, sp.q, K, st, /*f16=*/true));
  return launch_lora_down16(x, ldx, sp.q, T, K, R, u, u16, sp.rest, sp.rest_bytes, st);
}

int launch_lora_vproj(const uint16_t* dy, int64_t T, int64_t N, const float* B, int r, float* v,
                      uint16_t* v16, float* scratch, size_t scratch_bytes, cudaStream_t st) {
  LSQ_TRY(check_ranks(r));
  Split sp;
  LSQ_TRY(split_scratch(scratch, scratch_bytes, (size_t)N * r, &sp, "lora_vproj"));
  LSQ_TRY(convert_rows(B, N, r, r, sp.q, r, st));
  return launch_lora_vproj16(dy, T, N, sp.q, r, v, v16, sp.rest, sp.rest_bytes, st);
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
      const int64_t row = i / g.ld_out, col = i % g.ld_out;
      if (g.kind == 0) {  // A: fp16 copy, [rows][cols]
        dst[g.dst_off + i] = float_to_f16_bits(src[g.src_off + row * g.cols + col]);
      } else {            // B: bf16, block-diagonal [rows][n_parts r]
        int p = 0;
        while (p + 1 < g.n_parts && row >= g.part_end[p]) ++p;
        const int64_t j = col - (int64_t)p * g.cols;
        const float v = (j >= 0 && j < g.cols) ? src[g.src_off + row * g.cols + j] : 0.f;
        dst[g.dst_off + i] = float_to_bf16_bits(v);
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

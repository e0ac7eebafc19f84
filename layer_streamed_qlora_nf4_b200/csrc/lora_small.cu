// LoRA rank-r products around the fused NF4 GEMM (tensor cores, mma.sync).
//
// For y = x W^T + s (x A^T) B^T (Soup layer-streaming tutorial, "四段資料路徑"
// part 1) and its backward (part 3): u = x A^T (forward), v = dY B, and the
// trainable gradients dA = s v^T x, dB = s dY^T u.  All four are "tall x
// skinny" products: C[m, n] = sum_k P(m, k) Q(k, n) with n spanning at most
// 3 r <= 192 columns, P a bf16 activation and Q an fp32 LoRA tensor.
//
// One kernel serves all four.  A CTA owns 128 rows x BN columns of C over one
// slice of the reduction; P tiles arrive by cp.async (16-byte chunks along
// whichever index is contiguous in memory; ldmatrix, transposing where P's rows
// are the contiguous index, gives the A fragments), and each fp32 Q tile is
// rounded once to bf16 (nearest even) on its way to shared memory: bf16
// operands with fp32 accumulation, the compute precision of QLoRA's LoRA branch
// (the tutorial's part 1: the LoRA A/B matrices are computed at a higher
// precision than the NF4 storage).  The slices are summed by a second kernel in
// a fixed order, so results are deterministic (no atomics).
#include "common.cuh"

namespace lsq {

namespace {

constexpr int kBM = 128;  // rows of C per CTA
constexpr int kBK = 32;   // reduction elements per stage
constexpr int kThreads = 256;

struct SkinnyArgs {
  const uint16_t* P;   // bf16: P(m, k) = P[m * p_m + k * p_k]
  int64_t p_m, p_k;
  const float* Q;      // fp32: Q(k, n) = Q[k * q_k + n * q_n]
  int64_t q_k, q_n;
  int64_t M, N, K;     // C is M x N, reduction over K
  int64_t k_per_split;
  float* part;         // [splits][M][N]
};

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
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Shared-memory tiles per stage (bf16, rows padded by 8 elements so that the
// eight 16-byte rows an ldmatrix reads fall in distinct banks):
//   P_RED: P as [kBM m][kBK + 8]   else P as [kBK k][kBM + 8]
//   Q as [BN n][kBK + 8]
template <bool P_RED>
__host__ __device__ constexpr int p_stage_elems() {
  return P_RED ? kBM * (kBK + 8) : kBK * (kBM + 8);
}
template <int BN>
__host__ __device__ constexpr int q_stage_elems() {
  return BN * (kBK + 8);
}
template <bool P_RED, int BN>
constexpr size_t skinny_smem_bytes() {
  return 2 * (size_t)(p_stage_elems<P_RED>() + q_stage_elems<BN>()) * 2;
}

// P_RED: the reduction index is the contiguous one in P (else the row index m is).
// Q_RED: the reduction index is the contiguous one in Q (else the column n is).
template <bool P_RED, bool Q_RED, int BN>
__global__ void __launch_bounds__(kThreads) skinny_kernel(const SkinnyArgs a) {
  extern __shared__ __align__(16) uint16_t sk_smem[];
  constexpr int PE = p_stage_elems<P_RED>(), QE = q_stage_elems<BN>();
  uint16_t* Ps = sk_smem;        // [2][PE]
  uint16_t* Qh = Ps + 2 * PE;    // [2][QE]
  constexpr int WN = BN / 2;     // columns per warp (warps: 4 along m x 2 along n)
  constexpr int NF = WN / 8;     // n8 fragments per warp
  constexpr int QV = BN * kBK / 4 / kThreads;  // float4 of Q per thread per stage
  static_assert(QV >= 1 && (BN * kBK / 4) % kThreads == 0, "Q tile split");
  static_assert(NF % 2 == 0, "B fragments are loaded in pairs");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp & 3, wn = warp >> 2;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int64_t n0 = (int64_t)blockIdx.y * BN;
  const int64_t k_begin = (int64_t)blockIdx.z * a.k_per_split;
  const int64_t k_end = min(a.K, k_begin + a.k_per_split);

  float acc[2][NF][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < NF; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  // ---- P tile of the stage starting at kb: 512 chunks of 8 bf16 (two per thread)
  auto load_p = [&](int st, int64_t kb) {
    uint16_t* dst = Ps + st * PE;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + i * kThreads;
      if (P_RED) {  // row m, 4 chunks of k per row
        const int mm = c >> 2, kc = (c & 3) * 8;
        const int64_t m = m0 + mm, k = kb + kc;
        const bool in = m < a.M && k < k_end;
        cp_async16(smem_u32(dst + mm * (kBK + 8) + kc), a.P + (in ? m * a.p_m + k : 0),
                   in ? 16u : 0u);
      } else {      // row k, 16 chunks of m per row
        const int kk = c >> 4, mc = (c & 15) * 8;
        const int64_t m = m0 + mc, k = kb + kk;
        const bool in = m < a.M && k < k_end;
        cp_async16(smem_u32(dst + kk * (kBM + 8) + mc), a.P + (in ? k * a.p_k + m : 0),
                   in ? 16u : 0u);
      }
    }
  };
  // ---- Q tile: QV float4 per thread into registers, then rounded to bf16
  float4 qr[QV];
  auto load_q = [&](int64_t kb) {
#pragma unroll
    for (int i = 0; i < QV; ++i) {
      const int c = tid + i * kThreads;
      int nn, kk;
      if (Q_RED) {
        nn = c / (kBK / 4);
        kk = (c % (kBK / 4)) * 4;
      } else {
        kk = c / (BN / 4);
        nn = (c % (BN / 4)) * 4;
      }
      const int64_t n = n0 + nn, k = kb + kk;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n < a.N && k < k_end)
        v = __ldg(reinterpret_cast<const float4*>(a.Q + k * a.q_k + n * a.q_n));
      qr[i] = v;
    }
  };
  auto store_q = [&](int st) {
    uint16_t* qs = Qh + st * QE;
#pragma unroll
    for (int i = 0; i < QV; ++i) {
      const int c = tid + i * kThreads;
      const float v[4] = {qr[i].x, qr[i].y, qr[i].z, qr[i].w};
      uint16_t h[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) h[e] = float_to_bf16_bits(v[e]);
      if (Q_RED) {  // four consecutive k of one n: one 8-byte store
        const int nn = c / (kBK / 4), kk = (c % (kBK / 4)) * 4;
        *reinterpret_cast<uint2*>(qs + nn * (kBK + 8) + kk) =
            make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
      } else {      // one k of four consecutive n
        const int kk = c / (BN / 4), nn = (c % (BN / 4)) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) qs[(nn + e) * (kBK + 8) + kk] = h[e];
      }
    }
  };

  int st = 0;
  if (k_begin < k_end) {
    load_p(0, k_begin);
    cp_async_commit();
    load_q(k_begin);
    store_q(0);
  }
  for (int64_t kb = k_begin; kb < k_end; kb += kBK) {
    const bool has_next = kb + kBK < k_end;
    if (has_next) {
      load_p(st ^ 1, kb + kBK);
      cp_async_commit();
      load_q(kb + kBK);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // P and Q of stage st visible to every warp
    const uint16_t* ps = Ps + st * PE;
    const uint16_t* qh = Qh + st * QE;
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
      }
#pragma unroll
      for (int nj = 0; nj < NF; nj += 2) {
        const int nr = wn * WN + nj * 8 + (lane & 7) + 8 * (lane >> 4);
        const int kc = k16 + 8 * ((lane >> 3) & 1);
        uint32_t bh[4];
        ldsm4(bh, smem_u32(qh + nr * (kBK + 8) + kc));
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          mma_bf16(acc[mi][nj], af[mi], bh[0], bh[1]);
          mma_bf16(acc[mi][nj + 1], af[mi], bh[2], bh[3]);
        }
      }
    }
    if (has_next) store_q(st ^ 1);  // stage st ^ 1 was last read before the previous sync
    __syncthreads();                // every warp is done with stage st
    st ^= 1;
  }

  float* out = a.part + (size_t)blockIdx.z * a.M * a.N;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
    for (int nj = 0; nj < NF; ++nj) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t m = m0 + wm * 32 + mi * 16 + (lane >> 2) + 8 * h;
        const int64_t n = n0 + wn * WN + nj * 8 + 2 * (lane & 3);
        if (m >= a.M) continue;
        if (n < a.N) out[m * a.N + n] = acc[mi][nj][2 * h];
        if (n + 1 < a.N) out[m * a.N + n + 1] = acc[mi][nj][2 * h + 1];
      }
    }
  }
}

// dst[m * c_m + n * c_n] = alpha * sum_z part[z][m][n] (+ dst if accumulate), z in order
__global__ void split_sum_kernel(const float* __restrict__ part, int splits, int64_t M, int64_t N,
                                 float alpha, int accumulate, float* __restrict__ dst, int64_t c_m,
                                 int64_t c_n) {
  const int64_t n_el = M * N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < splits; ++z) s += part[(size_t)z * n_el + i];
    const int64_t m = i / N, n = i % N;
    float* d = dst + m * c_m + n * c_n;
    *d = (accumulate ? *d : 0.f) + alpha * s;
  }
}

int bn_for(int64_t N) { return N <= 64 ? 64 : N <= 128 ? 128 : 192; }

// Splits of the reduction for a product: about two waves of CTAs on 148 SMs,
// each slice at least two stages long.
int splits_for(int64_t M, int64_t N, int64_t K) {
  const int bn = bn_for(N);
  const int64_t xy = ((M + kBM - 1) / kBM) * ((N + bn - 1) / bn);
  int64_t z = (2 * 148 + xy - 1) / xy;
  const int64_t zmax = std::max<int64_t>(1, K / (2 * kBK));
  z = std::max<int64_t>(1, std::min<int64_t>(z, std::min<int64_t>(zmax, 64)));
  const int64_t kps = ((K + z - 1) / z + kBK - 1) / kBK * kBK;
  return (int)((K + kps - 1) / kps);
}

template <bool P_RED, bool Q_RED, int BN>
int launch_bn(const SkinnyArgs& a, dim3 grid, cudaStream_t st) {
  constexpr size_t smem = skinny_smem_bytes<P_RED, BN>();
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    LSQ_CUDA(cudaFuncSetAttribute(skinny_kernel<P_RED, Q_RED, BN>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr_done[dev] = true;
  }
  skinny_kernel<P_RED, Q_RED, BN><<<grid, kThreads, smem, st>>>(a);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

template <bool P_RED, bool Q_RED>
int run(const SkinnyArgs& a0, int splits, cudaStream_t st) {
  SkinnyArgs a = a0;
  a.k_per_split = ((a.K + splits - 1) / splits + kBK - 1) / kBK * kBK;
  const int bn = bn_for(a.N);
  dim3 grid((unsigned)((a.M + kBM - 1) / kBM), (unsigned)((a.N + bn - 1) / bn), (unsigned)splits);
  switch (bn) {
    case 64: return launch_bn<P_RED, Q_RED, 64>(a, grid, st);
    case 128: return launch_bn<P_RED, Q_RED, 128>(a, grid, st);
    default: return launch_bn<P_RED, Q_RED, 192>(a, grid, st);
  }
}

int finish(const float* part, int splits, int64_t M, int64_t N, float alpha, int accumulate,
           float* dst, int64_t c_m, int64_t c_n, cudaStream_t st) {
  int64_t g = (M * N + 255) / 256;
  if (g > 148 * 8) g = 148 * 8;
  split_sum_kernel<<<(unsigned)g, 256, 0, st>>>(part, splits, M, N, alpha, accumulate, dst, c_m,
                                                c_n);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

}  // namespace

size_t lora_scratch_bytes(int64_t T, int64_t K, int R) {
  // the largest partial buffer a product of these sizes needs:
  // u or v: M = T, N = R, reduction K;  dA or dB: M = K, N = R, reduction T
  const size_t a = (size_t)splits_for(T, R, K) * T * R;
  const size_t b = (size_t)splits_for(K, R, T) * K * R;
  return std::max(a, b) * sizeof(float);
}

int launch_lora_down(const uint16_t* x, int64_t ldx, const float* A, int64_t T, int64_t K, int R,
                     float* u, float* scratch, size_t scratch_bytes, cudaStream_t st) {
  const int s = splits_for(T, R, K);
  const size_t need = (size_t)s * T * R * sizeof(float);
  if (!scratch || scratch_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "lora_down: scratch %zu < %zu", scratch_bytes, need);
  // C[t, j] = sum_k x[t, k] A[j, k]
  SkinnyArgs a{x, ldx, 1, A, 1, K, T, R, K, 0, scratch};
  const int prof = prof_begin(st);
  LSQ_TRY((run<true, true>(a, s, st)));
  LSQ_TRY(finish(scratch, s, T, R, 1.f, 0, u, R, 1, st));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r", 2.0 * T * R * K, 2.0 * T * K + 4.0 * R * K);
  return LSQ_OK;
}

int launch_lora_vproj(const uint16_t* dy, int64_t T, int64_t N, const float* B, int r, int n_parts,
                      const int64_t* part_end, float* v, float* scratch, size_t scratch_bytes,
                      cudaStream_t st) {
  const int R = n_parts * r;
  int64_t start = 0;
  for (int p = 0; p < n_parts; ++p) {
    const int64_t Np = part_end[p] - start;
    const int s = splits_for(T, r, Np);
    const size_t need = (size_t)s * T * r * sizeof(float);
    if (!scratch || scratch_bytes < need)
      return set_error(LSQ_ERR_WORKSPACE, "lora_vproj: scratch %zu < %zu", scratch_bytes, need);
    // C[t, j] = sum_n dy[t, start + n] B[start + n, j]
    SkinnyArgs a{dy + start, N, 1, B + start * r, r, 1, T, r, Np, 0, scratch};
    const int prof = prof_begin(st);
    LSQ_TRY((run<true, false>(a, s, st)));
    LSQ_TRY(finish(scratch, s, T, r, 1.f, 0, v + p * r, R, 1, st));
    if (prof >= 0)
      prof_end(prof, st, "lora_rank_r", 2.0 * T * r * Np, 2.0 * T * Np + 4.0 * r * Np);
    start = part_end[p];
  }
  return LSQ_OK;
}

int launch_lora_grad_a(const float* v, const uint16_t* x, int64_t T, int64_t K, int R, float s,
                       int accumulate, float* dA, float* scratch, size_t scratch_bytes,
                       cudaStream_t st) {
  // C[k, j] = sum_t x[t, k] v[t, j];  dA[j, k] (+)= s C[k, j]
  const int z = splits_for(K, R, T);
  const size_t need = (size_t)z * K * R * sizeof(float);
  if (!scratch || scratch_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "lora_grad_a: scratch %zu < %zu", scratch_bytes, need);
  SkinnyArgs a{x, 1, K, v, R, 1, K, R, T, 0, scratch};
  const int prof = prof_begin(st);
  LSQ_TRY((run<false, false>(a, z, st)));
  LSQ_TRY(finish(scratch, z, K, R, s, accumulate, dA, 1, K, st));
  if (prof >= 0) prof_end(prof, st, "lora_rank_r", 2.0 * T * R * K, 2.0 * T * K + 4.0 * T * R);
  return LSQ_OK;
}

int launch_lora_grad_b(const uint16_t* dy, const float* u, int64_t T, int64_t N, int r, int R,
                       int n_parts, const int64_t* part_end, float s, int accumulate, float* dB,
                       float* scratch, size_t scratch_bytes, cudaStream_t st) {
  int64_t start = 0;
  for (int p = 0; p < n_parts; ++p) {
    const int64_t Np = part_end[p] - start;
    // C[n, j] = sum_t dy[t, start + n] u[t, p r + j];  dB[start + n, j] (+)= s C[n, j]
    const int z = splits_for(Np, r, T);
    const size_t need = (size_t)z * Np * r * sizeof(float);
    if (!scratch || scratch_bytes < need)
      return set_error(LSQ_ERR_WORKSPACE, "lora_grad_b: scratch %zu < %zu", scratch_bytes, need);
    SkinnyArgs a{dy + start, 1, N, u + p * r, R, 1, Np, r, T, 0, scratch};
    const int prof = prof_begin(st);
    LSQ_TRY((run<false, false>(a, z, st)));
    LSQ_TRY(finish(scratch, z, Np, r, s, accumulate, dB + start * r, r, 1, st));
    if (prof >= 0)
      prof_end(prof, st, "lora_rank_r", 2.0 * T * r * Np, 2.0 * T * Np + 4.0 * T * r);
    start = part_end[p];
  }
  return LSQ_OK;
}

}  // namespace lsq

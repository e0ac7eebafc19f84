// LoRA rank-r products around the fused NF4 GEMM (CUDA cores, fp32).
//
// For y = x W^T + s (x A^T) B^T (Soup layer-streaming tutorial, "四段資料路徑"
// part 1) and its backward (part 3): u = x A^T (forward), v = dY B, and the
// trainable gradients dA = s v^T x, dB = s dY^T u.  All four are "tall x
// skinny" products: C[m, n] = sum_k P(m, k) Q(k, n) with n spanning at most a
// few r = 16 columns, P a bf16 activation and Q an fp32 LoRA tensor.
//
// One tiled kernel serves all four: a CTA owns 64 rows x BN columns of C over
// one slice of the reduction; bf16 P and fp32 Q tiles are staged through shared
// memory with coalesced loads along whichever index is contiguous in memory,
// each thread keeps a 4 x (BN/16) register tile, and the slices are summed by
// a second kernel in a fixed order - so results are deterministic (no atomics)
// and keep fp32 precision end to end.
#include "common.cuh"

namespace lsq {

namespace {

constexpr int kBM = 64;   // rows of C per CTA
constexpr int kBK = 32;   // reduction elements per smem tile
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

// P_RED: the reduction index is the contiguous one in P (else the row index m is).
// Q_RED: the reduction index is the contiguous one in Q (else the column n is).
template <bool P_RED, bool Q_RED, int BN>
__global__ void __launch_bounds__(kThreads) skinny_kernel(const SkinnyArgs a) {
  __shared__ float Ps[kBK][kBM + 4];
  __shared__ float Qs[kBK][BN + 4];
  constexpr int TN = BN / 16;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int64_t n0 = (int64_t)blockIdx.y * BN;
  const int z = blockIdx.z;
  const int64_t k_begin = (int64_t)z * a.k_per_split;
  const int64_t k_end = min(a.K, k_begin + a.k_per_split);
  float acc[4][TN];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  for (int64_t kb = k_begin; kb < k_end; kb += kBK) {
    // stage P tile (64 x 32) -> Ps[k][m]
#pragma unroll
    for (int it = 0; it < (kBM * kBK) / kThreads; ++it) {
      const int idx = tid + it * kThreads;
      int mm, kk;
      if (P_RED) {
        mm = idx / kBK;
        kk = idx % kBK;
      } else {
        kk = idx / kBM;
        mm = idx % kBM;
      }
      const int64_t m = m0 + mm, k = kb + kk;
      float v = 0.f;
      if (m < a.M && k < k_end) v = bf16_bits_to_float(__ldg(a.P + m * a.p_m + k * a.p_k));
      Ps[kk][mm] = v;
    }
    // stage Q tile (32 x BN) -> Qs[k][n]
#pragma unroll
    for (int it = 0; it < (kBK * BN + kThreads - 1) / kThreads; ++it) {
      const int idx = tid + it * kThreads;
      if (idx < kBK * BN) {
        int nn, kk;
        if (Q_RED) {
          nn = idx / kBK;
          kk = idx % kBK;
        } else {
          kk = idx / BN;
          nn = idx % BN;
        }
        const int64_t n = n0 + nn, k = kb + kk;
        float v = 0.f;
        if (n < a.N && k < k_end) v = __ldg(a.Q + k * a.q_k + n * a.q_n);
        Qs[kk][nn] = v;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kBK; ++kk) {
      float pv[4], qv[TN];
#pragma unroll
      for (int i = 0; i < 4; ++i) pv[i] = Ps[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < TN; ++j) qv[j] = Qs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(pv[i], qv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = a.part + (size_t)z * a.M * a.N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int64_t n = n0 + tx + 16 * j;
      if (n < a.N) out[m * a.N + n] = acc[i][j];
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

int bn_for(int64_t N) { return N <= 16 ? 16 : N <= 32 ? 32 : N <= 48 ? 48 : 64; }

// Splits of the reduction for a product: about two waves of CTAs on 148 SMs,
// each slice at least two smem tiles long.
int splits_for(int64_t M, int64_t N, int64_t K) {
  const int bn = bn_for(N);
  const int64_t xy = ((M + kBM - 1) / kBM) * ((N + bn - 1) / bn);
  int64_t z = (2 * 148 + xy - 1) / xy;
  const int64_t zmax = std::max<int64_t>(1, K / (2 * kBK));
  z = std::max<int64_t>(1, std::min<int64_t>(z, std::min<int64_t>(zmax, 64)));
  const int64_t kps = ((K + z - 1) / z + kBK - 1) / kBK * kBK;
  return (int)((K + kps - 1) / kps);
}

template <bool P_RED, bool Q_RED>
int run(const SkinnyArgs& a0, int splits, cudaStream_t st) {
  SkinnyArgs a = a0;
  a.k_per_split = ((a.K + splits - 1) / splits + kBK - 1) / kBK * kBK;
  const int bn = bn_for(a.N);
  dim3 grid((unsigned)((a.M + kBM - 1) / kBM), (unsigned)((a.N + bn - 1) / bn), (unsigned)splits);
  switch (bn) {
    case 16: skinny_kernel<P_RED, Q_RED, 16><<<grid, kThreads, 0, st>>>(a); break;
    case 32: skinny_kernel<P_RED, Q_RED, 32><<<grid, kThreads, 0, st>>>(a); break;
    case 48: skinny_kernel<P_RED, Q_RED, 48><<<grid, kThreads, 0, st>>>(a); break;
    default: skinny_kernel<P_RED, Q_RED, 64><<<grid, kThreads, 0, st>>>(a); break;
  }
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
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
  LSQ_TRY((run<true, true>(a, s, st)));
  return finish(scratch, s, T, R, 1.f, 0, u, R, 1, st);
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
    LSQ_TRY((run<true, false>(a, s, st)));
    LSQ_TRY(finish(scratch, s, T, r, 1.f, 0, v + p * r, R, 1, st));
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
  LSQ_TRY((run<false, false>(a, z, st)));
  return finish(scratch, z, K, R, s, accumulate, dA, 1, K, st);
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
    LSQ_TRY((run<false, false>(a, z, st)));
    LSQ_TRY(finish(scratch, z, Np, r, s, accumulate, dB + start * r, r, 1, st));
    start = part_end[p];
  }
  return LSQ_OK;
}

}  // namespace lsq

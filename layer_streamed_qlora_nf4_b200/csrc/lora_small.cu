// LoRA rank-r products around the fused NF4 GEMM (CUDA cores, fp32).
//
// For y = x W^T + s (x A^T) B^T (Soup layer-streaming tutorial, "四段資料路徑"
// part 1) and its backward (part 3): u = x A^T (forward), v = dY B, and the
// trainable gradients dA = s v^T x, dB = s dY^T u.  These are skinny (r = 16
// columns per projection) and bandwidth-light; every output element is a
// fixed-order fp32 sum, so the results are deterministic (no atomics).
#include "common.cuh"

namespace lsq {

namespace {

constexpr int kKChunk = 128;   // contraction chunk per CTA in the K-split products
constexpr int kTTile = 32;     // tokens per CTA

// C[t, j] partial over a K chunk: part[kc][t][j] = sum_{k in chunk} X[t, k] * Y(j, k)
// with Y(j, k) = Yp[j * ysj + k * ysk].  X bf16 [T, ldx].
__global__ void skinny_partial_kernel(const uint16_t* __restrict__ X, int64_t ldx,
                                      const float* __restrict__ Y, int64_t ysj, int64_t ysk,
                                      int64_t T, int64_t K, int R, float* __restrict__ part,
                                      int64_t part_ld, int col0) {
  extern __shared__ float sm[];
  float* xs = sm;                              // [kTTile][kKChunk]
  float* ys = sm + kTTile * kKChunk;           // [R][kKChunk + 1]
  const int64_t t0 = (int64_t)blockIdx.x * kTTile;
  const int kc = blockIdx.y;
  const int64_t k0 = (int64_t)kc * kKChunk;
  const int kn = (int)((kKChunk) < (K - k0) ? (kKChunk) : (K - k0));
  for (int i = threadIdx.x; i < kTTile * kKChunk; i += blockDim.x) {
    const int tt = i / kKChunk, kk = i % kKChunk;
    const int64_t t = t0 + tt;
    xs[i] = (t < T && kk < kn) ? bf16_bits_to_float(X[t * ldx + k0 + kk]) : 0.f;
  }
  for (int i = threadIdx.x; i < R * kKChunk; i += blockDim.x) {
    const int j = i / kKChunk, kk = i % kKChunk;
    ys[j * (kKChunk + 1) + kk] = (kk < kn) ? Y[(int64_t)j * ysj + (k0 + kk) * ysk] : 0.f;
  }
  __syncthreads();
  for (int o = threadIdx.x; o < kTTile * R; o += blockDim.x) {
    const int tt = o / R, j = o % R;
    const float* xr = xs + tt * kKChunk;
    const float* yr = ys + j * (kKChunk + 1);
    float acc = 0.f;
#pragma unroll 8
    for (int kk = 0; kk < kKChunk; ++kk) acc = fmaf(xr[kk], yr[kk], acc);
    const int64_t t = t0 + tt;
    if (t < T) part[((int64_t)kc * T + t) * part_ld + col0 + j] = acc;
  }
}

// out[t, j] = sum_kc part[kc][t][j]  (fixed order)
__global__ void partial_sum_kernel(const float* __restrict__ part, int nkc, int64_t T, int64_t ld,
                                   int col0, int R, float* __restrict__ out, int64_t ldo) {
  const int64_t n = T * R;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / R;
    const int j = (int)(i % R);
    float acc = 0.f;
    for (int c = 0; c < nkc; ++c) acc += part[((int64_t)c * T + t) * ld + col0 + j];
    out[t * ldo + col0 + j] = acc;
  }
}

// dA[j, k] (+)= s * sum_t v[t, j] * x[t, k]; thread = one k, 8 consecutive j
__global__ void lora_grad_a_kernel(const float* __restrict__ v, const uint16_t* __restrict__ x,
                                   int64_t T, int64_t K, int R, float s, int accumulate,
                                   float* __restrict__ dA) {
  __shared__ float vs[64][8];
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int j0 = blockIdx.y * 8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int64_t tb = 0; tb < T; tb += 64) {
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 8; i += blockDim.x) {
      const int tt = i / 8, jj = i % 8;
      const int64_t t = tb + tt;
      vs[tt][jj] = (t < T && j0 + jj < R) ? v[t * R + j0 + jj] : 0.f;
    }
    __syncthreads();
    if (k < K) {
      const int tn = (int)((64) < (T - tb) ? (64) : (T - tb));
      for (int tt = 0; tt < tn; ++tt) {
        const float xv = bf16_bits_to_float(x[(tb + tt) * K + k]);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[jj] = fmaf(vs[tt][jj], xv, acc[jj]);
      }
    }
  }
  if (k < K) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = j0 + jj;
      if (j < R) {
        float* d = dA + (int64_t)j * K + k;
        *d = (accumulate ? *d : 0.f) + s * acc[jj];
      }
    }
  }
}

// dB[n, j] (+)= s * sum_t dy[t, n] * u[t, part(n) r + j]; thread = one n, all r (<= 64) j
template <int RMAX>
__global__ void lora_grad_b_kernel(const uint16_t* __restrict__ dy, const float* __restrict__ u,
                                   int64_t T, int64_t N, int r, int R, int n_parts, int64_t pe0,
                                   int64_t pe1, int64_t pe2, int64_t pe3, float s, int accumulate,
                                   float* __restrict__ dB) {
  __shared__ float us[32][RMAX * 4];  // 32 tokens x (up to 4 parts x r)
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t pe[4] = {pe0, pe1, pe2, pe3};
  int part = 0;
  if (n < N)
    while (part + 1 < n_parts && n >= pe[part]) ++part;
  float acc[RMAX];
#pragma unroll
  for (int j = 0; j < RMAX; ++j) acc[j] = 0.f;
  for (int64_t tb = 0; tb < T; tb += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * R; i += blockDim.x) {
      const int tt = i / R, jj = i % R;
      const int64_t t = tb + tt;
      us[tt][jj] = (t < T) ? u[t * R + jj] : 0.f;
    }
    __syncthreads();
    if (n < N) {
      const int tn = (int)((32) < (T - tb) ? (32) : (T - tb));
      for (int tt = 0; tt < tn; ++tt) {
        const float g = bf16_bits_to_float(dy[(tb + tt) * N + n]);
        const float* ur = &us[tt][part * r];
#pragma unroll
        for (int j = 0; j < RMAX; ++j)
          if (j < r) acc[j] = fmaf(g, ur[j], acc[j]);
      }
    }
  }
  if (n < N) {
#pragma unroll
    for (int j = 0; j < RMAX; ++j) {
      if (j < r) {
        float* d = dB + n * r + j;
        *d = (accumulate ? *d : 0.f) + s * acc[j];
      }
    }
  }
}

int run_skinny(const uint16_t* X, int64_t ldx, const float* Y, int64_t ysj, int64_t ysk, int64_t T,
               int64_t K, int R, float* out, int64_t ldo, int col0, float* part, cudaStream_t st) {
  const int nkc = (int)((K + kKChunk - 1) / kKChunk);
  dim3 grid((unsigned)((T + kTTile - 1) / kTTile), (unsigned)nkc);
  const size_t smem = (size_t)(kTTile * kKChunk + R * (kKChunk + 1)) * sizeof(float);
  if (smem > 200 * 1024) return set_error(LSQ_ERR_SHAPE, "lora: rank too large");
  static bool attr = false;
  if (!attr) {
    LSQ_CUDA(cudaFuncSetAttribute(skinny_partial_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
    attr = true;
  }
  skinny_partial_kernel<<<grid, 256, smem, st>>>(X, ldx, Y, ysj, ysk, T, K, R, part, ldo, col0);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  const int64_t n = T * R;
  partial_sum_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(
      part, nkc, T, ldo, col0, R, out, ldo);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

}  // namespace

size_t lora_scratch_bytes(int64_t T, int64_t K, int R) {
  const int64_t nkc = (K + kKChunk - 1) / kKChunk;
  return (size_t)(nkc * T * R) * sizeof(float);
}

int launch_lora_down(const uint16_t* x, int64_t ldx, const float* A, int64_t T, int64_t K, int R,
                     float* u, float* scratch, size_t scratch_bytes, cudaStream_t st) {
  const size_t need = lora_scratch_bytes(T, K, R);
  if (!scratch || scratch_bytes < need)
    return set_error(LSQ_ERR_WORKSPACE, "lora_down: scratch %zu < %zu", scratch_bytes, need);
  return run_skinny(x, ldx, A, K, 1, T, K, R, u, R, 0, scratch, st);
}

int launch_lora_vproj(const uint16_t* dy, int64_t T, int64_t N, const float* B, int r, int n_parts,
                      const int64_t* part_end, float* v, float* scratch, size_t scratch_bytes,
                      cudaStream_t st) {
  const int R = n_parts * r;
  int64_t start = 0;
  for (int p = 0; p < n_parts; ++p) {
    const int64_t end = part_end[p];
    const int64_t Np = end - start;
    const size_t need = lora_scratch_bytes(T, Np, R);
    if (!scratch || scratch_bytes < need)
      return set_error(LSQ_ERR_WORKSPACE, "lora_vproj: scratch %zu < %zu", scratch_bytes, need);
    LSQ_TRY(run_skinny(dy + start, N, B + start * r, 1, r, T, Np, r, v, R, p * r, scratch, st));
    start = end;
  }
  return LSQ_OK;
}

int launch_lora_grad_a(const float* v, const uint16_t* x, int64_t T, int64_t K, int R, float s,
                       int accumulate, float* dA, cudaStream_t st) {
  dim3 grid((unsigned)((K + 127) / 128), (unsigned)((R + 7) / 8));
  lora_grad_a_kernel<<<grid, 128, 0, st>>>(v, x, T, K, R, s, accumulate, dA);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

int launch_lora_grad_b(const uint16_t* dy, const float* u, int64_t T, int64_t N, int r, int R,
                       int n_parts, const int64_t* part_end, float s, int accumulate, float* dB,
                       cudaStream_t st) {
  if (n_parts < 1 || n_parts > 4 || R > 256) return set_error(LSQ_ERR_SHAPE, "lora_grad_b: parts");
  int64_t pe[4] = {N, N, N, N};
  for (int p = 0; p < n_parts; ++p) pe[p] = part_end[p];
  const unsigned grid = (unsigned)((N + 127) / 128);
  if (r <= 16)
    lora_grad_b_kernel<16><<<grid, 128, 0, st>>>(dy, u, T, N, r, R, n_parts, pe[0], pe[1], pe[2],
                                                 pe[3], s, accumulate, dB);
  else if (r <= 32)
    lora_grad_b_kernel<32><<<grid, 128, 0, st>>>(dy, u, T, N, r, R, n_parts, pe[0], pe[1], pe[2],
                                                 pe[3], s, accumulate, dB);
  else if (r <= 64)
    lora_grad_b_kernel<64><<<grid, 128, 0, st>>>(dy, u, T, N, r, R, n_parts, pe[0], pe[1], pe[2],
                                                 pe[3], s, accumulate, dB);
  else
    return set_error(LSQ_ERR_SHAPE, "lora_grad_b: r > 64 unsupported");
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

}  // namespace lsq

// NF4 codebook (derived on the host from its definition), blockwise-absmax
// quantisation and dequantisation kernels.
//
// Definition followed (Soup layer-streaming tutorial, "四段資料路徑" part 1: the
// frozen Linear weights are stored as 4-bit NormalFloat, NF4, computed offline):
//   levels: standard-normal quantiles with an exact zero - 8 positive levels at
//   p = delta + i (1/2 - delta) / 8 (i = 0..7), 7 negative levels at
//   -Phi^-1(delta + i (1/2 - delta) / 7) (i = 0..6), plus 0, divided by
//   Phi^-1(delta), with delta = ((1 - 1/30) + (1 - 1/32)) / 2; each level is
//   rounded once to fp32.  Phi^-1 here is found by bisection on
//   Phi(x) = erfc(-x / sqrt 2) / 2 in long double.
//   block of 64 consecutive elements, absmax = max |w| (fp32);
//   code = #{ fp32 midpoints strictly below fl32(w / absmax) }; absmax 0 -> 7;
//   two codes per byte, even element in the high nibble.
#include <math.h>

#include <mutex>

#include "common.cuh"

namespace lsq {

namespace {

float g_levels[16];
float g_mids[15];

long double phi_inv(long double p) {
  long double lo = -12.0L, hi = 12.0L;
  const long double rs2 = 0.70710678118654752440084436210484903928L;
  for (int i = 0; i < 200; ++i) {
    long double mid = 0.5L * (lo + hi);
    long double cdf = 0.5L * erfcl(-mid * rs2);
    if (cdf < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5L * (lo + hi);
}

void build_codebook() {
  const long double delta = ((1.0L - 1.0L / 30.0L) + (1.0L - 1.0L / 32.0L)) / 2.0L;
  long double v[16];
  int n = 0;
  for (int i = 0; i < 7; ++i) v[n++] = -phi_inv(delta + i * (0.5L - delta) / 7.0L);
  v[n++] = 0.0L;
  for (int i = 7; i >= 0; --i) v[n++] = phi_inv(delta + i * (0.5L - delta) / 8.0L);
  const long double top = phi_inv(delta);
  for (int i = 0; i < 16; ++i) g_levels[i] = (float)(v[i] / top);
  g_levels[0] = -1.0f;   // -Phi^-1(delta)/Phi^-1(delta), exact
  g_levels[7] = 0.0f;
  g_levels[15] = 1.0f;
  for (int i = 0; i < 15; ++i) {
    volatile float s = g_levels[i] + g_levels[i + 1];  // fp32 sum, then exact halving
    g_mids[i] = s * 0.5f;
  }
}

std::once_flag g_once;

struct QuantParams {
  float mids[15];
};

// One warp per 64-element block; lane l owns elements 2l and 2l+1 (one byte).
__global__ void nf4_quantize_kernel(const float* __restrict__ W, int64_t n_blocks,
                                    uint8_t* __restrict__ codes, float* __restrict__ absmax,
                                    QuantParams qp, int* dev_err) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t b = warp_global; b < n_blocks; b += n_warps) {
    const float2 w = reinterpret_cast<const float2*>(W + b * 64)[lane];
    // non-finite, or beyond the fp16 range the fused GEMM's forward operand has
    const bool finite = fabsf(w.x) <= kF16Max && fabsf(w.y) <= kF16Max;
    if (!__all_sync(0xFFFFFFFFu, finite) && lane == 0) atomicOr(dev_err, DEV_ERR_NONFINITE);
    float am = fmaxf(fabsf(w.x), fabsf(w.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    uint32_t c0 = 7, c1 = 7;
    if (am > 0.f) {
      const float v0 = __fdiv_rn(w.x, am), v1 = __fdiv_rn(w.y, am);
      c0 = 0;
      c1 = 0;
#pragma unroll
      for (int i = 0; i < 15; ++i) {
        c0 += (v0 > qp.mids[i]) ? 1u : 0u;
        c1 += (v1 > qp.mids[i]) ? 1u : 0u;
      }
    }
    codes[b * 32 + lane] = (uint8_t)((c0 << 4) | c1);
    if (lane == 0) absmax[b] = am;
  }
}

struct LevelParams {
  float lv[16];
};

__global__ void nf4_dequantize_kernel(const uint8_t* __restrict__ codes,
                                      const float* __restrict__ absmax, int64_t n_bytes,
                                      float* __restrict__ W, LevelParams lp) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n_bytes;
       j += (int64_t)gridDim.x * blockDim.x) {
    const uint8_t c = codes[j];
    const float am = absmax[j >> 5];  // 32 bytes per 64-element block
    W[2 * j] = lp.lv[c >> 4] * am;
    W[2 * j + 1] = lp.lv[c & 15] * am;
  }
}

// Double quantisation of the absmax: one CTA of 256 threads per run of 256
// absmax values (the last run may be short).  s = fl32(max / 255), q =
// rint(fl32(a / s)) (half to even), at most 255; a run of zeros gets s = 0, q = 0.
__global__ void absmax_q8_kernel(const float* __restrict__ absmax, int64_t n,
                                 uint8_t* __restrict__ q, float* __restrict__ scale) {
  __shared__ float wmax[8];
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const float a = (i < n) ? absmax[i] : 0.f;
  float m = a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  float mx = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, wmax[w]);
  const float s = (mx > 0.f) ? __fdiv_rn(mx, 255.f) : 0.f;
  if (i < n) {
    int v = 0;
    if (mx > 0.f) v = min(255, __float2int_rn(__fdiv_rn(a, s)));
    q[i] = (uint8_t)v;
  }
  if (threadIdx.x == 0) scale[blockIdx.x] = s;
}

__global__ void nf4_dequantize_dq_kernel(const uint8_t* __restrict__ codes,
                                         const uint8_t* __restrict__ q,
                                         const float* __restrict__ scale, int64_t n_bytes,
                                         float* __restrict__ W, LevelParams lp) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n_bytes;
       j += (int64_t)gridDim.x * blockDim.x) {
    const uint8_t c = codes[j];
    const int64_t b = j >> 5;  // 32 bytes per 64-element block
    const float am = (float)q[b] * scale[b >> 8];
    W[2 * j] = lp.lv[c >> 4] * am;
    W[2 * j + 1] = lp.lv[c & 15] * am;
  }
}

}  // namespace

const float* nf4_levels() {
  std::call_once(g_once, build_codebook);
  return g_levels;
}
const float* nf4_midpoints() {
  std::call_once(g_once, build_codebook);
  return g_mids;
}

}  // namespace lsq

using namespace lsq;

extern "C" int lsq_nf4_codebook(float out_levels[16]) {
  if (!out_levels) return set_error(LSQ_ERR_INVALID, "lsq_nf4_codebook: null output");
  const float* lv = nf4_levels();
  for (int i = 0; i < 16; ++i) out_levels[i] = lv[i];
  return LSQ_OK;
}

static int check_nf4_shape(int64_t N, int64_t K, int32_t block, const char* who) {
  if (block != 64) return set_error(LSQ_ERR_SHAPE, "%s: block must be 64 (got %d)", who, block);
  if (N <= 0 || K <= 0) return set_error(LSQ_ERR_SHAPE, "%s: N and K must be positive", who);
  if (K % 64 != 0) return set_error(LSQ_ERR_SHAPE, "%s: K %% 64 != 0 (K=%lld)", who, (long long)K);
  if ((N * K) % 2 != 0) return set_error(LSQ_ERR_SHAPE, "%s: N*K must be even", who);
  return LSQ_OK;
}

extern "C" int nf4_quantize(const float* W, int64_t N, int64_t K, int32_t block, uint8_t* codes,
                            float* absmax, void* stream) {
  LSQ_TRY(check_nf4_shape(N, K, block, "nf4_quantize"));
  if (!W || !codes || !absmax) return set_error(LSQ_ERR_INVALID, "nf4_quantize: null pointer");
  if (!aligned16(W) || !aligned16(codes) || !aligned16(absmax))
    return set_error(LSQ_ERR_ALIGN, "nf4_quantize: pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err = device_status_ptr();
  if (!err) return set_error(LSQ_ERR_CUDA, "nf4_quantize: no device status word");
  int h_before = 0;
  LSQ_CUDA(cudaMemcpyAsync(&h_before, err, sizeof(int), cudaMemcpyDeviceToHost, st));
  LSQ_CUDA(cudaStreamSynchronize(st));
  if (h_before & DEV_ERR_NONFINITE) {
    int v = h_before & ~DEV_ERR_NONFINITE;
    LSQ_CUDA(cudaMemcpyAsync(err, &v, sizeof(int), cudaMemcpyHostToDevice, st));
  }
  QuantParams qp;
  const float* m = nf4_midpoints();
  for (int i = 0; i < 15; ++i) qp.mids[i] = m[i];
  const int64_t n_blocks = N * K / 64;
  const int threads = 256;
  int64_t grid = (n_blocks * 32 + threads - 1) / threads;
  const int64_t cap = (int64_t)gemm_num_sms() * 32;
  if (grid > cap) grid = cap;
  nf4_quantize_kernel<<<(unsigned)grid, threads, 0, st>>>(W, n_blocks, codes, absmax, qp, err);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  int h_after = 0;
  LSQ_CUDA(cudaMemcpyAsync(&h_after, err, sizeof(int), cudaMemcpyDeviceToHost, st));
  LSQ_CUDA(cudaStreamSynchronize(st));
  if (h_after & DEV_ERR_NONFINITE) {
    int v = h_after & ~DEV_ERR_NONFINITE;
    LSQ_CUDA(cudaMemcpy(err, &v, sizeof(int), cudaMemcpyHostToDevice));
    return set_error(LSQ_ERR_INVALID,
                     "nf4_quantize: W holds a NaN, an Inf or a value beyond 65504 in magnitude");
  }
  return LSQ_OK;
}

extern "C" int nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t N, int64_t K,
                              int32_t block, float* W_out, void* stream) {
  LSQ_TRY(check_nf4_shape(N, K, block, "nf4_dequantize"));
  if (!W_out || !codes || !absmax) return set_error(LSQ_ERR_INVALID, "nf4_dequantize: null pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LevelParams lp;
  const float* lv = nf4_levels();
  for (int i = 0; i < 16; ++i) lp.lv[i] = lv[i];
  const int64_t n_bytes = N * K / 2;
  int64_t grid = (n_bytes + 255) / 256;
  const int64_t cap = (int64_t)gemm_num_sms() * 16;
  if (grid > cap) grid = cap;
  nf4_dequantize_kernel<<<(unsigned)grid, 256, 0, st>>>(codes, absmax, n_bytes, W_out, lp);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

extern "C" int nf4_absmax_quantize8(const float* absmax, int64_t n_blocks, uint8_t* q,
                                    float* scale, void* stream) {
  if (n_blocks <= 0) return set_error(LSQ_ERR_SHAPE, "nf4_absmax_quantize8: n_blocks must be positive");
  if (!absmax || !q || !scale) return set_error(LSQ_ERR_INVALID, "nf4_absmax_quantize8: null pointer");
  if (!aligned16(q)) return set_error(LSQ_ERR_ALIGN, "nf4_absmax_quantize8: q must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t groups = (n_blocks + 255) / 256;
  if (groups > INT32_MAX) return set_error(LSQ_ERR_SHAPE, "nf4_absmax_quantize8: too many blocks");
  absmax_q8_kernel<<<(unsigned)groups, 256, 0, st>>>(absmax, n_blocks, q, scale);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

extern "C" int nf4_dequantize_dq(const uint8_t* codes, const uint8_t* q, const float* scale,
                                 int64_t N, int64_t K, int32_t block, float* W_out, void* stream) {
  LSQ_TRY(check_nf4_shape(N, K, block, "nf4_dequantize_dq"));
  if (!W_out || !codes || !q || !scale)
    return set_error(LSQ_ERR_INVALID, "nf4_dequantize_dq: null pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LevelParams lp;
  const float* lv = nf4_levels();
  for (int i = 0; i < 16; ++i) lp.lv[i] = lv[i];
  const int64_t n_bytes = N * K / 2;
  int64_t grid = (n_bytes + 255) / 256;
  const int64_t cap = (int64_t)gemm_num_sms() * 16;
  if (grid > cap) grid = cap;
  nf4_dequantize_dq_kernel<<<(unsigned)grid, 256, 0, st>>>(codes, q, scale, n_bytes, W_out, lp);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

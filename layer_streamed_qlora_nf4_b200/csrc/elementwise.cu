// Memory-bound kernels of the decoder layer and the stack ends: split-K reduce,
// RMSNorm fwd/bwd, rotate-half RoPE fwd/bwd, SwiGLU fwd/bwd, embedding gather,
// cross-entropy, AdamW.  Vectorised 16-byte accesses, warp-shuffle reductions
// in a fixed order (deterministic), fp32 arithmetic.  Storage: the residual
// stream is fp32, forward activations fp16 (the forward GEMMs' operand type),
// gradients bf16 or fp32.
//
// Definitions (Llama-style decoder named by the Soup layer-streaming tutorial,
// "維護者的 4GB／8B 成績"; norms kept at higher precision, "四段資料路徑" part 1):
//   RMSNorm  y = x (mean(x^2) + eps)^-1/2 g
//   RoPE     rotate-half pairs (i, i + d/2), angle = pos theta^(-2i/d)
//   SwiGLU   m = silu(gate) * up
//   SFT loss mean cross-entropy of next-token targets
//   AdamW    decoupled weight decay, bias-corrected moments
#include <math.h>

#include "common.cuh"

namespace lsq {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

unsigned grid_for(int64_t n, int threads, int per_thread = 1) {
  int64_t g = (n + (int64_t)threads * per_thread - 1) / ((int64_t)threads * per_thread);
  const int64_t cap = (int64_t)gemm_num_sms() * 32;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (unsigned)g;
}

// ------------------------------------------------------------------ split-K reduce
// out = sum over splits in order (+ fp32 residual); out_kind OUT_F32, OUT_BF16 or
// OUT_F16 (an fp16 result beyond the fp16 range latches the non-finite bit)
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, int64_t T,
                                     int64_t M, void* __restrict__ out, int out_kind, int64_t ldo,
                                     const float* __restrict__ res, int64_t ldr, int* dev_err) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t n4 = T * M / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 4;
    const int64_t t = e / M, m = e % M;
    float4 acc = reinterpret_cast<const float4*>(part)[i];
    for (int s = 1; s < splits; ++s) {
      const float4 v = reinterpret_cast<const float4*>(part + (size_t)s * T * M)[i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (res) {
      const float4 r = *reinterpret_cast<const float4*>(res + t * ldr + m);
      acc.x += r.x;
      acc.y += r.y;
      acc.z += r.z;
      acc.w += r.w;
    }
    if (out_kind == OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + t * ldo + m) = acc;
    } else if (out_kind == OUT_F16) {
      if (!(fmaxf(fmaxf(fabsf(acc.x), fabsf(acc.y)), fmaxf(fabsf(acc.z), fabsf(acc.w))) <= kF16Max))
        atomicOr(dev_err, DEV_ERR_NONFINITE);
      uint2 o;
      o.x = pack_f16x2(acc.x, acc.y);
      o.y = pack_f16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + t * ldo + m) = o;
    } else {
      uint2 o;
      o.x = pack_bf16x2(acc.x, acc.y);
      o.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + t * ldo + m) = o;
    }
  }
}

// ------------------------------------------------------------------ RMSNorm
// One CTA per row, 8 elements (two 16-byte loads of fp32) per thread per pass; D % 8 == 0.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += red[i];  // fixed order
  return t;
}

template <bool F16OUT>
__global__ void rmsnorm_fwd_kernel(const float* __restrict__ x, const uint16_t* __restrict__ g,
                                   int64_t D, float eps, uint16_t* __restrict__ y,
                                   float* __restrict__ rstd, int* dev_err) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + row * D);
  const uint4* gr = reinterpret_cast<const uint4*>(g);
  uint4* yr = reinterpret_cast<uint4*>(y + row * D);
  const int nv = (int)(D / 8);
  float ss = 0.f;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 a = xr[2 * i], b = xr[2 * i + 1];
    ss = fmaf(a.x, a.x, ss);
    ss = fmaf(a.y, a.y, ss);
    ss = fmaf(a.z, a.z, ss);
    ss = fmaf(a.w, a.w, ss);
    ss = fmaf(b.x, b.x, ss);
    ss = fmaf(b.y, b.y, ss);
    ss = fmaf(b.z, b.z, ss);
    ss = fmaf(b.w, b.w, ss);
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)D + eps);
  if (threadIdx.x == 0 && rstd) rstd[row] = r;
  bool big = false;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 a = xr[2 * i], b = xr[2 * i + 1];
    const uint4 gv = gr[i];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 gg = unpack_bf16x2(gw[q]);
      const float y0 = f[2 * q] * r * gg.x, y1 = f[2 * q + 1] * r * gg.y;
      if (F16OUT) {
        big |= !(fmaxf(fabsf(y0), fabsf(y1)) <= kF16Max);
        o[q] = pack_f16x2(y0, y1);
      } else {
        o[q] = pack_bf16x2(y0, y1);
      }
    }
    yr[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (F16OUT && big) atomicOr(dev_err, DEV_ERR_NONFINITE);
}

// dx = dres + r (g dy) - x r^3 sum(g dy x) / D;  one CTA per row, 4 elements per thread per pass
__global__ void rmsnorm_bwd_kernel(const float* __restrict__ dy, const float* __restrict__ x,
                                   const uint16_t* __restrict__ g, const float* __restrict__ rstd,
                                   const float* __restrict__ dres, int64_t D,
                                   float* __restrict__ dx, uint16_t* __restrict__ dxb) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int nv = (int)(D / 4);
  const float4* dyr = reinterpret_cast<const float4*>(dy + row * D);
  const float4* xr = reinterpret_cast<const float4*>(x + row * D);
  const uint2* gr = reinterpret_cast<const uint2*>(g);
  float dot = 0.f;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 d = dyr[i], xv = xr[i];
    const uint2 gv = gr[i];
    const float2 g0 = unpack_bf16x2(gv.x), g1 = unpack_bf16x2(gv.y);
    dot += d.x * g0.x * xv.x + d.y * g0.y * xv.y + d.z * g1.x * xv.z + d.w * g1.y * xv.w;
  }
  dot = block_sum(dot, red);
  const float r = rstd[row];
  const float c = r * r * r * dot / (float)D;
  const float4* rr = dres ? reinterpret_cast<const float4*>(dres + row * D) : nullptr;
  float4* o = reinterpret_cast<float4*>(dx + row * D);
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 d = dyr[i], xv = xr[i];
    const uint2 gv = gr[i];
    const float2 g0 = unpack_bf16x2(gv.x), g1 = unpack_bf16x2(gv.y);
    float4 v;
    v.x = r * g0.x * d.x - xv.x * c;
    v.y = r * g0.y * d.y - xv.y * c;
    v.z = r * g1.x * d.z - xv.z * c;
    v.w = r * g1.y * d.w - xv.w * c;
    if (rr) {
      const float4 a = rr[i];
      v.x += a.x;
      v.y += a.y;
      v.z += a.z;
      v.w += a.w;
    }
    o[i] = v;
    if (dxb) {
      uint2 b;
      b.x = pack_bf16x2(v.x, v.y);
      b.y = pack_bf16x2(v.z, v.w);
      reinterpret_cast<uint2*>(dxb + row * D)[i] = b;
    }
  }
}

// RMSNorm of a split product's output: x_out = (sum of the n_parts partials, in
// slice order) + res, then y = RMSNorm(x_out) - the same sums, in the same order,
// as launch_splitk_reduce followed by rmsnorm_fwd_kernel (same thread mapping).
// The summed row is staged in shared memory (D floats) for the second pass.
template <bool F16OUT>
__global__ void rmsnorm_fwd_sum_kernel(const float* __restrict__ parts, int n_parts,
                                       int64_t pstride, const float* __restrict__ res, int64_t D,
                                       float eps, const uint16_t* __restrict__ g,
                                       float* __restrict__ xo, uint16_t* __restrict__ y,
                                       float* __restrict__ rstd, int* dev_err) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  extern __shared__ float4 row_sh[];
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int nv = (int)(D / 8);
  float ss = 0.f;
  bool big = false;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const int64_t e = row * D + 8 * (int64_t)i;
    float4 a = *reinterpret_cast<const float4*>(parts + e);
    float4 b = *reinterpret_cast<const float4*>(parts + e + 4);
    for (int s = 1; s < n_parts; ++s) {
      const float4 pa = *reinterpret_cast<const float4*>(parts + (size_t)s * pstride + e);
      const float4 pb = *reinterpret_cast<const float4*>(parts + (size_t)s * pstride + e + 4);
      a.x += pa.x; a.y += pa.y; a.z += pa.z; a.w += pa.w;
      b.x += pb.x; b.y += pb.y; b.z += pb.z; b.w += pb.w;
    }
    if (res) {
      const float4 ra = *reinterpret_cast<const float4*>(res + e);
      const float4 rb = *reinterpret_cast<const float4*>(res + e + 4);
      a.x += ra.x; a.y += ra.y; a.z += ra.z; a.w += ra.w;
      b.x += rb.x; b.y += rb.y; b.z += rb.z; b.w += rb.w;
    }
    *reinterpret_cast<float4*>(xo + e) = a;
    *reinterpret_cast<float4*>(xo + e + 4) = b;
    row_sh[2 * i] = a;
    row_sh[2 * i + 1] = b;
    ss = fmaf(a.x, a.x, ss);
    ss = fmaf(a.y, a.y, ss);
    ss = fmaf(a.z, a.z, ss);
    ss = fmaf(a.w, a.w, ss);
    ss = fmaf(b.x, b.x, ss);
    ss = fmaf(b.y, b.y, ss);
    ss = fmaf(b.z, b.z, ss);
    ss = fmaf(b.w, b.w, ss);
  }
  ss = block_sum(ss, red);  // (its barriers also publish row_sh)
  const float r = rsqrtf(ss / (float)D + eps);
  if (threadIdx.x == 0 && rstd) rstd[row] = r;
  const uint4* gr = reinterpret_cast<const uint4*>(g);
  uint4* yr = reinterpret_cast<uint4*>(y + row * D);
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 a = row_sh[2 * i], b = row_sh[2 * i + 1];
    const uint4 gv = gr[i];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 gg = unpack_bf16x2(gw[q]);
      const float y0 = f[2 * q] * r * gg.x, y1 = f[2 * q + 1] * r * gg.y;
      if (F16OUT) {
        big |= !(fmaxf(fabsf(y0), fabsf(y1)) <= kF16Max);
        o[q] = pack_f16x2(y0, y1);
      } else {
        o[q] = pack_bf16x2(y0, y1);
      }
    }
    yr[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (F16OUT && big) atomicOr(dev_err, DEV_ERR_NONFINITE);
}

// rmsnorm_bwd_kernel with dy the sum of a split product's partials (slice order),
// staged in shared memory (D floats) for the second pass.
__global__ void rmsnorm_bwd_sum_kernel(const float* __restrict__ parts, int n_parts,
                                       int64_t pstride, const float* __restrict__ x,
                                       const uint16_t* __restrict__ g,
                                       const float* __restrict__ rstd,
                                       const float* __restrict__ dres, int64_t D,
                                       float* __restrict__ dx, uint16_t* __restrict__ dxb) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  extern __shared__ float4 row_sh[];
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int nv = (int)(D / 4);
  const float4* xr = reinterpret_cast<const float4*>(x + row * D);
  const uint2* gr = reinterpret_cast<const uint2*>(g);
  float dot = 0.f;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const int64_t e = row * D + 4 * (int64_t)i;
    float4 d = *reinterpret_cast<const float4*>(parts + e);
    for (int s = 1; s < n_parts; ++s) {
      const float4 p = *reinterpret_cast<const float4*>(parts + (size_t)s * pstride + e);
      d.x += p.x; d.y += p.y; d.z += p.z; d.w += p.w;
    }
    row_sh[i] = d;
    const float4 xv = xr[i];
    const uint2 gv = gr[i];
    const float2 g0 = unpack_bf16x2(gv.x), g1 = unpack_bf16x2(gv.y);
    dot += d.x * g0.x * xv.x + d.y * g0.y * xv.y + d.z * g1.x * xv.z + d.w * g1.y * xv.w;
  }
  dot = block_sum(dot, red);  // (its barriers also publish row_sh)
  const float r = rstd[row];
  const float c = r * r * r * dot / (float)D;
  const float4* rr = dres ? reinterpret_cast<const float4*>(dres + row * D) : nullptr;
  float4* o = reinterpret_cast<float4*>(dx + row * D);
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 d = row_sh[i], xv = xr[i];
    const uint2 gv = gr[i];
    const float2 g0 = unpack_bf16x2(gv.x), g1 = unpack_bf16x2(gv.y);
    float4 v;
    v.x = r * g0.x * d.x - xv.x * c;
    v.y = r * g0.y * d.y - xv.y * c;
    v.z = r * g1.x * d.z - xv.z * c;
    v.w = r * g1.y * d.w - xv.w * c;
    if (rr) {
      const float4 a = rr[i];
      v.x += a.x;
      v.y += a.y;
      v.z += a.z;
      v.w += a.w;
    }
    o[i] = v;
    if (dxb) {
      uint2 b;
      b.x = pack_bf16x2(v.x, v.y);
      b.y = pack_bf16x2(v.z, v.w);
      reinterpret_cast<uint2*>(dxb + row * D)[i] = b;
    }
  }
}

// ------------------------------------------------------------------ RoPE
// cs[pos][i] = (cos, sin)(pos * theta^(-2i/d)), evaluated in double, rounded to fp32.
__global__ void rope_table_kernel(int seq, int half, int d, double log_theta, float2* __restrict__ cs) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int n = seq * half;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
    const int pos = k / half, i = k % half;
    const double ang = (double)pos * exp(-2.0 * (double)i / (double)d * log_theta);
    double sd, cd;
    sincos(ang, &sd, &cd);
    cs[k] = make_float2((float)cd, (float)sd);
  }
}

// In-place rotation of the q and k heads of the fused qkv buffer (fp16); a
// thread rotates 8 pairs (i, i + d/2).
__global__ void rope_kernel(uint16_t* __restrict__ qkv, int64_t T, int seq, int H, int Hkv, int d,
                            const float2* __restrict__ cs) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int half = d / 2, chunks = half / 8;
  const int64_t ld = (int64_t)(H + 2 * Hkv) * d;
  const int64_t n = T * (H + Hkv) * chunks;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int ch = (int)(i % chunks);
    const int64_t th = i / chunks;
    const int head = (int)(th % (H + Hkv));
    const int64_t t = th / (H + Hkv);
    const int pos = (int)(t % seq);
    uint16_t* base = qkv + t * ld + (int64_t)head * d + ch * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(base);
    const uint4 b = *reinterpret_cast<const uint4*>(base + half);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
    const float2* c = cs + (int64_t)pos * half + ch * 8;
    uint32_t oa[4], ob[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x1 = unpack_f16x2(aw[q]), x2 = unpack_f16x2(bw[q]);
      const float2 c0 = c[2 * q], c1 = c[2 * q + 1];
      oa[q] = pack_f16x2(x1.x * c0.x - x2.x * c0.y, x1.y * c1.x - x2.y * c1.y);
      ob[q] = pack_f16x2(x2.x * c0.x + x1.x * c0.y, x2.y * c1.x + x1.y * c1.y);
    }
    *reinterpret_cast<uint4*>(base) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
    *reinterpret_cast<uint4*>(base + half) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
  }
}

// The fused q|k|v product's partials summed (slice order) and rounded to fp16 -
// as launch_splitk_reduce writes them - then the q and k heads rotated as
// rope_kernel does; the v heads only summed.  Items [0, n_rot): 8 rotation
// pairs of a q or k head; the rest: 8 consecutive values of a v head.
__global__ void reduce_rope_kernel(const float* __restrict__ parts, int n_parts, int64_t T,
                                   int seq, int H, int Hkv, int d,
                                   const float2* __restrict__ cs, uint16_t* __restrict__ qkv,
                                   int* dev_err) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int half = d / 2, chunks = half / 8;
  const int64_t ld = (int64_t)(H + 2 * Hkv) * d;
  const int64_t pstride = T * ld;
  const int64_t n_rot = T * (H + Hkv) * chunks;
  const int vq = Hkv * d / 8;  // 8-value groups of the v heads per token
  const int64_t n = n_rot + T * vq;
  auto sum8 = [&](int64_t e, float* f) {
    float4 a = *reinterpret_cast<const float4*>(parts + e);
    float4 b = *reinterpret_cast<const float4*>(parts + e + 4);
    for (int s = 1; s < n_parts; ++s) {
      const float4 pa = *reinterpret_cast<const float4*>(parts + (size_t)s * pstride + e);
      const float4 pb = *reinterpret_cast<const float4*>(parts + (size_t)s * pstride + e + 4);
      a.x += pa.x; a.y += pa.y; a.z += pa.z; a.w += pa.w;
      b.x += pb.x; b.y += pb.y; b.z += pb.z; b.w += pb.w;
    }
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  };
  bool big = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (i < n_rot) {
      const int ch = (int)(i % chunks);
      const int64_t th = i / chunks;
      const int head = (int)(th % (H + Hkv));
      const int64_t t = th / (H + Hkv);
      const int pos = (int)(t % seq);
      const int64_t e = t * ld + (int64_t)head * d + ch * 8;
      float f1[8], f2[8];
      sum8(e, f1);
      sum8(e + half, f2);
      const float2* c = cs + (int64_t)pos * half + ch * 8;
      uint32_t oa[4], ob[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        big |= !(fmaxf(fmaxf(fabsf(f1[2 * q]), fabsf(f1[2 * q + 1])),
                       fmaxf(fabsf(f2[2 * q]), fabsf(f2[2 * q + 1]))) <= kF16Max);
        const float2 x1 = unpack_f16x2(pack_f16x2(f1[2 * q], f1[2 * q + 1]));
        const float2 x2 = unpack_f16x2(pack_f16x2(f2[2 * q], f2[2 * q + 1]));
        const float2 c0 = c[2 * q], c1 = c[2 * q + 1];
        oa[q] = pack_f16x2(x1.x * c0.x - x2.x * c0.y, x1.y * c1.x - x2.y * c1.y);
        ob[q] = pack_f16x2(x2.x * c0.x + x1.x * c0.y, x2.y * c1.x + x1.y * c1.y);
      }
      *reinterpret_cast<uint4*>(qkv + e) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
      *reinterpret_cast<uint4*>(qkv + e + half) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    } else {
      const int64_t j = i - n_rot;
      const int64_t t = j / vq;
      const int64_t e = t * ld + (int64_t)(H + Hkv) * d + (j % vq) * 8;
      float f[8];
      sum8(e, f);
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        big |= !(fmaxf(fabsf(f[2 * q]), fabsf(f[2 * q + 1])) <= kF16Max);
        o[q] = pack_f16x2(f[2 * q], f[2 * q + 1]);
      }
      *reinterpret_cast<uint4*>(qkv + e) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (big) atomicOr(dev_err, DEV_ERR_NONFINITE);
}

// dqkv (bf16) <- [rope^-1(dq), rope^-1(dk), dv].  dq is fp32 [T, H d]; dk and dv
// arrive per query head (fp32 [T, H d]) and are summed over each kv head's
// H/Hkv query heads in a fixed order here.  A thread handles 4 pairs.
__global__ void rope_grad_kernel(const float* __restrict__ dq, const float* __restrict__ dk,
                                 const float* __restrict__ dv, int64_t T, int seq, int H, int Hkv,
                                 int d, const float2* __restrict__ cs,
                                 uint16_t* __restrict__ dqkv) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int half = d / 2, chunks = half / 4, rep = H / Hkv;
  const int64_t ld = (int64_t)(H + 2 * Hkv) * d;
  const int64_t hd = (int64_t)H * d;
  const int64_t n = T * (H + 2 * Hkv) * chunks;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int ch = (int)(i % chunks);
    const int64_t th = i / chunks;
    const int head = (int)(th % (H + 2 * Hkv));
    const int64_t t = th / (H + 2 * Hkv);
    uint16_t* out = dqkv + t * ld + (int64_t)head * d + ch * 4;
    float4 g1 = make_float4(0, 0, 0, 0), g2 = make_float4(0, 0, 0, 0);
    const float* src;
    int nsum;
    if (head < H) {
      src = dq + t * hd + (int64_t)head * d;
      nsum = 1;
    } else if (head < H + Hkv) {
      src = dk + t * hd + (int64_t)(head - H) * rep * d;
      nsum = rep;
    } else {
      src = dv + t * hd + (int64_t)(head - H - Hkv) * rep * d;
      nsum = rep;
    }
    for (int k = 0; k < nsum; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(src + (int64_t)k * d + ch * 4);
      const float4 b = *reinterpret_cast<const float4*>(src + (int64_t)k * d + half + ch * 4);
      g1.x += a.x; g1.y += a.y; g1.z += a.z; g1.w += a.w;
      g2.x += b.x; g2.y += b.y; g2.z += b.z; g2.w += b.w;
    }
    if (head >= H + Hkv) {
      *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(g1.x, g1.y), pack_bf16x2(g1.z, g1.w));
      *reinterpret_cast<uint2*>(out + half) =
          make_uint2(pack_bf16x2(g2.x, g2.y), pack_bf16x2(g2.z, g2.w));
      continue;
    }
    const int pos = (int)(t % seq);
    const float2* c = cs + (int64_t)pos * half + ch * 4;
    const float2 c0 = c[0], c1 = c[1], c2 = c[2], c3 = c[3];
    *reinterpret_cast<uint2*>(out) =
        make_uint2(pack_bf16x2(g1.x * c0.x + g2.x * c0.y, g1.y * c1.x + g2.y * c1.y),
                   pack_bf16x2(g1.z * c2.x + g2.z * c2.y, g1.w * c3.x + g2.w * c3.y));
    *reinterpret_cast<uint2*>(out + half) =
        make_uint2(pack_bf16x2(g2.x * c0.x - g1.x * c0.y, g2.y * c1.x - g1.y * c1.y),
                   pack_bf16x2(g2.z * c2.x - g1.z * c2.y, g2.w * c3.x - g1.w * c3.y));
  }
}

// ------------------------------------------------------------------ SwiGLU
__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + expf(-z)); }

// 8 elements per thread (F % 8 == 0); fp16 in and out (a product beyond the
// fp16 range latches the non-finite status bit)
__global__ void swiglu_fwd_kernel(const uint16_t* __restrict__ gu, int64_t T, int64_t F,
                                  uint16_t* __restrict__ m, int* dev_err) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t nv = T * F / 8;
  bool big = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 8;
    const int64_t t = e / F, f = e % F;
    const uint4 gv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + f);
    const uint4 uv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + F + f);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 g = unpack_f16x2(gw[q]), u = unpack_f16x2(uw[q]);
      const float m0 = g.x * sigmoidf_(g.x) * u.x, m1 = g.y * sigmoidf_(g.y) * u.y;
      big |= !(fmaxf(fabsf(m0), fabsf(m1)) <= kF16Max);
      o[q] = pack_f16x2(m0, m1);
    }
    *reinterpret_cast<uint4*>(m + e) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (big) atomicOr(dev_err, DEV_ERR_NONFINITE);
}

__global__ void swiglu_bwd_kernel(const float* __restrict__ dm, const uint16_t* __restrict__ gu,
                                  int64_t T, int64_t F, uint16_t* __restrict__ dgu) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t nv = T * F / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 8;
    const int64_t t = e / F, f = e % F;
    const uint4 gv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + f);
    const uint4 uv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + F + f);
    const float4 d0 = *reinterpret_cast<const float4*>(dm + e);
    const float4 d1 = *reinterpret_cast<const float4*>(dm + e + 4);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 g = unpack_f16x2(gw[q]), u = unpack_f16x2(uw[q]);
      const float s0 = sigmoidf_(g.x), s1 = sigmoidf_(g.y);
      const float a = dd[2 * q], b = dd[2 * q + 1];
      og[q] = pack_bf16x2(a * u.x * s0 * (1.f + g.x * (1.f - s0)),
                          b * u.y * s1 * (1.f + g.y * (1.f - s1)));
      ou[q] = pack_bf16x2(a * g.x * s0, b * g.y * s1);
    }
    *reinterpret_cast<uint4*>(dgu + t * 2 * F + f) = make_uint4(og[0], og[1], og[2], og[3]);
    *reinterpret_cast<uint4*>(dgu + t * 2 * F + F + f) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  }
}

// ------------------------------------------------------------------ embedding, CE, AdamW
__global__ void embedding_kernel(const int32_t* __restrict__ tok, int64_t T,
                                 const uint16_t* __restrict__ emb, int64_t D, int64_t V,
                                 float* __restrict__ out) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  const int64_t nv = D / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T * nv;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / nv, c = i % nv;
    int64_t id = tok[t];
    if (id < 0 || id >= V) id = 0;  // ids are validated on the host side where possible
    const uint4 v = reinterpret_cast<const uint4*>(emb + id * D)[c];
    const float2 a = unpack_bf16x2(v.x), b = unpack_bf16x2(v.y), e = unpack_bf16x2(v.z),
                 f = unpack_bf16x2(v.w);
    float4* o = reinterpret_cast<float4*>(out + t * D + c * 8);
    o[0] = make_float4(a.x, a.y, b.x, b.y);
    o[1] = make_float4(e.x, e.y, f.x, f.y);
  }
}

// One CTA (512 threads) per row.  Rows whose position is the last of its
// sequence have no target: zero gradient, zero loss.
// One CTA per row: row_loss = lse - logit[target] (= -log p(target)); and, when
// dlogits is given, dlogits = scale * (softmax - onehot(target)) in bf16, with
// scale = inv_count, or seq_scale[row / seq] when seq_scale is given (the DPO
// step's per-sequence coefficient).  The last position of each sequence has no
// target: zero loss and zero gradient.
// Online (max, sum of exp) pair of a set of values, and the union of two such
// pairs: the sum is kept relative to the running maximum and rescaled when that
// grows (an empty set is (-inf, 0)).
__device__ __forceinline__ void lse_merge(float& m, float& s, float mo, float so) {
  const float mn = fmaxf(m, mo);
  if (mn == -INFINITY) return;  // both empty
  s = s * expf(m - mn) + so * expf(mo - mn);
  m = mn;
}

// One CTA per row: row_loss = logsumexp(logits) - logits[target] (target = the
// next token; the last position of a sequence has none and gets 0), and with
// dlogits the gradient (softmax - onehot) * scale in bf16.  One read of the row
// for the (max, sum) pair, one more for the gradient; rows are read as float4
// (V is a multiple of 8).
__global__ void cross_entropy_kernel(const float* __restrict__ logits,
                                     const int32_t* __restrict__ tok, int64_t T, int seq,
                                     int64_t V, float inv_count,
                                     const float* __restrict__ seq_scale,
                                     uint16_t* __restrict__ dlogits,
                                     float* __restrict__ row_loss) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  __shared__ float red_m[32], red_s[32];
  __shared__ float bcast_m, bcast_s;
  const int64_t row = blockIdx.x;
  const float* lr = logits + row * V;
  uint16_t* dr = dlogits ? dlogits + row * V : nullptr;
  const bool has_target = (row % seq) != (seq - 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int64_t n4 = V / 4;
  if (!has_target) {
    if (dr)
      for (int64_t i = threadIdx.x; i < n4; i += blockDim.x)
        reinterpret_cast<uint2*>(dr)[i] = make_uint2(0u, 0u);
    if (threadIdx.x == 0) row_loss[row] = 0.f;
    return;
  }
  const float4* l4 = reinterpret_cast<const float4*>(lr);
  float m = -INFINITY, s = 0.f;
  for (int64_t i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = l4[i];
    const float mv = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
    if (mv > m) {
      s *= expf(m - mv);
      m = mv;
    }
    s += expf(v.x - m) + expf(v.y - m) + expf(v.z - m) + expf(v.w - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float mo = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    const float so = __shfl_xor_sync(0xFFFFFFFFu, s, o);
    lse_merge(m, s, mo, so);
  }
  if (lane == 0) {
    red_m[warp] = m;
    red_s[warp] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = red_m[0], bs = red_s[0];
    for (int w = 1; w < nw; ++w) lse_merge(bm, bs, red_m[w], red_s[w]);  // fixed order
    bcast_m = bm;
    bcast_s = bs;
  }
  __syncthreads();
  const float mx = bcast_m, sum = bcast_s;
  const float lse = mx + logf(sum);
  const int64_t tgt = tok[row + 1];
  if (dr) {
    const float inv = 1.f / sum;
    const float scale = seq_scale ? seq_scale[row / seq] : inv_count;
    for (int64_t i = threadIdx.x; i < n4; i += blockDim.x) {
      const float4 v = l4[i];
      float p[4] = {expf(v.x - mx) * inv, expf(v.y - mx) * inv, expf(v.z - mx) * inv,
                    expf(v.w - mx) * inv};
      const int64_t i0 = 4 * i;
      if (tgt >= i0 && tgt < i0 + 4) p[tgt - i0] -= 1.f;
      reinterpret_cast<uint2*>(dr)[i] =
          make_uint2(pack_bf16x2(p[0] * scale, p[1] * scale), pack_bf16x2(p[2] * scale, p[3] * scale));
    }
  }
  if (threadIdx.x == 0) row_loss[row] = lse - lr[tgt];
}

__global__ void sum_rows_kernel(const float* __restrict__ v, int64_t n, float scale,
                                int accumulate, float* __restrict__ out) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  __shared__ float red[32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += v[i];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) *out = (accumulate ? *out : 0.f) + scale * t;
  }
}

__global__ void adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                             float* __restrict__ m, float* __restrict__ v, int64_t n, float lr,
                             float b1, float b2, float eps, float wd, float bc1, float bc2) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float gi = g[i];
    const float mi = b1 * m[i] + (1.f - b1) * gi;
    const float vi = b2 * v[i] + (1.f - b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    const float mh = mi / bc1, vh = vi / bc2;
    p[i] = p[i] * (1.f - lr * wd) - lr * mh / (sqrtf(vh) + eps);
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, int64_t n,
                                   uint16_t* __restrict__ y) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    y[i] = float_to_bf16_bits(x[i]);
}

}  // namespace

int launch_splitk_reduce(const float* partial, int splits, int64_t T, int64_t M, void* out,
                         int out_kind, int64_t ldo, const float* residual, int64_t ldr,
                         cudaStream_t st) {
  if (M % 4 != 0) return set_error(LSQ_ERR_SHAPE, "splitk_reduce: M %% 4 != 0");
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  splitk_reduce_kernel<<<grid_for(T * M / 4, 256), 256, 0, st>>>(
      partial, splits, T, M, out, out_kind, ldo, residual, ldr, dev_err);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

int threads_for_row(int64_t D, int per) {
  int t = (int)std::min<int64_t>(256, (D / per + 31) / 32 * 32);
  return t < 32 ? 32 : t;
}

// The launchers below bracket their kernel with a profiler region (a no-op unless
// profiling is on) that carries the kernel's algorithmic DRAM bytes: every
// tensor it must read and write, once.
int launch_rmsnorm_fwd(const float* x, const uint16_t* g, int64_t T, int64_t D, float eps,
                       uint16_t* y, int y_kind, float* rstd, cudaStream_t st) {
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  const int prof = prof_begin(st);
  if (y_kind == OUT_F16)
    rmsnorm_fwd_kernel<true><<<(unsigned)T, threads_for_row(D, 8), 0, st>>>(x, g, D, eps, y, rstd,
                                                                           dev_err);
  else
    rmsnorm_fwd_kernel<false><<<(unsigned)T, threads_for_row(D, 8), 0, st>>>(x, g, D, eps, y, rstd,
                                                                            dev_err);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  if (prof >= 0) prof_end(prof, st, "rmsnorm_fwd", 0.0, 6.0 * T * D + 2.0 * D + 4.0 * T);
  return LSQ_OK;
}

int launch_rmsnorm_bwd(const float* dy, const float* x, const uint16_t* g, const float* rstd,
                       const float* dres, int64_t T, int64_t D, float* dx, uint16_t* dx_bf16,
                       cudaStream_t st) {
  const int prof = prof_begin(st);
  rmsnorm_bwd_kernel<<<(unsigned)T, threads_for_row(D, 4), 0, st>>>(dy, x, g, rstd, dres, D, dx,
                                                                   dx_bf16);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  if (prof >= 0)
    prof_end(prof, st, "rmsnorm_bwd", 0.0,
             (12.0 + (dres ? 4.0 : 0.0) + (dx_bf16 ? 2.0 : 0.0)) * T * D + 2.0 * D + 4.0 * T);
  return LSQ_OK;
}

int launch_rmsnorm_fwd_sum(const float* parts, int n_parts, const float* res, int64_t T,
                           int64_t D, float* x_out, const uint16_t* g, float eps, uint16_t* y,
                           int y_kind, float* rstd, cudaStream_t st) {
  if (n_parts < 1 || D % 8 != 0) return set_error(LSQ_ERR_SHAPE, "rmsnorm_fwd_sum: bad shape");
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  const size_t smem = (size_t)D * sizeof(float);
  if (smem > 48 * 1024) {
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr[dev]) {
      LSQ_CUDA(cudaFuncSetAttribute(rmsnorm_fwd_sum_kernel<true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
      LSQ_CUDA(cudaFuncSetAttribute(rmsnorm_fwd_sum_kernel<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
      attr[dev] = true;
    }
    if (smem > 200 * 1024) return set_error(LSQ_ERR_SHAPE, "rmsnorm_fwd_sum: row too long");
  }
  const int prof = prof_begin(st);
  const int64_t ps = T * D;
  if (y_kind == OUT_F16)
    rmsnorm_fwd_sum_kernel<true><<<(unsigned)T, threads_for_row(D, 8), smem, st>>>(
        parts, n_parts, ps, res, D, eps, g, x_out, y, rstd, dev_err);
  else
    rmsnorm_fwd_sum_kernel<false><<<(unsigned)T, threads_for_row(D, 8), smem, st>>>(
        parts, n_parts, ps, res, D, eps, g, x_out, y, rstd, dev_err);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  // the product's output read once (as if reduced), the residual, x_out and y written
  if (prof >= 0)
    prof_end(prof, st, "rmsnorm_fwd", 0.0,
             (4.0 + (res ? 4.0 : 0.0) + 4.0 + 2.0) * T * D + 2.0 * D + 4.0 * T);
  return LSQ_OK;
}

int launch_rmsnorm_bwd_sum(const float* parts, int n_parts, const float* x, const uint16_t* g,
                           const float* rstd, const float* dres, int64_t T, int64_t D, float* dx,
                           uint16_t* dx_bf16, cudaStream_t st) {
  if (n_parts < 1 || D % 4 != 0) return set_error(LSQ_ERR_SHAPE, "rmsnorm_bwd_sum: bad shape");
  const size_t smem = (size_t)D * sizeof(float);
  if (smem > 48 * 1024) {
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr[dev]) {
      LSQ_CUDA(cudaFuncSetAttribute(rmsnorm_bwd_sum_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
      attr[dev] = true;
    }
    if (smem > 200 * 1024) return set_error(LSQ_ERR_SHAPE, "rmsnorm_bwd_sum: row too long");
  }
  const int prof = prof_begin(st);
  rmsnorm_bwd_sum_kernel<<<(unsigned)T, threads_for_row(D, 4), smem, st>>>(
      parts, n_parts, T * D, x, g, rstd, dres, D, dx, dx_bf16);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  if (prof >= 0)
    prof_end(prof, st, "rmsnorm_bwd", 0.0,
             (12.0 + (dres ? 4.0 : 0.0) + (dx_bf16 ? 2.0 : 0.0)) * T * D + 2.0 * D + 4.0 * T);
  return LSQ_OK;
}

int launch_reduce_rope(const float* parts, int n_parts, int64_t T, int seq, int H, int Hkv, int d,
                       const float2* cs, uint16_t* qkv, cudaStream_t st) {
  if (n_parts < 1 || d % 16 != 0) return set_error(LSQ_ERR_SHAPE, "reduce_rope: bad shape");
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  const int64_t n = T * (H + Hkv) * (d / 16) + T * Hkv * (d / 8);
  const int prof = prof_begin(st);
  reduce_rope_kernel<<<grid_for(n, 256), 256, 0, st>>>(parts, n_parts, T, seq, H, Hkv, d, cs, qkv,
                                                       dev_err);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  // the product's output read once (fp32, as if reduced), q|k|v written (fp16), the table
  if (prof >= 0)
    prof_end(prof, st, "rope", 0.0, 6.0 * T * (H + 2 * Hkv) * d + 4.0 * seq * d);
  return LSQ_OK;
}

int launch_rope_table(int seq, int d, float theta, float2* cs, cudaStream_t st) {
  const int n = seq * (d / 2);
  rope_table_kernel<<<(unsigned)std::max(1, std::min(1024, (n + 255) / 256)), 256, 0, st>>>(
      seq, d / 2, d, log((double)theta), cs);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

int launch_rope(uint16_t* qkv, int64_t T, int seq, int H, int Hkv, int d, const float2* cs,
                cudaStream_t st) {
  const int64_t n = T * (H + Hkv) * (d / 16);
  const int prof = prof_begin(st);
  rope_kernel<<<grid_for(n, 256), 256, 0, st>>>(qkv, T, seq, H, Hkv, d, cs);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  // q and k read and written in place (fp16), plus the table rows once
  if (prof >= 0) prof_end(prof, st, "rope", 0.0, 4.0 * T * (H + Hkv) * d + 4.0 * seq * d);
  return LSQ_OK;
}

int launch_rope_grad(const float* dq, const float* dk, const float* dv, int64_t T, int seq, int H,
                     int Hkv, int d, const float2* cs, uint16_t* dqkv, cudaStream_t st) {
  const int64_t n = T * (H + 2 * Hkv) * (d / 8);
  const int prof = prof_begin(st);
  rope_grad_kernel<<<grid_for(n, 256), 256, 0, st>>>(dq, dk, dv, T, seq, H, Hkv, d, cs, dqkv);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  // fp32 dq, dk, dv per query head in; bf16 dq|dk|dv out
  if (prof >= 0)
    prof_end(prof, st, "rope_grad", 0.0, 12.0 * T * H * d + 2.0 * T * (H + 2 * Hkv) * d);
  return LSQ_OK;
}

int launch_swiglu_fwd(const uint16_t* gu, int64_t T, int64_t F, uint16_t* m, cudaStream_t st) {
  int* dev_err = device_status_ptr();
  if (!dev_err) return set_error(LSQ_ERR_CUDA, "device status word unavailable");
  const int prof = prof_begin(st);
  swiglu_fwd_kernel<<<grid_for(T * F / 8, 256), 256, 0, st>>>(gu, T, F, m, dev_err);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  if (prof >= 0) prof_end(prof, st, "swiglu_fwd", 0.0, 6.0 * T * F);
  return LSQ_OK;
}

int launch_swiglu_bwd(const float* dm, const uint16_t* gu, int64_t T, int64_t F, uint16_t* dgu,
                      cudaStream_t st) {
  const int prof = prof_begin(st);
  swiglu_bwd_kernel<<<grid_for(T * F / 8, 256), 256, 0, st>>>(dm, gu, T, F, dgu);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  if (prof >= 0) prof_end(prof, st, "swiglu_bwd", 0.0, 12.0 * T * F);
  return LSQ_OK;
}

int launch_embedding(const int32_t* tokens, int64_t T, const uint16_t* emb, int64_t D, int64_t V,
                     float* out, cudaStream_t st) {
  const int prof = prof_begin(st);
  embedding_kernel<<<grid_for(T * D / 8, 256), 256, 0, st>>>(tokens, T, emb, D, V, out);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  if (prof >= 0) prof_end(prof, st, "embedding", 0.0, 6.0 * T * D + 4.0 * T);
  return LSQ_OK;
}

int launch_cross_entropy(const float* logits, const int32_t* tokens, int64_t T, int seq, int64_t V,
                         float inv_count, uint16_t* dlogits, float* row_loss, cudaStream_t st,
                         const float* seq_scale) {
  const int prof = prof_begin(st);
  cross_entropy_kernel<<<(unsigned)T, 512, 0, st>>>(logits, tokens, T, seq, V, inv_count, seq_scale,
                                                    dlogits, row_loss);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  // fp32 logits read once, bf16 dlogits written once (when asked for)
  if (prof >= 0)
    prof_end(prof, st, "cross_entropy", 0.0, (4.0 + (dlogits ? 2.0 : 0.0)) * T * V + 8.0 * T);
  return LSQ_OK;
}

// DPO loss of P pairs from the per-row losses (-log p) of the policy and the
// reference (rows: sequence q = 2 p + {0 chosen, 1 rejected}, seq positions
// each).  One CTA: each sequence's log-probability is summed in a fixed order
// (fp64), then z_p = beta ((lp_c - lr_c) - (lp_r - lr_r)), loss = mean
// softplus(-z_p); seq_scale gets -dloss/dlp per sequence (the scale of
// softmax - onehot in dlogits); logps gets (lp_c, lp_r, lr_c, lr_r) per pair.
__global__ void dpo_loss_kernel(const float* __restrict__ row_pol,
                                const float* __restrict__ row_ref, int pairs, int seq, float beta,
                                float* __restrict__ seq_scale, float* __restrict__ logps,
                                float* __restrict__ loss_out) {
  pdl_trigger();  // the next kernel may launch once all CTAs of this one run
  __shared__ double red[2][32];
  __shared__ double lp[2][64];  // [pol/ref][sequence], pairs <= 32
  const int nseq = 2 * pairs;
  for (int q = 0; q < nseq; ++q) {
    double a = 0.0, b = 0.0;
    for (int t = threadIdx.x; t < seq - 1; t += blockDim.x) {
      a += (double)row_pol[(int64_t)q * seq + t];
      b += (double)row_ref[(int64_t)q * seq + t];
    }
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
      b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
    }
    if ((threadIdx.x & 31) == 0) {
      red[0][threadIdx.x >> 5] = a;
      red[1][threadIdx.x >> 5] = b;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double sa = 0.0, sb = 0.0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        sa += red[0][w];
        sb += red[1][w];
      }
      lp[0][q] = -sa;
      lp[1][q] = -sb;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    double loss = 0.0;
    for (int p = 0; p < pairs; ++p) {
      const double z = (double)beta * ((lp[0][2 * p] - lp[1][2 * p]) - (lp[0][2 * p + 1] - lp[1][2 * p + 1]));
      loss += fmax(-z, 0.0) + log1p(exp(-fabs(z)));
      const double sig_neg = 1.0 / (1.0 + exp(z));
      seq_scale[2 * p] = (float)((double)beta * sig_neg / pairs);
      seq_scale[2 * p + 1] = (float)(-(double)beta * sig_neg / pairs);
      logps[4 * p + 0] = (float)lp[0][2 * p];
      logps[4 * p + 1] = (float)lp[0][2 * p + 1];
      logps[4 * p + 2] = (float)lp[1][2 * p];
      logps[4 * p + 3] = (float)lp[1][2 * p + 1];
    }
    loss_out[0] = (float)(loss / pairs);
  }
}

int launch_dpo_loss(const float* row_pol, const float* row_ref, int pairs, int seq, float beta,
                    float* seq_scale, float* logps, float* loss_out, cudaStream_t st) {
  if (pairs <= 0 || pairs > 32) return set_error(LSQ_ERR_SHAPE, "dpo: 1..32 pairs per step");
  dpo_loss_kernel<<<1, 256, 0, st>>>(row_pol, row_ref, pairs, seq, beta, seq_scale, logps,
                                     loss_out);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

int launch_sum_rows(const float* row_loss, int64_t T, float scale, int accumulate, float* out,
                    cudaStream_t st) {
  sum_rows_kernel<<<1, 1024, 0, st>>>(row_loss, T, scale, accumulate, out);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

int launch_adamw(float* p, const float* g, float* m, float* v, int64_t n, float lr, float b1,
                 float b2, float eps, float wd, int step, cudaStream_t st) {
  const float bc1 = (float)(1.0 - pow((double)b1, (double)step));
  const float bc2 = (float)(1.0 - pow((double)b2, (double)step));
  const int prof = prof_begin(st);
  adamw_kernel<<<grid_for(n, 256), 256, 0, st>>>(p, g, m, v, n, lr, b1, b2, eps, wd, bc1, bc2);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  // p, g, m, v read; p, m, v written (fp32)
  if (prof >= 0) prof_end(prof, st, "adamw", 0.0, 28.0 * n);
  return LSQ_OK;
}

int launch_f32_to_bf16(const float* x, int64_t n, uint16_t* y, cudaStream_t st) {
  f32_to_bf16_kernel<<<grid_for(n, 256), 256, 0, st>>>(x, n, y);
  LSQ_CUDA(::lsq::launched(cudaGetLastError()));
  return LSQ_OK;
}

}  // namespace lsq

extern "C" int lsq_bf16_from_f32(const float* x, int64_t n, uint16_t* y, void* stream) {
  using namespace lsq;
  if (n <= 0) return set_error(LSQ_ERR_SHAPE, "lsq_bf16_from_f32: n must be positive");
  if (!x || !y) return set_error(LSQ_ERR_INVALID, "lsq_bf16_from_f32: null pointer");
  return launch_f32_to_bf16(x, n, y, static_cast<cudaStream_t>(stream));
}

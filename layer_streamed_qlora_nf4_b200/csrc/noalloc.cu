// Allocation-free variant of the fused NF4 + LoRA linear forward.
//
// Some callers cannot hand the library a device workspace: for example a host
// framework that has already reserved all device memory for its own pool and
// gives plugins no allocator, or a latency-critical caller that cannot afford
// the device-wide synchronisation cudaMalloc / cudaFree may cause.  For them,
// nf4_lora_linear_fwd_noalloc runs exactly the kernels of nf4_lora_linear_fwd
// but takes its scratch (the x A^T product, the fixed-order split partials of
// the rank-r product and of the split-K GEMM) from a file-scope device array of
// kNoAllocScratchBytes.  It calls no allocating routine.
//
// Host code must not use the array's name as a device address (on the host it
// only names a stand-in); the device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on it.
// Under CUDA's lazy module loading (the default since CUDA 12.2) this file's
// module, and with it the 32 MiB array, is loaded onto a device by that first
// lookup: the first call on a device reserves the array's device memory (and
// can fail if the device is full); every later call allocates nothing.  The
// array then stays on the device until the process exits.
#include <mutex>

#include "common.cuh"

namespace lsq {

namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;  // 32 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (looked up once).
int noalloc_scratch(void** out) {
  int dev = -1;
  LSQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return set_error(LSQ_ERR_INVALID, "noalloc: unsupported device index");
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_error(LSQ_ERR_CUDA, "noalloc: cudaGetSymbolAddress failed: %s",
                       cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return LSQ_OK;
}

}  // namespace
}  // namespace lsq

using namespace lsq;

extern "C" int nf4_lora_linear_fwd_noalloc(const uint16_t* x, int64_t T, int64_t K, int64_t N,
                                           const uint8_t* codes, const float* absmax,
                                           int32_t block, const float* A, const float* B,
                                           int32_t r, float scale, const float* residual,
                                           void* y, int32_t y_fp32, float* u_out, void* stream) {
  const size_t need = nf4_lora_linear_workspace_bytes(T, K, N, r);
  if (need == 0)
    return set_error(LSQ_ERR_SHAPE, "nf4_lora_linear_fwd_noalloc: empty or invalid shape");
  if (need > kNoAllocScratchBytes)
    return set_error(LSQ_ERR_WORKSPACE,
                     "nf4_lora_linear_fwd_noalloc: these sizes need %zu bytes of scratch, more "
                     "than the built-in %zu (use nf4_lora_linear_fwd with a caller workspace)",
                     need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  LSQ_TRY(noalloc_scratch(&scratch));
  // Nothing in the scratch needs to start at zero: every byte the kernels read
  // is written earlier in the same call.
  return nf4_lora_linear_fwd(x, T, K, N, codes, absmax, block, A, B, r, scale, residual, y,
                             y_fp32, u_out, scratch, kNoAllocScratchBytes, stream);
}

// Projection GEMM for callers that cannot allocate device memory.
//
// dory_gemm_bf16 leaves split-K partial slices in a caller buffer of 8 * M * N
// floats and lets the caller add them.  Some callers cannot provide that
// buffer: code running while a CUDA graph is being recorded (where cudaMalloc
// is not allowed), servers whose device memory is one pre-sized arena owned by
// another component, or real-time paths that forbid allocation after start-up.
// dory_gemm_bf16_noalloc keeps the partial slices in a fixed array compiled
// into this library instead, and returns the finished product in Y.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoAllocScratchFloats floats (8 MiB) until the process exits.
// All calls share it, so two calls whose kernels overlap on the GPU (different
// streams, or different host threads) overwrite each other's partial sums;
// serialise such calls.  Each call writes every partial value it later reads,
// so nothing in the array has to start at zero.
#include <cuda_runtime.h>

#include <mutex>

#include "dory.h"
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace dory {
void set_last_error(const char* msg);
}

namespace {

constexpr size_t kNoAllocScratchFloats = size_t(2) << 20;  // 8 MiB of fp32 partial sums

__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_addr[kMaxDevices] = {};

dory_status noalloc_fail(dory_status s, const char* msg) {
  dory::set_last_error(msg);
  return s;
}

}  // namespace

extern "C" dory_status dory_gemm_bf16_noalloc(int32_t M, int32_t N, int32_t K, const void* X, const void* W,
                                              float* Y, int32_t batch_hint, dory_stream stream) {
  if (M < 1 || N < 1 || K < 1 || !X || !W || !Y)
    return noalloc_fail(DORY_ERR_INVALID_ARG, "dory_gemm_bf16_noalloc: bad sizes or NULL pointer");
  if ((size_t)dory::kMaxSplitK * (size_t)M * (size_t)N > kNoAllocScratchFloats)
    return noalloc_fail(DORY_ERR_CAPACITY,
                        "dory_gemm_bf16_noalloc: 8 * M * N must not exceed 2097152 (the 8 MiB built-in scratch)");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return noalloc_fail(DORY_ERR_CUDA, "dory_gemm_bf16_noalloc: no usable current device");
  float* scratch = nullptr;
  {
    // The host-side name of the array is not a device address; look up the
    // device address once per device, with that device current.
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return noalloc_fail(DORY_ERR_CUDA, "dory_gemm_bf16_noalloc: cudaGetSymbolAddress failed");
      g_scratch_addr[dev] = (float*)p;
    }
    scratch = g_scratch_addr[dev];
  }
  cudaStream_t st = (cudaStream_t)stream;
  int S = 1;
  size_t ps = 0;
  cudaError_t e = dory::launch_gemm_tc(M, N, K, (const dory::bf16*)X, K, (const dory::bf16*)W, scratch, N, (size_t)M,
                                       nullptr, batch_hint < 1 ? 1 : batch_hint, true, &S, &ps, st);
  if (e == cudaErrorNotSupported)
    return noalloc_fail(DORY_ERR_UNSUPPORTED,
                        "dory_gemm_bf16_noalloc: needs N % 128 == 0, K % 64 == 0 and 16-byte aligned X, W");
  if (e != cudaSuccess) return noalloc_fail(DORY_ERR_CUDA, cudaGetErrorString(e));
  e = dory::launch_split_reduce(M, N, scratch, S, ps, Y, st);
  if (e != cudaSuccess) return noalloc_fail(DORY_ERR_CUDA, cudaGetErrorString(e));
  return DORY_OK;
}

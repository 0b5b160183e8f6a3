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
//
// A second file-scope word records a bounded wait of the GEMM that gave up
// (its partial sums are then incomplete).  The reduction writes NaN into Y
// for every call made while the word is set, and
// dory_gemm_bf16_noalloc_status() reads and clears it.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "dory.h"
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace dory {
void set_last_error(const char* msg);
}

namespace {

dory_status noalloc_fail(dory_status s, const char* msg) {
  dory::set_last_error(msg);
  return s;
}

constexpr size_t kNoAllocScratchFloats = size_t(2) << 20;  // 8 MiB of fp32 partial sums

__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];
__device__ int g_noalloc_err = 0;  // DEV_ERR_* of a GEMM wait that gave up; 0 while none did

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_addr[kMaxDevices] = {};
int* g_err_addr[kMaxDevices] = {};

// Y = in-order sum of the S partial slices, or NaN everywhere once a GEMM
// wait has given up (the slices may then hold another call's values).
__global__ void k_noalloc_reduce(size_t total, const float* __restrict__ part, int S, size_t ps, float* out,
                                 const int* err) {
  const bool bad = *(volatile const int*)err != 0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < S; ++s) a += part[s * ps + i];
    out[i] = bad ? __int_as_float(0x7fc00000) : a;
  }
}

// Device addresses of the scratch array and the error word on the current
// device (looked up once per device, with that device current).
dory_status addresses(float** scratch, int** err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return noalloc_fail(DORY_ERR_CUDA, "dory_gemm_bf16_noalloc: no usable current device");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    // The host-side names of the arrays are not device addresses.
    void* p = nullptr;
    void* q = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&q, g_noalloc_err);
    if (e != cudaSuccess || !p || !q)
      return noalloc_fail(DORY_ERR_CUDA, "dory_gemm_bf16_noalloc: cudaGetSymbolAddress failed");
    g_err_addr[dev] = (int*)q;
    g_scratch_addr[dev] = (float*)p;
  }
  *scratch = g_scratch_addr[dev];
  *err = g_err_addr[dev];
  return DORY_OK;
}


}  // namespace

extern "C" dory_status dory_gemm_bf16_noalloc(int32_t M, int32_t N, int32_t K, const void* X, const void* W,
                                              float* Y, int32_t batch_hint, dory_stream stream) {
  if (M < 1 || N < 1 || K < 1 || !X || !W || !Y)
    return noalloc_fail(DORY_ERR_INVALID_ARG, "dory_gemm_bf16_noalloc: bad sizes or NULL pointer");
  if ((size_t)dory::kMaxSplitK * (size_t)M * (size_t)N > kNoAllocScratchFloats)
    return noalloc_fail(DORY_ERR_CAPACITY,
                        "dory_gemm_bf16_noalloc: 8 * M * N must not exceed 2097152 (the 8 MiB built-in scratch)");
  float* scratch = nullptr;
  int* err = nullptr;
  {
    const dory_status r = addresses(&scratch, &err);
    if (r != DORY_OK) return r;
  }
  cudaStream_t st = (cudaStream_t)stream;
  int S = 1;
  size_t ps = 0;
  cudaError_t e = dory::launch_gemm_tc(M, N, K, (const dory::bf16*)X, K, (const dory::bf16*)W, scratch, N, (size_t)M,
                                       err, batch_hint < 1 ? 1 : batch_hint, true, &S, &ps, st);
  if (e == cudaErrorNotSupported)
    return noalloc_fail(DORY_ERR_UNSUPPORTED,
                        "dory_gemm_bf16_noalloc: needs N % 128 == 0, K % 64 == 0 and 16-byte aligned X, W");
  if (e != cudaSuccess) return noalloc_fail(DORY_ERR_CUDA, cudaGetErrorString(e));
  const size_t total = (size_t)M * N;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
  k_noalloc_reduce<<<blocks, 256, 0, st>>>(total, scratch, S, ps, Y, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return noalloc_fail(DORY_ERR_CUDA, cudaGetErrorString(e));
  return DORY_OK;
}

extern "C" dory_status dory_gemm_bf16_noalloc_status(dory_stream stream) {
  float* scratch = nullptr;
  int* err = nullptr;
  {
    const dory_status r = addresses(&scratch, &err);
    if (r != DORY_OK) return r;
  }
  cudaStream_t st = (cudaStream_t)stream;
  int word = 0;
  const int zero = 0;
  cudaError_t e = cudaMemcpyAsync(&word, err, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && word != 0) {
    e = cudaMemcpyAsync(err, &zero, sizeof(int), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  if (e != cudaSuccess) return noalloc_fail(DORY_ERR_CUDA, cudaGetErrorString(e));
  if (word == dory::DEV_ERR_TIMEOUT)
    return noalloc_fail(DORY_ERR_TIMEOUT, "dory_gemm_bf16_noalloc: a GEMM wait gave up; Y of the calls since "
                                          "the last status check holds NaN");
  if (word != 0) return noalloc_fail(DORY_ERR_CUDA, "dory_gemm_bf16_noalloc: device error word set");
  return DORY_OK;
}

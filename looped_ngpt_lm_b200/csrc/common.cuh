// Shared device helpers for the looped nGPT kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dory {

typedef __nv_bfloat16 bf16;

// Device error word codes (the host reads them in dory_synchronize).
enum : int {
  DEV_ERR_NONE = 0,
  DEV_ERR_TIMEOUT = 1,   // a bounded wait gave up
  DEV_ERR_BAD_TOKEN = 2, // token id outside [0, vocab)
  DEV_ERR_BAD_INDEX = 3, // a cache index check failed
  DEV_ERR_RANGE = 4      // a value outside a kernel's supported range (non-finite weight, |x| >= 2^64)
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum with a fixed reduction order (per-thread value -> xor tree in
// each warp -> warps added in index order).  Every thread gets the result.
// red must hold 33 floats.  blockDim.x must be a multiple of 32.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    red[32] = t;
  }
  __syncthreads();
  float r = red[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ void set_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

}  // namespace dory

namespace dory {

// Programmatic dependent launch.  Every kernel of the forward is launched
// with programmatic stream serialization allowed, so it may start while its
// predecessor in the stream is still running.  pdl_wait() blocks until the
// predecessor grid has completed and its memory is visible; a kernel calls it
// before touching anything an earlier kernel writes or reads.  pdl_trigger()
// lets the next kernel in the stream start early (it still waits in its own
// pdl_wait()).  Both are no-ops for a kernel launched without the attribute.
//
// Ordering invariant.  The decode attention reads the row metadata (and the
// cache) before its pdl_wait().  Kernels that wait before they trigger
// guarantee that everything two launches back has completed when a kernel
// launches; the kernels that open a pass (planning, embedding, stash copies,
// loop re-injection) keep that order, so no attention launches before the
// planning kernel of its pass has finished.  The add + norm and SwiGLU
// kernels between two projection GEMMs trigger first instead: the GEMM that
// follows is then scheduled while the GEMM before them drains and takes each
// SM as soon as that GEMM's block there exits (a dependent grid launches only
// once every block of this grid has started, so this cannot starve it).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Host switch for programmatic launches (tests can turn it off).
extern bool g_pdl;

template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace dory

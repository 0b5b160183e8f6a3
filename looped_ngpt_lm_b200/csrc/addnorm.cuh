// The nGPT layer update h <- N(h + sum_s y_s) of one row, shared by the
// standalone kernel (k_addnorm) and the operand stage of the decode GEMM, so
// both produce the same bits whichever of them runs (a decode row and the
// same row inside a longer speculative chunk must agree exactly).
//
// The row is handled by 128 threads.  Thread t owns the float4 chunks
// t, t + 128, ... of the row.  The S split-K slices of y are added in order
// to a sum that starts at zero, then h is added.  Each thread sums the
// squares of its chunks (x, y, z, w, chunk by chunk, with explicit FMAs), the
// warps reduce by xor trees and the four warp sums are added in index order.
// N(v) = v / max(||v||_2, 1e-12).
#pragma once

#include "common.cuh"

namespace dory {

constexpr int AN_THREADS = 128;  // threads per row
constexpr int AN_MAXC = 8;       // float4 chunks per thread: d <= 4096
constexpr int AN_MAXS = 8;       // split-K slices

// Chunk c of v = h + sum_{s<S} y_s for one row (y_s = y + s * ps).
__device__ __forceinline__ float4 an_chunk(const float* h, const float* y, int S, size_t ps, int c) {
  float4 p[AN_MAXS];
#pragma unroll
  for (int s = 0; s < AN_MAXS; ++s)
    p[s] = s < S ? __ldcg(reinterpret_cast<const float4*>(y + s * ps) + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 hv = __ldcg(reinterpret_cast<const float4*>(h) + c);
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < AN_MAXS; ++s)
    if (s < S) {
      a.x += p[s].x;
      a.y += p[s].y;
      a.z += p[s].z;
      a.w += p[s].w;
    }
  return make_float4(hv.x + a.x, hv.y + a.y, hv.z + a.z, hv.w + a.w);
}

__device__ __forceinline__ float an_squares(float ss, float4 v) {
  ss = __fmaf_rn(v.x, v.x, ss);
  ss = __fmaf_rn(v.y, v.y, ss);
  ss = __fmaf_rn(v.z, v.z, ss);
  return __fmaf_rn(v.w, v.w, ss);
}

// 1 / max(||v||, 1e-12) from the 128 threads' partial sums of squares; t is
// the thread's index among the 128, red holds 4 floats, sync() is a barrier
// over exactly those 128 threads.
template <typename Sync>
__device__ __forceinline__ float an_inv_norm(float ss, float* red, int t, Sync sync) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((t & 31) == 0) red[t >> 5] = ss;
  sync();
  const float tot = ((red[0] + red[1]) + red[2]) + red[3];
  sync();  // red may be written again
  return 1.f / fmaxf(sqrtf(tot), 1e-12f);
}

__device__ __forceinline__ float4 an_scale(float4 v, float inv) {
  return make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
}

}  // namespace dory

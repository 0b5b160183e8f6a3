// The nGPT layer update h <- N(h + sum_s y_s) of one row, shared by the
// standalone kernel (k_addnorm) and the operand stage of the decode GEMM, so
// both produce the same bits whichever of them runs (a decode row and the
// same row inside a longer speculative chunk must agree exactly).
//
// The arithmetic is defined over 512 virtual threads: virtual thread v owns
// elements v, v + 512, ... of the row.  Each element is h plus the S split-K
// slices of y added in order to a sum that starts at zero.  A virtual thread
// sums the squares of its elements in order with explicit FMAs; each virtual
// warp (32 consecutive virtual threads) reduces by an xor tree; the 16 warp
// sums are added in index order.  N(v) = v / max(||v||_2, 1e-12).  The
// standalone kernel runs one real thread per virtual thread (many warps hide
// the latency of the loads); the operand stage's 128 threads run four each.
#pragma once

#include "common.cuh"

namespace dory {

constexpr int AN_VT = 512;   // virtual threads per row
constexpr int AN_CPT = 8;    // elements per virtual thread: d <= 4096
constexpr int AN_MAXS = 8;   // split-K slices

// Element i of v = h + sum_{s<S} y_s for one row (y_s = y + s * ps).
__device__ __forceinline__ float an_elem(const float* h, const float* y, int S, size_t ps, int i) {
  float p[AN_MAXS];
#pragma unroll
  for (int s = 0; s < AN_MAXS; ++s) p[s] = s < S ? __ldcg(y + s * ps + i) : 0.f;
  const float hv = __ldcg(h + i);
  float a = 0.f;
#pragma unroll
  for (int s = 0; s < AN_MAXS; ++s)
    if (s < S) a += p[s];
  return hv + a;
}

// A virtual thread's elements and the sum of their squares.
__device__ __forceinline__ float an_load(const float* h, const float* y, int S, size_t ps, int d, int v,
                                         float (&e)[AN_CPT]) {
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < AN_CPT; ++c) {
    const int i = v + c * AN_VT;
    e[c] = 0.f;
    if (i < d) {
      e[c] = an_elem(h, y, S, ps, i);
      ss = __fmaf_rn(e[c], e[c], ss);
    }
  }
  return ss;
}

__device__ __forceinline__ float an_warp_tree(float ss) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  return ss;
}

// 1 / max(||v||, 1e-12) from the 16 virtual-warp sums (in index order).
__device__ __forceinline__ float an_inv_from_warps(const float* red16) {
  float t = red16[0];
#pragma unroll
  for (int w = 1; w < AN_VT / 32; ++w) t += red16[w];
  return 1.f / fmaxf(sqrtf(t), 1e-12f);
}

}  // namespace dory

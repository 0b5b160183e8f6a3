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

// A virtual thread's elements (element i of v = h + sum_{s<S} y_s, with
// y_s = y + s * ps) and the sum of their squares.  Every load of every
// element is issued before the first one is used (elements past d read
// element 0 and are dropped), so a row costs one round trip to L2.
__device__ __forceinline__ float an_load(const float* h, const float* y, int S, size_t ps, int d, int v,
                                         float (&e)[AN_CPT]) {
  float p[AN_CPT][AN_MAXS], hv[AN_CPT];
#pragma unroll
  for (int c = 0; c < AN_CPT; ++c) {
    const bool live = c * AN_VT < d;  // the same for every thread of the row
    const int i = v + c * AN_VT < d ? v + c * AN_VT : 0;
    hv[c] = live ? __ldcg(h + i) : 0.f;
#pragma unroll
    for (int s = 0; s < AN_MAXS; ++s) p[c][s] = live && s < S ? __ldcg(y + s * ps + i) : 0.f;
  }
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < AN_CPT; ++c) {
    float a = 0.f;
#pragma unroll
    for (int s = 0; s < AN_MAXS; ++s)
      if (s < S) a += p[c][s];
    e[c] = 0.f;
    if (v + c * AN_VT < d) {
      e[c] = hv[c] + a;
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

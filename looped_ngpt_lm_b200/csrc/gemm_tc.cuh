// bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM, TMA-fed).
#pragma once

#include "common.cuh"

namespace dory {

// Largest split-K factor the GEMM may choose; callers size partial buffers
// for kMaxSplitK slices.
constexpr int kMaxSplitK = 8;

// Weight stream of one forward pass: the weight matrices in the order the
// pass's GEMMs read them, each at a byte offset of one concatenated stream.
struct PfSeg {
  const char* p;
  unsigned long long off, bytes;
};

// L2 look-ahead of one GEMM launch: the byte range [lo, hi) of the stream,
// past this GEMM's own weights, that its CTAs prefetch into L2 once their
// own loads have landed (CTA b takes the b-th of gridDim.x equal pieces).
// The following attention, norms and the next GEMM's ramp-up then overlap
// HBM reads of the weights that come next.  lo >= hi: off.
struct PfCtl {
  const PfSeg* segs = nullptr;
  int nseg = 0;
  int first = 0;  // a segment at or before the one holding lo
  unsigned long long lo = 0, hi = 0;
};

// Y = X . W^T for X [M, K] (row stride ldx) and W [N, K], both bf16, fp32
// accumulation.  Writes S partial products to Y + s * (*part_stride)
// (row stride ldy); the consumer adds them in order s = 0..S-1.
// invariant: 16-token MMA groups and a split chosen from (N, K, batch) only,
// so each row's result is bit-identical for every M; otherwise 128 x 256
// tiles without split.  part_rows: rows available per
// slice (>= M).  Returns cudaErrorNotSupported for shapes the kernel does not
// handle (N % 128, K % 64, unaligned pointers).  variant 1 forces one
// 64-column sub-tile per pipeline stage (for comparisons).
// packed: W is in the packed tile layout below.  pf: L2 look-ahead (decode
// tiles only; ignored for prefill tiles).
cudaError_t launch_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const bf16* W, float* Y, int ldy,
                           size_t part_rows, int* err, int batch, bool invariant, int* S, size_t* part_stride,
                           cudaStream_t st, int variant = 0, bool packed = false, const PfCtl* pf = nullptr);

// act[m, j] = silu(g) * u (bf16, row stride dff) with g = X[m] . Wgu[j] and
// u = X[m] . Wgu[dff + j] for the concatenated [gate; up] weight Wgu
// [2 dff, K]: the gate-up projection and SwiGLU of a long chunk in one
// tensor-core GEMM (fp32 accumulation, no split).  dff % 128 == 0.
cudaError_t launch_gemm_glu(int M, int dff, int K, const bf16* X, int ldx, const bf16* Wgu, bf16* act,
                            int* err, cudaStream_t st);

// Repack a row-major [N, K] bf16 weight (N % 128 == 0, K % 64 == 0) into the
// packed tile layout the tensor-core GEMM streams with bulk copies: 128 x 64
// tiles, each stored as its 16 KB 128-byte-swizzled shared-memory image
// (row r's 16-byte chunk c at r*128 + (c ^ (r % 8))*16), tile (n, k) at
// ((n * K/64) + k) * 16 KB.  dst holds N*K*2 bytes.
cudaError_t launch_pack_weight(const bf16* W, void* dst, int N, int K, cudaStream_t st);

}  // namespace dory

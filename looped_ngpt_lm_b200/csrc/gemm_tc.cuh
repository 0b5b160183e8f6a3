// bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM, TMA-fed).
#pragma once

#include "common.cuh"

namespace dory {

// Largest split-K factor the GEMM may choose; callers size partial buffers
// for kMaxSplitK slices.
constexpr int kMaxSplitK = 8;
// Device counters a split GEMM needs (one per output tile; zero between
// launches, and left zero by every launch).
constexpr int kTileCounters = 4096;

// Y = X . W^T for X [M, K] (row stride ldx) and W [N, K], both bf16, fp32
// accumulation.  Writes S partial products to Y + s * (*part_stride)
// (row stride ldy); the consumer adds them in order s = 0..S-1.
// invariant: 16-token MMA groups and a split chosen from (N, K, batch) only,
// so each row's result is bit-identical for every M; otherwise 128 x 256
// tiles without split.  part_rows: rows available per
// slice (>= M).  Returns cudaErrorNotSupported for shapes the kernel does not
// handle (N % 128, K % 64, unaligned pointers).  variant 1 forces one
// 64-column sub-tile per pipeline stage (for comparisons).  With
// tile_counters (kTileCounters zeros), the last split of each output tile
// adds the slices in order s = 0..S-1 inside the kernel and *S is 1.
// packed: W is in the packed tile layout below.
cudaError_t launch_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const bf16* W, float* Y, int ldy,
                           size_t part_rows, int* err, int batch, bool invariant, int* S, size_t* part_stride,
                           cudaStream_t st, int variant = 0, unsigned* tile_counters = nullptr,
                           bool packed = false);

// Repack a row-major [N, K] bf16 weight (N % 128 == 0, K % 64 == 0) into the
// packed tile layout the tensor-core GEMM streams with bulk copies: 128 x 64
// tiles, each stored as its 16 KB 128-byte-swizzled shared-memory image
// (row r's 16-byte chunk c at r*128 + (c ^ (r % 8))*16), tile (n, k) at
// ((n * K/64) + k) * 16 KB.  dst holds N*K*2 bytes.
cudaError_t launch_pack_weight(const bf16* W, void* dst, int N, int K, cudaStream_t st);

}  // namespace dory

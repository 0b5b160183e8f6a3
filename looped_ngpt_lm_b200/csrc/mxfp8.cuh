// MXFP8 weights: quantiser and the decode GEMV that streams them.
#pragma once

#include "common.cuh"

namespace dory {

// Weights per E8M0 scale (one block of a weight row, along K).
constexpr int kMxBlock = 32;

// MXFP8 copy of a row-major bf16 weight W [N, K] (K % 32 == 0): E4M3 codes
// q [N, K] and E8M0 scale bytes s [N, K/32], scale of (n, k) at s[n*K/32 +
// k/32].  Per block: shared = floor(log2(max |w|)) - 8, clamped to
// [-127, 127] (-127 for a zero block); code = E4M3(w * 2^-shared) rounded to
// nearest-even, magnitudes above 448 clamped to 448, a value that rounds to
// zero keeps its sign; s = shared + 127.  deq (nullable) receives the
// dequantised weights 2^shared * E4M3 as bf16 [N, K].  A non-finite weight
// sets DEV_ERR_RANGE in *err.  W, q and deq 16-byte aligned.
cudaError_t launch_mx_quantize(const bf16* W, int N, int K, uint8_t* q, uint8_t* s, bf16* deq, int* err,
                               cudaStream_t st);

// Y[m, n] = sum_k X[m, k] * 2^(s[n, k/32] - 127) * E4M3(q[n, k]) for
// m < M, n < N: bf16 activations X (row stride ldx), fp32 result Y (row
// stride ldy), fp32 sums.  Each Y[m, n] is computed in an order fixed by K
// alone, so its bits do not depend on M.  K % 32 == 0 and q 16-byte aligned,
// else cudaErrorNotSupported.
// impl 2: tensor cores (mma.sync, f16 operands, fp32 accumulators; K <= 10240;
//   finite X, else DEV_ERR_RANGE in *err; |x| below 2^-124 contributes
//   nothing).
// impl 1: CUDA cores (|X| < 2^64, else DEV_ERR_RANGE; scale bytes <= 198,
//   the quantiser's output for |w| < 2^80; K <= 40960).
// impl 0: 1 (the faster of the two at every 4B decode shape).
cudaError_t launch_mx_gemv(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s,
                           float* Y, int ldy, int* err, cudaStream_t st, int impl = 0);

}  // namespace dory

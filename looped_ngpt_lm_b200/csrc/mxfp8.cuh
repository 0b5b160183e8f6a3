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
// impl 3: the TMA-fed tensor-core GEMM below, unsplit (N % 128 == 0,
//   K % 128 == 0, X 16-byte aligned with ldx % 8 == 0, |X| < 4).
// impl 4: impl 1's arithmetic (the same bits) with the weight rows streamed
//   into shared memory by bulk copies (8-row units, N % 8 == 0, at most
//   24 KB of weights per unit, the staged activations and two units within
//   75 KB); other shapes take impl 1.
// impl 0: 4 where it takes the shape, else 1 (the same bits either way;
//   measured faster than 1 and 2 in a 4B decode step).
// S > 1 (impl 0 / 1 only, K % (32 S) == 0): split K into S equal ranges;
// split s writes its partial products to Y + s * part_stride and the
// consumer adds them in order s = 0..S-1.
cudaError_t launch_mx_gemv(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s,
                           float* Y, int ldy, int* err, cudaStream_t st, int impl = 0, int S = 1,
                           size_t part_stride = 0);
// Splits for the CUDA-core GEMV inside a decode step: doubled while the rows
// fill fewer than 48 warps per SM, at most 8, each split at least 512
// weights.  Depends on (N, K) only.
int mx_gemv_splits(int N, int K);

// Low-bit decode GEMMs on the tensor cores, fed by TMA (mx_gemm_tc.cu): S
// partial products at Y + s * part_stride (row stride ldy) that the consumer
// adds in order s = 0..S-1, for X [M, K] bf16 (row stride ldx), any M.  The
// K range of each split depends on (K, S) only and the tokens are
// independent MMA columns, so a row's bits do not depend on M.  Limits:
// N % 128 == 0, K % 128 (MXFP8) or K % 256 (NVFP4) == 0, X and q 16-byte
// aligned, ldx % 8 == 0 (else cudaErrorNotSupported); |X| < 4 (else
// DEV_ERR_RANGE).
// MXFP8: q [N, K] E4M3 codes, s [N, K/32] E8M0 scales.
cudaError_t launch_mx_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s,
                              float* Y, int ldy, size_t part_stride, int S, int* err, cudaStream_t st);
// NVFP4: q [N, K/2] E2M1 code pairs (even k in the low nibble), s [N, K/16]
// E4M3 block scales, g the per-tensor scale (one device float).
cudaError_t launch_nv_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s,
                              const float* g, float* Y, int ldy, size_t part_stride, int S, int* err,
                              cudaStream_t st);

// NVFP4 copy of a row-major bf16 W [N, K] (K % 16 == 0): g (one device float)
// receives the power-of-two tensor scale, q [N, K/2] the E2M1 code pairs, s
// [N, K/16] the E4M3 block scales, deq (nullable) the exact bf16
// dequantisation.  Three launches on st.  W, deq 16-byte aligned, q 8-byte
// aligned.  A non-finite weight sets DEV_ERR_RANGE.
cudaError_t launch_nv_quantize(const bf16* W, int N, int K, uint8_t* q, uint8_t* s, float* g, bf16* deq, int* err,
                               cudaStream_t st);

// Splits for the two GEMMs: enough (N / 128, split) units to cover the SMs,
// at most 8 and at most one per chunk.  Depend on (N, K) only.
int mx_gemm_splits(int N, int K);
int nv_gemm_splits(int N, int K);

}  // namespace dory

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
// early: issued by the MMA warp before the launch waits for its predecessor
// (a GEMM launched early next to a latency-bound kernel then streams the
// following weights while HBM would idle), not after its own loads.
struct PfCtl {
  const PfSeg* segs = nullptr;
  int nseg = 0;
  int first = 0;  // a segment at or before the one holding lo
  unsigned long long lo = 0, hi = 0;
  int early = 0;
  // decode tiles: before waiting for the previous kernel, the producer asks
  // L2 for up to `own` more of this CTA's own weight tiles past those its
  // shared-memory ring takes (0: none)
  int own = 0;
};

// Operand stage of a decode GEMM (M <= 16 rows).  Instead of loading X by
// TMA, the four epilogue warps build the bf16 operand in shared memory from
// the previous kernel's fp32 outputs, so the elementwise step between two
// GEMMs costs no launch of its own:
//   kPrepAddNorm: X = N(h_in + sum_{s<S} y_s) (rows of d = K floats, the
//                 arithmetic of addnorm.cuh); the first CTA also writes the
//                 fp32 result to h_out (a buffer other than h_in);
//   kPrepSwiglu:  X[m, j] = silu(sum_s y_s[m, j]) * sum_s y_s[m, K + j], the
//                 SwiGLU of a split gate-up product (rows of ldy = 2K floats).
// y_s = y + s * ps.  X and ldx are unused.
enum : int { kPrepNone = 0, kPrepAddNorm = 1, kPrepSwiglu = 2 };
struct Prep {
  int mode = kPrepNone;
  const float* h_in = nullptr;
  float* h_out = nullptr;
  const float* y = nullptr;
  int S = 1;
  size_t ps = 0;
  int ldy = 0;
};

// Prefetch this CTA's piece of the look-ahead range into L2 (CTA b takes
// the b-th of gridDim.x equal pieces); called by `nthreads` threads, thread
// t taking every nthreads-th 128-byte line.  Segment sizes and offsets are
// multiples of 128 bytes.
__device__ __forceinline__ void l2_look_ahead(const PfCtl& pf, int t, int nthreads) {
  const unsigned long long span = pf.hi - pf.lo;
  const unsigned long long piece = ((span + gridDim.x - 1) / gridDim.x + 127) & ~127ull;
  const unsigned long long a0 = pf.lo + piece * blockIdx.x;
  const unsigned long long a1 = a0 + piece < pf.hi ? a0 + piece : pf.hi;
  if (a0 >= a1) return;
  for (int q = pf.first; q < pf.nseg && pf.segs[q].off < a1; ++q) {
    const unsigned long long so = pf.segs[q].off, se = so + pf.segs[q].bytes;
    if (se <= a0) continue;
    const unsigned long long lo = a0 > so ? a0 : so, hi = a1 < se ? a1 : se;
    const char* base = pf.segs[q].p - so;
    for (unsigned long long a = (lo & ~127ull) + 128ull * t; a < hi; a += 128ull * nthreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(base + a));
  }
}

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
// tiles only; ignored for prefill tiles).  prep (decode tiles, M <= 16): the
// operand stage above; cudaErrorNotSupported when this shape cannot take it
// (the caller then runs the elementwise step and a plain GEMM).  A GEMM with
// an operand stage computes the same bits as the plain one on the operand
// the standalone kernels would have written.
// cta_cap (decode tiles): when the weight tiles allow it, split K only so
// far that the units fit in this many CTAs, leaving the other SMs to a
// kernel that runs alongside (the decode attention that precedes an O
// projection: the whole projection then loads its weights while the
// attention runs).  Depends on the number of sequences only, never on M.
cudaError_t launch_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const bf16* W, float* Y, int ldy,
                           size_t part_rows, int* err, int batch, bool invariant, int* S, size_t* part_stride,
                           cudaStream_t st, int variant = 0, bool packed = false, const PfCtl* pf = nullptr,
                           const Prep* prep = nullptr, int cta_cap = 0);

// act[m, j] = silu(g) * u (bf16, row stride dff) with g = X[m] . Wgu[j] and
// u = X[m] . Wgu[dff + j] for the concatenated [gate; up] weight Wgu
// [2 dff, K]: the gate-up projection and SwiGLU of a long chunk in one
// tensor-core GEMM (fp32 accumulation, no split).  dff % 128 == 0.
cudaError_t launch_gemm_glu(int M, int dff, int K, const bf16* X, int ldx, const bf16* Wgu, bf16* act,
                            int* err, cudaStream_t st);

// Whether a decode GEMM of this shape (M rows, `batch` sequences) can take
// the operand stage `p` (the checks launch_gemm_tc makes, without launching).
bool gemm_tc_prep_ok(int M, int N, int K, int batch, const Prep& p);

// Repack a row-major [N, K] bf16 weight (N % 128 == 0, K % 64 == 0) into the
// packed tile layout the tensor-core GEMM streams with bulk copies: 128 x 64
// tiles, each stored as its 16 KB 128-byte-swizzled shared-memory image
// (row r's 16-byte chunk c at r*128 + (c ^ (r % 8))*16), tile (n, k) at
// ((n * K/64) + k) * 16 KB.  dst holds N*K*2 bytes.
cudaError_t launch_pack_weight(const bf16* W, void* dst, int N, int K, cudaStream_t st);

}  // namespace dory

// NVFP4 weights: the quantiser.  E2M1 codes (two per byte, the even k in the
// low nibble), one E4M3 scale per 16 consecutive weights of a row, and one
// per-tensor scale g: w = E2M1(code) * E4M3(scale) * g.
//
// The pages list NVFP4 among the released weight formats and give its batch-1
// decode speed over BF16 ("NVIDIA, 반복 연산형 4B 언어 모델 Dory 공개",
// section "KV 캐시와 실행 환경"; lucasainews formats article, section
// "학습 방식과 변형").  The recipe:
// - g = the smallest power of two with 6 * 448 * g >= max |w| (1 for a zero
//   tensor), so the largest block scale lies in (224, 448];
// - block scale = E4M3(amax_b / (6 g)), round-to-nearest-even, saturating;
// - code = E2M1(w / (scale * g)), round-to-nearest-even, saturating at 6;
//   0 for a block whose scale is 0; a value that rounds to zero keeps its
//   sign.
// Both divisions are done in double precision: the quotient of a bf16 value
// by 6 * 2^k or by an E4M3 value times 2^k either is exact or has an infinite
// binary expansion, so double rounding cannot move it onto a tie of the
// 4-bit or 2-bit mantissa, and the rounding equals that of the exact
// quotient.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "mxfp8.cuh"

namespace dory {
namespace {

constexpr int NV_BLOCK = 16;

// largest |w| over the tensor, as bf16 magnitude bits (monotone in the value)
__global__ void k_nv_amax(const bf16* __restrict__ W, long long n, unsigned* amax, int* err) {
  const unsigned short* b = reinterpret_cast<const unsigned short*>(W);
  unsigned m = 0;
  bool bad = false;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const unsigned v = b[i] & 0x7FFFu;
    bad |= v >= 0x7F80u;
    m = v > m ? v : m;
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) atomicMax(amax, m);
  if (bad) set_error(err, DEV_ERR_RANGE);
}

// g from the largest magnitude (written over it as a float)
__global__ void k_nv_gscale(unsigned* amax_then_g) {
  const float amax = __uint_as_float(*amax_then_g << 16);
  float g = 1.f;
  if (amax > 0.f) {
    const float top = 6.f * 448.f;
    int e;
    frexpf(amax / top, &e);
    int k = e;
    while (ldexpf(top, k) < amax) ++k;
    while (ldexpf(top, k - 1) >= amax) --k;
    g = ldexpf(1.f, k);
  }
  *reinterpret_cast<float*>(amax_then_g) = g;
}

__global__ void k_nv_quantize(const bf16* __restrict__ W, long long nblk, const float* __restrict__ gp,
                              uint8_t* __restrict__ q, uint8_t* __restrict__ s, bf16* __restrict__ deq) {
  const long long blk = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= nblk) return;
  const double g = (double)*gp;
  const uint4* src = reinterpret_cast<const uint4*>(W + blk * NV_BLOCK);
  const uint4 a = src[0], b = src[1];
  const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t amax = 0;
#pragma unroll
  for (int j = 0; j < NV_BLOCK; ++j) {
    const uint32_t mag = (wv[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
    amax = mag > amax ? mag : amax;
  }
  const double am = (double)__uint_as_float(amax << 16);
  const uint8_t sc = (uint8_t)__nv_cvt_double_to_fp8(am / (6.0 * g), __NV_SATFINITE, __NV_E4M3);
  const __half_raw sh = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sc, __NV_E4M3);
  const double sv = (double)__half2float(__half(sh));
  uint32_t packed[2] = {0u, 0u};
  float dv[NV_BLOCK];
#pragma unroll
  for (int j = 0; j < NV_BLOCK; ++j) {
    const uint32_t bits = (wv[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
    const double x = (double)__uint_as_float(bits << 16);
    uint32_t c = sv > 0.0 ? (uint32_t)__nv_cvt_double_to_fp4(x / (sv * g), __NV_E2M1, cudaRoundNearest) & 0xFu : 0u;
    if ((c & 0x7u) == 0u) c = (bits & 0x8000u) ? 0x8u : 0x0u;  // zero keeps the weight's sign
    packed[j >> 3] |= c << (4 * (j & 7));
    if (deq) {
      const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)c, __NV_E2M1);
      dv[j] = __half2float(__half(__half_raw{h.x})) * (float)sv * (float)g;  // exact: short mantissas, 2^k
    }
  }
  *reinterpret_cast<uint2*>(q + blk * (NV_BLOCK / 2)) = make_uint2(packed[0], packed[1]);
  s[blk] = sc;
  if (deq) {
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < NV_BLOCK; j += 2) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(dv[j], dv[j + 1]);
      o[j >> 1] = *reinterpret_cast<const uint32_t*>(&p);
    }
    uint4* dd = reinterpret_cast<uint4*>(deq + blk * NV_BLOCK);
    dd[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dd[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

cudaError_t launch_nv_quantize(const bf16* W, int N, int K, uint8_t* q, uint8_t* s, float* g, bf16* deq, int* err,
                               cudaStream_t st) {
  if (N <= 0 || K <= 0 || K % NV_BLOCK || !g) return cudaErrorNotSupported;
  if (((uintptr_t)W & 15) || ((uintptr_t)q & 7) || ((uintptr_t)deq & 15) || ((uintptr_t)g & 3))
    return cudaErrorNotSupported;
  const long long n = (long long)N * K, nblk = n / NV_BLOCK;
  cudaError_t e = cudaMemsetAsync(g, 0, sizeof(float), st);
  if (e != cudaSuccess) return e;
  k_nv_amax<<<296, 256, 0, st>>>(W, n, reinterpret_cast<unsigned*>(g), err);
  k_nv_gscale<<<1, 1, 0, st>>>(reinterpret_cast<unsigned*>(g));
  const long long grid = (nblk + 255) / 256;
  if (grid > 0x7FFFFFFFLL) return cudaErrorNotSupported;
  k_nv_quantize<<<(unsigned)grid, 256, 0, st>>>(W, nblk, g, q, s, deq);
  return cudaGetLastError();
}

}  // namespace dory

// MXFP8 weights (OCP Microscaling Formats v1.0: FP8 E4M3 elements, one E8M0
// scale per 32 consecutive weights of a row): the quantiser, and the decode
// GEMV that reads them.
//
// The pages list MXFP8 among the released weight formats.  They measure it
// against BF16 at batch 1, where decoding is bound by weight bytes
// ("NVIDIA, 반복 연산형 4B 언어 모델 Dory 공개", section "KV 캐시와 실행 환경";
// lucasainews formats article, section "학습 방식과 변형").  A decode step at
// small batch is a matrix-vector product per weight matrix, bound by HBM, so
// the GEMV runs on the CUDA cores.  Each warp streams one weight row at a
// time in 16-byte chunks.  The activations, pre-scaled, are staged once per
// CTA in shared memory.
#include <cuda_fp8.h>
#include <float.h>

#include <map>

#include "mxfp8.cuh"

namespace dory {

namespace {

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// ------------------------------------------------------------------ quantiser
// One thread per 32-weight block (64 bytes of bf16 in, 32 code bytes and one
// scale byte out).
__global__ void k_mx_quantize(const bf16* __restrict__ W, long long nblk, uint8_t* __restrict__ q,
                              uint8_t* __restrict__ s, bf16* __restrict__ deq, int* err) {
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblk) return;
  const uint4* src = reinterpret_cast<const uint4*>(W + b * kMxBlock);
  uint32_t wv[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = src[i];
    wv[4 * i] = v.x;
    wv[4 * i + 1] = v.y;
    wv[4 * i + 2] = v.z;
    wv[4 * i + 3] = v.w;
  }
  // largest magnitude from the bf16 bit patterns (integer order = magnitude
  // order for finite values)
  uint32_t amax = 0;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kMxBlock; ++j) {
    const uint32_t mag = (wv[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
    bad |= mag >= 0x7F80u;
    amax = mag > amax ? mag : amax;
  }
  if (bad) set_error(err, DEV_ERR_RANGE);
  const int ebits = (int)(amax >> 7);  // biased exponent of the block maximum (0: zero or subnormal)
  int shared = ebits == 0 ? -127 : ebits - 127 - 8;
  shared = shared < -127 ? -127 : (shared > 127 ? 127 : shared);
  const float inv = __uint_as_float((uint32_t)(127 - shared) << 23);  // 2^-shared, exponent in [-119, 127]
  uint32_t cw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) cw[i] = 0u;
#pragma unroll
  for (int j = 0; j < kMxBlock; ++j) {
    const uint32_t bits = (wv[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
    const float y = __uint_as_float(bits << 16) * inv;  // exact: a power-of-two scaling
    uint32_t c = (uint32_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
    if ((c & 0x7Fu) == 0u) c = (bits & 0x8000u) ? 0x80u : 0x00u;  // zero keeps the weight's sign
    cw[j >> 2] |= c << (8 * (j & 3));
  }
  uint4* dq = reinterpret_cast<uint4*>(q + b * kMxBlock);
  dq[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  dq[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
  s[b] = (uint8_t)(shared + 127);
  if (deq) {
    uint32_t dv[16];
#pragma unroll
    for (int j = 0; j < kMxBlock; j += 2) {
      float v[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint32_t c = (cw[(j + t) >> 2] >> (8 * ((j + t) & 3))) & 0xFFu;
        // the code's value times 2^-120 (see e4m3_scaled below), then exact rescaling
        const float e = __uint_as_float(((c & 0x80u) << 24) | ((c & 0x7Fu) << 20)) * 0x1p120f;
        v[t] = ldexpf(e, shared);
      }
      const __nv_bfloat162 p = __floats2bfloat162_rn(v[0], v[1]);
      dv[j >> 1] = *reinterpret_cast<const uint32_t*>(&p);
    }
    uint4* dd = reinterpret_cast<uint4*>(deq + b * kMxBlock);
#pragma unroll
    for (int i = 0; i < 4; ++i) dd[i] = make_uint4(dv[4 * i], dv[4 * i + 1], dv[4 * i + 2], dv[4 * i + 3]);
  }
}

// ------------------------------------------------------------------ GEMV
constexpr int GV_T = 256;  // threads per CTA
constexpr int GV_W = GV_T / 32;
constexpr int GV_U = 4;    // 16-byte weight chunks per lane in flight
constexpr int GV_SMEM_CAP = 160 * 1024;

// The E4M3 code in the top byte of v, as a float equal to its value times
// 2^-120, exactly: after the arithmetic shift the code's exponent and
// mantissa (bits 0..6) sit in float bits 20..26 and its sign in bit 31, so
// the 4-bit exponent (bias 7) is read with the float's bias 127, and E4M3
// subnormals (exponent 0) become float subnormals.
__device__ __forceinline__ float e4m3_scaled(uint32_t v) {
  return __uint_as_float((uint32_t)((int32_t)v >> 4) & 0x87F00000u);
}

// Products are formed against x * 2^64 (staged), so with the codes' 2^-120
// each product is the true one times 2^-56: normal floats for |q x| >= 2^-70.
// The block scale 2^(s - 127) then enters as 2^(s - 127 + 56) = 2^(s - 71).
__device__ __forceinline__ float block_scale(uint32_t sb) {
  const uint32_t e = sb + 56u;
  return __uint_as_float((e < 255u ? e : 255u) << 23);  // +inf past the supported range
}

template <int MT>
__global__ void __launch_bounds__(GV_T) k_mx_gemv(int M, int N, int K, const bf16* __restrict__ X, int ldx,
                                                  const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                                                  float* __restrict__ Y, int ldy, int* err) {
  extern __shared__ float4 xs[];  // [MT][4][nch]: float4 i of chunk c of token m at (m*4 + i)*nch + c
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = K >> 4, nsb = K >> 5, K4 = K >> 2;
  const int gw = blockIdx.x * GV_W + warp, nw = gridDim.x * GV_W;

  // The weights do not depend on earlier kernels: ask L2 for this warp's
  // first row while the previous kernel finishes.
  if (gw < N) {
    const char* row = reinterpret_cast<const char*>(q) + (size_t)gw * K;
    for (int a = lane * 128; a < K; a += 32 * 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + a));
    if (lane * 128 < nsb) asm volatile("prefetch.global.L2 [%0];" ::"l"(s + (size_t)gw * nsb + lane * 128));
  }
  pdl_wait();

  for (int m0 = 0; m0 < M; m0 += MT) {
    const int mc = M - m0 < MT ? M - m0 : MT;
    if (m0 > 0) __syncthreads();  // every warp is done with the previous tokens
    // stage x * 2^64 (exact for |x| < 2^64) in the chunk-major layout
    bool bad = false;
    for (int e = threadIdx.x; e < MT * K4; e += GV_T) {
      const int m = e / K4, r = e - m * K4;  // elements 4r..4r+3 of token m
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m < mc) {
        const bf16* xr = X + (size_t)(m0 + m) * ldx + 4 * r;
        v.x = __bfloat162float(xr[0]) * 0x1p64f;
        v.y = __bfloat162float(xr[1]) * 0x1p64f;
        v.z = __bfloat162float(xr[2]) * 0x1p64f;
        v.w = __bfloat162float(xr[3]) * 0x1p64f;
        bad |= !(fabsf(v.x) <= FLT_MAX && fabsf(v.y) <= FLT_MAX && fabsf(v.z) <= FLT_MAX && fabsf(v.w) <= FLT_MAX);
      }
      xs[((m << 2) + (r & 3)) * nch + (r >> 2)] = v;
    }
    if (bad) set_error(err, DEV_ERR_RANGE);
    __syncthreads();
    if (m0 == 0) pdl_trigger();

    for (int n = gw; n < N; n += nw) {
      const uint4* qrow = reinterpret_cast<const uint4*>(q + (size_t)n * K);
      const uint8_t* srow = s + (size_t)n * nsb;
      float acc[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.f;
      for (int c0 = lane; c0 < nch; c0 += 32 * GV_U) {
        uint4 w[GV_U];
        uint32_t sb[GV_U];
#pragma unroll
        for (int u = 0; u < GV_U; ++u) {
          const int c = c0 + 32 * u;
          if (c < nch) {
            w[u] = __ldcs(qrow + c);
            sb[u] = srow[c >> 1];
          }
        }
#pragma unroll
        for (int u = 0; u < GV_U; ++u) {
          const int c = c0 + 32 * u;
          if (c < nch) {
            float f[16];
            const uint32_t wd[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              f[4 * i] = e4m3_scaled(wd[i] << 24);
              f[4 * i + 1] = e4m3_scaled(wd[i] << 16);
              f[4 * i + 2] = e4m3_scaled(wd[i] << 8);
              f[4 * i + 3] = e4m3_scaled(wd[i]);
            }
            const float sc = block_scale(sb[u]);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const float4* xp = xs + (m << 2) * nch + c;
              float p[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 a = xp[i * nch];
                float t = __fmul_rn(f[4 * i], a.x);
                t = __fmaf_rn(f[4 * i + 1], a.y, t);
                t = __fmaf_rn(f[4 * i + 2], a.z, t);
                p[i] = __fmaf_rn(f[4 * i + 3], a.w, t);
              }
              acc[m] = __fmaf_rn(__fadd_rn(__fadd_rn(p[0], p[1]), __fadd_rn(p[2], p[3])), sc, acc[m]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float v = warp_sum(acc[m]);
        if (lane == 0 && m < mc) Y[(size_t)(m0 + m) * ldy + n] = v;
      }
    }
  }
}

template <int MT>
cudaError_t run_gemv(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s, float* Y,
                     int ldy, int* err, cudaStream_t st) {
  const int smem = MT * K * 4;
  static int attr_smem = 0;
  static std::map<int, int> per_sm;  // dynamic shared memory -> resident CTAs per SM
  if (smem > attr_smem) {
    cudaError_t e = cudaFuncSetAttribute(k_mx_gemv<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_smem = smem;
  }
  auto it = per_sm.find(smem);
  if (it == per_sm.end()) {
    int b = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_mx_gemv<MT>, GV_T, smem);
    if (e != cudaSuccess) return e;
    it = per_sm.emplace(smem, b < 1 ? 1 : b).first;
  }
  const long long want = ((long long)N + GV_W - 1) / GV_W;
  const long long cap = (long long)num_sms() * it->second;
  const int grid = (int)(want < cap ? want : cap);
  return launch(k_mx_gemv<MT>, grid, GV_T, smem, st, M, N, K, X, ldx, q, s, Y, ldy, err);
}

}  // namespace

cudaError_t launch_mx_quantize(const bf16* W, int N, int K, uint8_t* q, uint8_t* s, bf16* deq, int* err,
                               cudaStream_t st) {
  if (N <= 0 || K <= 0 || K % kMxBlock) return cudaErrorNotSupported;
  if (((uintptr_t)W & 15) || ((uintptr_t)q & 15) || ((uintptr_t)deq & 15)) return cudaErrorNotSupported;
  const long long nblk = (long long)N * (K / kMxBlock);
  const long long grid = (nblk + 255) / 256;
  if (grid > 0x7FFFFFFFLL) return cudaErrorNotSupported;
  k_mx_quantize<<<(unsigned)grid, 256, 0, st>>>(W, nblk, q, s, deq, err);
  return cudaGetLastError();
}

cudaError_t launch_mx_gemv(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s,
                           float* Y, int ldy, int* err, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kMxBlock || ((uintptr_t)q & 15)) return cudaErrorNotSupported;
  // tokens per pass: the smallest power of two covering M, up to 8, within
  // the staged-activation budget
  int cap = GV_SMEM_CAP / (K * 4);
  if (cap < 1) return cudaErrorNotSupported;
  int MT = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  while (MT > cap) MT >>= 1;
  switch (MT) {
    case 1: return run_gemv<1>(M, N, K, X, ldx, q, s, Y, ldy, err, st);
    case 2: return run_gemv<2>(M, N, K, X, ldx, q, s, Y, ldy, err, st);
    case 4: return run_gemv<4>(M, N, K, X, ldx, q, s, Y, ldy, err, st);
    default: return run_gemv<8>(M, N, K, X, ldx, q, s, Y, ldy, err, st);
  }
}

}  // namespace dory

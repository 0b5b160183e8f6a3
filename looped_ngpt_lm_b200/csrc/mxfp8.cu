// MXFP8 weights (OCP Microscaling Formats v1.0: FP8 E4M3 elements, one E8M0
// scale per 32 consecutive weights of a row): the quantiser, and two decode
// GEMVs that read them.
//
// The pages list MXFP8 among the released weight formats.  They measure it
// against BF16 at batch 1, where decoding is bound by weight bytes
// ("NVIDIA, 반복 연산형 4B 언어 모델 Dory 공개", section "KV 캐시와 실행 환경";
// lucasainews formats article, section "학습 방식과 변형").  A decode step at
// small batch is a matrix-vector product per weight matrix, bound by HBM.
//
// k_mx_gemv (the default) runs on the CUDA cores.  Each warp streams one
// weight row at a time in 16-byte chunks, against activations staged once
// per CTA in shared memory.  k_mx_gemv_tc puts the products on the tensor
// cores (mma.sync).  Measured on the 4B decode shapes, both are
// latency-bound: each warp keeps its own loads in registers.  The
// CUDA-core kernel is the faster of the two.
#include <cuda_fp8.h>
#include <float.h>

#include <map>

#include "mxfp8.cuh"
#include "umma.cuh"
#include "warp_mma.cuh"

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

// Split-K: blockIdx.y = split s takes weights [s Ks, (s + 1) Ks) of every
// row and writes its partial dot products to Y + s * part_stride.
template <int MT>
__global__ void __launch_bounds__(GV_T) k_mx_gemv(int M, int N, int K, const bf16* __restrict__ X, int ldx,
                                                  const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                                                  float* __restrict__ Y, int ldy, int* err, int Ks,
                                                  size_t part_stride) {
  extern __shared__ float4 xs[];  // [MT][4][nch]: float4 i of chunk c of token m at (m*4 + i)*nch + c
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = blockIdx.y * Ks;
  const int nch = Ks >> 4, nsb = K >> 5, K4 = Ks >> 2;
  const int gw = blockIdx.x * GV_W + warp, nw = gridDim.x * GV_W;
  q += k0;
  s += k0 >> 5;
  X += k0;
  Y += blockIdx.y * part_stride;

  // The weights do not depend on earlier kernels: ask L2 for this warp's
  // first row while the previous kernel finishes.
  if (gw < N) {
    const char* row = reinterpret_cast<const char*>(q) + (size_t)gw * K;
    for (int a = lane * 128; a < Ks; a += 32 * 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + a));
    if (lane * 128 < (Ks >> 5)) asm volatile("prefetch.global.L2 [%0];" ::"l"(s + (size_t)gw * nsb + lane * 128));
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

// ------------------------------------------------------------------ GEMV fed by bulk copies
// The same per-row arithmetic as k_mx_gemv (lane l takes the 16-weight
// chunks l, l + 32, ... of its row, in that order), with the weight rows
// streamed into shared memory by bulk copies instead of each warp's own
// loads: one producer warp keeps a ring of RG_MAX_STAGES units of 8 rows in
// flight (the weights do not depend on earlier kernels, so it starts before
// the predecessor grid has finished), and eight consumer warps take one row
// each; three CTAs share an SM.  blockIdx.y is the K split, as in k_mx_gemv.  Every mbarrier wait is
// bounded; on expiry the CTA sets the error word, stops, and the producer
// waits (bounded) for its copies in flight.
constexpr int RG_RPU = 8;                // weight rows per unit
constexpr int RG_NC = 8;                 // consumer warps, one row each
constexpr int RG_T = (RG_NC + 1) * 32;   // + the producer warp
constexpr int RG_MAX_STAGES = 3;
constexpr int RG_STAGE_CAP = 24 * 1024;  // weight bytes of one unit (8 rows x the split's K range)
constexpr int RG_MAXC = RG_STAGE_CAP / RG_RPU / 16 / 32;  // 16-weight chunks of a row per lane: 6
constexpr int RG_SMEM_CAP = 75 * 1024;   // three CTAs per SM

__device__ __forceinline__ void rg_bulk(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

template <int MT>
__global__ void __launch_bounds__(RG_T) k_mx_gemv_ring(int M, int N, int K, const bf16* __restrict__ X, int ldx,
                                                       const uint8_t* __restrict__ q,
                                                       const uint8_t* __restrict__ s, float* __restrict__ Y,
                                                       int ldy, int* err, int Ks, size_t part_stride, int stages) {
  using namespace tc;
  extern __shared__ __align__(128) uint8_t rg_smem[];
  const int unit_bytes = RG_RPU * Ks;
  uint8_t* wbuf = rg_smem;                                              // [stages][8 rows][Ks]
  float4* xs = reinterpret_cast<float4*>(rg_smem + stages * unit_bytes);  // [MT][4][nch]
  uint64_t* full = reinterpret_cast<uint64_t*>(rg_smem + stages * unit_bytes + MT * Ks * 4);
  uint64_t* empty = full + RG_MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + RG_MAX_STAGES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = blockIdx.y * Ks;
  const int nch = Ks >> 4, nsb = K >> 5, K4 = Ks >> 2;
  const int n_units = N / RG_RPU;
  q += k0;
  s += k0 >> 5;
  X += k0;
  Y += blockIdx.y * part_stride;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], RG_NC);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == RG_NC) {
    // ---------------- producer: weights need nothing from earlier kernels
    if (lane == 0) {
      int i = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++i) {
        const int st = i % stages;
        if (i >= stages && !mbar_wait(&empty[st], ((i / stages) + 1) & 1, abort_flag, err)) break;
        const uint32_t dst = smem_u32(wbuf + (size_t)st * unit_bytes);
        mbar_expect_tx(&full[st], (uint32_t)unit_bytes);
        if (Ks == K) {
          rg_bulk(dst, q + (size_t)u * RG_RPU * K, (uint32_t)unit_bytes, &full[st]);
        } else {
          for (int r = 0; r < RG_RPU; ++r)
            rg_bulk(dst + r * Ks, q + ((size_t)u * RG_RPU + r) * K, (uint32_t)Ks, &full[st]);
        }
      }
      // copies still in flight land before the CTA can exit
      for (int j = i - stages < 0 ? 0 : i - stages; j < i; ++j) mbar_wait_drain(&full[j % stages], (j / stages) & 1);
    }
    return;
  }

  // ---------------- consumers
  pdl_wait();
  for (int m0 = 0; m0 < M; m0 += MT) {
    const int mc = M - m0 < MT ? M - m0 : MT;
    if (m0 > 0) asm volatile("bar.sync 1, %0;" ::"r"(RG_NC * 32) : "memory");  // done with the previous tokens
    bool bad = false;
    for (int e = threadIdx.x; e < MT * K4; e += RG_NC * 32) {
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
    asm volatile("bar.sync 1, %0;" ::"r"(RG_NC * 32) : "memory");
    if (m0 == 0 && threadIdx.x == 0) pdl_trigger();

    int i = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++i) {
      const int st = i % stages;
      const int rl = warp, n = u * RG_RPU + rl;
      // this lane's scale bytes, requested before the weights are waited for
      const uint8_t* srow = s + (size_t)n * nsb;
      uint32_t sbv[RG_MAXC];
#pragma unroll
      for (int t = 0; t < RG_MAXC; ++t) {
        const int c = lane + 32 * t;
        sbv[t] = c < nch ? __ldg(srow + (c >> 1)) : 0u;
      }
      // launches have M <= MT: one token pass, each unit streamed once
      if (!mbar_wait(&full[st], (i / stages) & 1, abort_flag, err)) break;
      {
        const uint4* qrow = reinterpret_cast<const uint4*>(wbuf + (size_t)st * unit_bytes + (size_t)rl * Ks);
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.f;
#pragma unroll
        for (int t = 0; t < RG_MAXC; ++t) {
          const int c = lane + 32 * t;
          if (c >= nch) break;
          const uint4 w = qrow[c];
          const uint32_t sb = sbv[t];
          float f[16];
          const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            f[4 * j] = e4m3_scaled(wd[j] << 24);
            f[4 * j + 1] = e4m3_scaled(wd[j] << 16);
            f[4 * j + 2] = e4m3_scaled(wd[j] << 8);
            f[4 * j + 3] = e4m3_scaled(wd[j]);
          }
          const float sc = block_scale(sb);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float4* xp = xs + (m << 2) * nch + c;
            float p[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 a = xp[j * nch];
              float t = __fmul_rn(f[4 * j], a.x);
              t = __fmaf_rn(f[4 * j + 1], a.y, t);
              t = __fmaf_rn(f[4 * j + 2], a.z, t);
              p[j] = __fmaf_rn(f[4 * j + 3], a.w, t);
            }
            acc[m] = __fmaf_rn(__fadd_rn(__fadd_rn(p[0], p[1]), __fadd_rn(p[2], p[3])), sc, acc[m]);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float v = warp_sum(acc[m]);
          if (lane == 0 && m < mc) Y[(size_t)(m0 + m) * ldy + n] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
  }
}

// Launches k_mx_gemv_ring when its shapes fit (8-row units whose split of K
// is at most RG_STAGE_CAP bytes, at least two stages in shared memory, one
// token pass); cudaErrorNotSupported otherwise.
template <int MT>
cudaError_t run_gemv_ring(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s, float* Y,
                          int ldy, int* err, cudaStream_t st, int S, size_t part_stride) {
  const int Ks = K / S;
  if (N % RG_RPU || M > MT || Ks % 16 || ((uintptr_t)q & 15) || RG_RPU * Ks > RG_STAGE_CAP)
    return cudaErrorNotSupported;
  const int fixed = MT * Ks * 4 + 2 * RG_MAX_STAGES * 8 + 16;
  int stages = (RG_SMEM_CAP - fixed) / (RG_RPU * Ks);
  if (stages > RG_MAX_STAGES) stages = RG_MAX_STAGES;
  if (stages < 2) return cudaErrorNotSupported;
  const int smem = stages * RG_RPU * Ks + fixed;
  static int attr_smem = 0;
  if (smem > attr_smem) {
    cudaError_t e = cudaFuncSetAttribute(k_mx_gemv_ring<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, RG_SMEM_CAP);
    if (e != cudaSuccess) return e;
    attr_smem = RG_SMEM_CAP;
  }
  const int units = N / RG_RPU;
  int gx = 3 * num_sms() / S;
  if (gx < 1) gx = 1;
  if (gx > units) gx = units;
  return launch(k_mx_gemv_ring<MT>, dim3(gx, S), dim3(RG_T), smem, st, M, N, K, X, ldx, q, s, Y, ldy, err, Ks,
                part_stride, stages);
}

template <int MT>
cudaError_t run_gemv(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s, float* Y,
                     int ldy, int* err, cudaStream_t st, int S, size_t part_stride) {
  const int Ks = K / S;
  const int smem = MT * Ks * 4;
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
  long long cap = (long long)num_sms() * it->second / S;
  if (cap < 1) cap = 1;
  const int grid = (int)(want < cap ? want : cap);
  return launch(k_mx_gemv<MT>, dim3(grid, S), dim3(GV_T), smem, st, M, N, K, X, ldx, q, s, Y, ldy, err, Ks,
                part_stride);
}

// ------------------------------------------------------------------ GEMV on the tensor cores
// One CTA computes 16 weight rows x up to 8 tokens at a time with
// mma.sync m16n8k16 (f16 operands, fp32 accumulators); its 8 warps split K
// into 8 fixed ranges of 32-weight blocks and their partial sums are added
// in warp order.  Each k16 step stays inside one block, so a block's partial
// product leaves the tensor core in fp32 and takes the block scale with one
// FMA.  The E4M3 codes become f16 in registers (exact: every E4M3 value is
// an f16 value); the activations are staged as f16 after a per-token
// power-of-two scaling 2^p that puts the token's largest |x| in [2^14, 2^15),
// exact for bf16 inputs whose magnitude is within 2^28 of that maximum, and
// the result is scaled back by 2^-p.
//
// k permutation: thread t of a quad (lane & 3) holds codes 8t..8t+7 of the
// block for its two rows (one 8-byte load each).  The MMA's k slots 2t, 2t+1
// and 2t+8, 2t+9 take codes (0, 1) and (2, 3) in the first k16 step and
// (4, 5), (6, 7) in the second; the activation fragment of the same thread
// reads x[8t .. 8t+7] of its token (one 16-byte shared-memory load), which
// applies the same permutation to x.  The dot product is unchanged.
constexpr int TV_T = 256;  // threads per CTA
constexpr int TV_W = TV_T / 32;
constexpr int TV_U = 8;    // blocks per warp in flight

__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// 2^(byte - 127), E8M0 (byte 0 is 2^-127, a float subnormal)
__device__ __forceinline__ float e8m0(uint32_t b) {
  return __uint_as_float(b == 0u ? 0x00400000u : b << 23);
}

__global__ void __launch_bounds__(TV_T) k_mx_gemv_tc(int M, int N, int K, const bf16* __restrict__ X, int ldx,
                                                     const uint8_t* __restrict__ q, const uint8_t* __restrict__ s,
                                                     float* __restrict__ Y, int ldy, int* err) {
  extern __shared__ __align__(16) unsigned char tv_smem[];
  __half* xs = reinterpret_cast<__half*>(tv_smem);  // [mc][K] f16, x * 2^p
  __shared__ float red[TV_W][32][4];
  __shared__ int s_p[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int nb = K >> 5, ntile = (N + 15) >> 4;
  const int kb0 = warp * nb / TV_W, kb1 = (warp + 1) * nb / TV_W;  // this warp's blocks

  // the first tile's weights do not depend on earlier kernels: ask L2 now
  if (blockIdx.x < ntile) {
    const int r = blockIdx.x * 16 + (threadIdx.x & 15);
    if (r < N) {
      const char* row = reinterpret_cast<const char*>(q) + (size_t)r * K;
      for (int a = (threadIdx.x >> 4) * 128; a < K; a += 16 * 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + a));
    }
  }
  pdl_wait();

  for (int m0 = 0; m0 < M; m0 += 8) {
    const int mc = M - m0 < 8 ? M - m0 : 8;
    if (m0 > 0) __syncthreads();  // every warp is done with the previous tokens
    // per-token exponent p from the largest |x| (bf16 bits), warp w: token w
    if (warp < mc) {
      const unsigned short* xr = reinterpret_cast<const unsigned short*>(X + (size_t)(m0 + warp) * ldx);
      uint32_t mx = 0;
      for (int k = lane; k < K; k += 32) {
        const uint32_t v = xr[k] & 0x7FFFu;
        mx = v > mx ? v : mx;
      }
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (lane == 0) {
        if (mx >= 0x7F80u) set_error(err, DEV_ERR_RANGE);  // inf or NaN
        // |x| < 2^128 needs p >= -113; below 2^-124 f16 keeps no bits of x * 2^100
        int p = mx == 0 ? 0 : 14 - ((int)(mx >> 7) - 127);
        s_p[warp] = p < -113 ? -113 : (p > 100 ? 100 : p);
      }
    }
    __syncthreads();
    // stage x * 2^p as f16 pairs
    const int K2 = K >> 1;
    for (int e = threadIdx.x; e < mc * K2; e += TV_T) {
      const int m = e / K2, k2 = e - m * K2;
      const float sc = __uint_as_float((uint32_t)(s_p[m] + 127) << 23);
      const bf16* xr = X + (size_t)(m0 + m) * ldx + 2 * k2;
      reinterpret_cast<__half2*>(xs)[e] = __floats2half2_rn(__bfloat162float(xr[0]) * sc,
                                                            __bfloat162float(xr[1]) * sc);
    }
    __syncthreads();
    if (m0 == 0) pdl_trigger();

    const bool hasx = g < mc;
    const __half* xg = xs + (size_t)(hasx ? g : 0) * K + 8 * t;
    for (int rt = blockIdx.x; rt < ntile; rt += gridDim.x) {
      const int r0 = rt * 16 + g, r1 = r0 + 8;
      // rows past N read row 0 (in bounds) and are never written
      const uint8_t* q0 = q + (size_t)(r0 < N ? r0 : 0) * K + 8 * t;
      const uint8_t* q1 = q + (size_t)(r1 < N ? r1 : 0) * K + 8 * t;
      const uint8_t* s0 = s + (size_t)(r0 < N ? r0 : 0) * nb;
      const uint8_t* s1 = s + (size_t)(r1 < N ? r1 : 0) * nb;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int b0 = kb0; b0 < kb1; b0 += TV_U) {
        uint2 w0[TV_U], w1[TV_U];
        uint32_t sa[TV_U], sb[TV_U];
#pragma unroll
        for (int u = 0; u < TV_U; ++u) {
          const int b = b0 + u;
          if (b < kb1) {
            w0[u] = __ldcs(reinterpret_cast<const uint2*>(q0 + (size_t)b * 32));
            w1[u] = __ldcs(reinterpret_cast<const uint2*>(q1 + (size_t)b * 32));
            sa[u] = s0[b];
            sb[u] = s1[b];
          }
        }
#pragma unroll
        for (int u = 0; u < TV_U; ++u) {
          const int b = b0 + u;
          if (b < kb1) {
            const uint4 xv = hasx ? *reinterpret_cast<const uint4*>(xg + (size_t)b * 32) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t a0[4] = {e4m3x2_f16x2(w0[u].x), e4m3x2_f16x2(w1[u].x), e4m3x2_f16x2(w0[u].x >> 16),
                                    e4m3x2_f16x2(w1[u].x >> 16)};
            const uint32_t a1[4] = {e4m3x2_f16x2(w0[u].y), e4m3x2_f16x2(w1[u].y), e4m3x2_f16x2(w0[u].y >> 16),
                                    e4m3x2_f16x2(w1[u].y >> 16)};
            float blk[4] = {0.f, 0.f, 0.f, 0.f};
            wm::mma_f16(blk, a0, xv.x, xv.y);
            wm::mma_f16(blk, a1, xv.z, xv.w);
            const float sc0 = e8m0(sa[u]), sc1 = e8m0(sb[u]);
            acc[0] = __fmaf_rn(blk[0], sc0, acc[0]);
            acc[1] = __fmaf_rn(blk[1], sc0, acc[1]);
            acc[2] = __fmaf_rn(blk[2], sc1, acc[2]);
            acc[3] = __fmaf_rn(blk[3], sc1, acc[3]);
          }
        }
      }
      // add the 8 warps' partial sums in warp order
#pragma unroll
      for (int j = 0; j < 4; ++j) red[warp][lane][j] = acc[j];
      __syncthreads();
      if (warp == 0) {
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[j] = red[0][lane][j];
#pragma unroll
          for (int w = 1; w < TV_W; ++w) v[j] = __fadd_rn(v[j], red[w][lane][j]);
        }
        // thread t holds tokens 2t, 2t+1 of rows r0 (v0, v1) and r1 (v2, v3)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int m = 2 * t + j;
          if (m < mc) {
            const float un = __uint_as_float((uint32_t)(127 - s_p[m]) << 23);
            if (r0 < N) Y[(size_t)(m0 + m) * ldy + r0] = v[j] * un;
            if (r1 < N) Y[(size_t)(m0 + m) * ldy + r1] = v[2 + j] * un;
          }
        }
      }
      __syncthreads();  // red is reused by the next tile
    }
  }
}

cudaError_t run_gemv_tc(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s, float* Y,
                        int ldy, int* err, cudaStream_t st) {
  const int mc = M < 8 ? M : 8;
  const int smem = mc * K * 2;
  static int attr_smem = 0;
  static std::map<int, int> per_sm;
  if (smem > attr_smem) {
    cudaError_t e = cudaFuncSetAttribute(k_mx_gemv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_smem = smem;
  }
  auto it = per_sm.find(smem);
  if (it == per_sm.end()) {
    int b = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_mx_gemv_tc, TV_T, smem);
    if (e != cudaSuccess) return e;
    it = per_sm.emplace(smem, b < 1 ? 1 : b).first;
  }
  const long long want = ((long long)N + 15) / 16;
  const long long cap = (long long)num_sms() * it->second;
  const int grid = (int)(want < cap ? want : cap);
  return launch(k_mx_gemv_tc, grid, TV_T, smem, st, M, N, K, X, ldx, q, s, Y, ldy, err);
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

int mx_gemv_splits(int N, int K) {
  int S = 1;
  while (S < 8 && (long long)N * S < 48LL * num_sms() && K % (2 * S * kMxBlock) == 0 && K / (2 * S) >= 512) S *= 2;
  return S;
}

cudaError_t launch_mx_gemv(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* s,
                           float* Y, int ldy, int* err, cudaStream_t st, int impl, int S, size_t part_stride) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kMxBlock || ((uintptr_t)q & 15)) return cudaErrorNotSupported;
  if (S < 1 || K % (S * kMxBlock) || (S > 1 && impl != 0 && impl != 1 && impl != 4)) return cudaErrorNotSupported;
  if (impl == 3) return launch_mx_gemm_tc(M, N, K, X, ldx, q, s, Y, ldy, 0, 1, err, st);
  // the mma.sync kernel only by request: measured slower at every 4B decode shape
  if (impl == 2) {
    if (K * 16 > GV_SMEM_CAP) return cudaErrorNotSupported;  // 8 staged f16 tokens
    return run_gemv_tc(M, N, K, X, ldx, q, s, Y, ldy, err, st);
  }
  // tokens per pass: the smallest power of two covering M, up to 8, within
  // the staged-activation budget
  int cap = GV_SMEM_CAP / ((K / S) * 4);
  if (cap < 1) return cudaErrorNotSupported;
  int MT = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  while (MT > cap) MT >>= 1;
  if ((impl == 4 || impl == 0) && M <= MT) {
    // the same arithmetic with the rows streamed by bulk copies, where it fits
    cudaError_t e = cudaErrorNotSupported;
    switch (MT) {
      case 1: e = run_gemv_ring<1>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride); break;
      case 2: e = run_gemv_ring<2>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride); break;
      case 4: e = run_gemv_ring<4>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride); break;
      default: e = run_gemv_ring<8>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride); break;
    }
    if (e != cudaErrorNotSupported) return e;
  }
  switch (MT) {
    case 1: return run_gemv<1>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride);
    case 2: return run_gemv<2>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride);
    case 4: return run_gemv<4>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride);
    default: return run_gemv<8>(M, N, K, X, ldx, q, s, Y, ldy, err, st, S, part_stride);
  }
}

}  // namespace dory

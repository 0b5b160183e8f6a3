// Block-scaled low-bit decode GEMM on the tensor cores, fed by TMA (tcgen05,
// sm_100a), for two weight formats:
//   MXFP8: E4M3 codes, one E8M0 scale per 32 weights of a row;
//   NVFP4: E2M1 codes (two per byte, the even k in the low nibble), one E4M3
//          scale per 16 weights of a row, times a per-tensor scale g.
//
// The codes stream through a deep ring of raw 128-row x 128-byte tiles (TMA,
// no swizzle), as the bf16 decode GEMM streams its weights.  Four converter
// warps turn each tile into the 128-byte-swizzled K-major f16 image the MMA
// reads (both formats convert to f16 exactly), and the bf16 activations into
// f16(x * 2^14) (exact for |x| < 4, else DEV_ERR_RANGE).  tcgen05.mma
// kind::f16 accumulates each scale block into its own TMEM columns, and four
// epilogue warps apply the block's scale with one FMA per token and keep the
// sums in registers.  Work units are (weight tile of 128 rows, token tile of
// 16, K split); a split's K range depends on (K, S) only and tokens are
// independent MMA columns, so a row's bits do not depend on M.
// Warps: 0 TMA producer, 1 MMA issuer, 2-5 epilogue, 6-9 converters.  Every
// wait is bounded; on a timeout the kernel sets DEV_ERR_TIMEOUT, drains its
// copies, frees TMEM and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "mxfp8.cuh"
#include "umma.cuh"

namespace dory {
namespace {

using namespace tc;

constexpr int BM = 128;  // weight rows per tile
constexpr int MT = 16;   // tokens per tile (MMA N)
constexpr int RAW_A = BM * 128;  // 16 KB of codes per chunk (128 bytes of every row)
constexpr int NTH = 320;
constexpr float kXScale = 16384.f;  // activations are staged as f16(x * 2^14)

// FMT 0: MXFP8, FMT 1: NVFP4
template <int FMT>
struct Fmt {
  static constexpr int CK = FMT == 0 ? 128 : 256;      // weights per row per chunk
  static constexpr int BW = FMT == 0 ? 32 : 16;        // weights per scale block
  static constexpr int NB = CK / BW;                   // blocks per chunk: 4 or 16
  static constexpr int SUB = CK / 64;                  // 64-column f16 sub-tiles: 2 or 4
  static constexpr int RAW_B = MT * CK * 2;            // bf16 activations of the chunk
  static constexpr int RAW_STAGE = RAW_A + RAW_B;
  static constexpr int CONV_A = BM * CK * 2;           // f16 weights
  static constexpr int CONV_B = MT * CK * 2;           // f16 activations
  static constexpr int CONV_STAGE = CONV_A + CONV_B;
  static constexpr int RS = FMT == 0 ? 7 : 3;          // raw ring
  static constexpr int CS = 2;                         // converted ring
  static constexpr int SLOT = NB * MT;                 // TMEM columns per chunk: 64 or 256
  static constexpr int TS = FMT == 0 ? 4 : 2;          // TMEM slots
  static constexpr int TMEM_COLS = TS * SLOT;          // 256 or 512
  static constexpr int SMEM = RS * RAW_STAGE + CS * CONV_STAGE + 1024 + 512;
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(TMEM_COLS <= 512, "tensor memory");
};

__host__ __device__ constexpr uint32_t idesc_f16(int m, int n) {
  // fp32 accumulator, A and B f16 (format 0), both K-major
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
  const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xFFu), __NV_E2M1);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// units: (weight tile, token tile, split); the split's chunk range depends on (chunks, S)
struct Units {
  int n_tiles, m_tiles, S, nch;
  __device__ __forceinline__ void decode(int u, int& nt, int& mt, int& s, int& c0, int& c1) const {
    s = u % S;
    const int t = u / S;
    mt = t % m_tiles;
    nt = t / m_tiles;
    c0 = s * nch / S;
    c1 = (s + 1) * nch / S;
  }
};

// The scale bytes of one chunk of a weight row: 4 (MXFP8) or 16 (NVFP4).
template <int FMT>
struct ChunkScales {
  uint32_t w[FMT == 0 ? 1 : 4];
};

template <int FMT>
__device__ __forceinline__ ChunkScales<FMT> load_scales(const uint8_t* srow, int c) {
  ChunkScales<FMT> r;
  if constexpr (FMT == 0) {
    r.w[0] = __ldg(reinterpret_cast<const uint32_t*>(srow + c * 4));
  } else {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(srow + c * 16));
    r.w[0] = v.x;
    r.w[1] = v.y;
    r.w[2] = v.z;
    r.w[3] = v.w;
  }
  return r;
}

// The scale of block b of a chunk (from its scale bytes), times 2^-14 for
// the staged activations.
template <int FMT>
__device__ __forceinline__ float block_scale(const ChunkScales<FMT>& cs, int b, float g) {
  const uint32_t byte = (cs.w[b >> 2] >> (8 * (b & 3))) & 0xFFu;
  if constexpr (FMT == 0) {
    const int e = (int)byte - 127 - 14;
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : ldexpf(1.f, e);
  } else {
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3);
    return __half2float(__half(h)) * g * (1.f / kXScale);
  }
}

// tcgen05.ld of 16 columns without the wait (the caller waits once for a group).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <int FMT>
__global__ void __launch_bounds__(NTH, 1)
    k_lowbit_gemm(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapX,
                  const uint8_t* __restrict__ scales, const float* __restrict__ gptr, int K, float* Y, int ldy,
                  size_t part_stride, int M, Units un, int* err) {
  using F = Fmt<FMT>;
  constexpr int RS = F::RS, CS = F::CS, TS = F::TS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* raw = smem;                          // [RS][RAW_STAGE]
  uint8_t* conv = smem + RS * F::RAW_STAGE;     // [CS][CONV_STAGE]
  uint64_t* bars = (uint64_t*)(conv + CS * F::CONV_STAGE);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + RS;
  uint64_t* conv_full = raw_empty + RS;
  uint64_t* conv_empty = conv_full + CS;
  uint64_t* tfull = conv_empty + CS;
  uint64_t* tempty = tfull + TS;
  uint64_t* mma_done = tempty + TS;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsb = K / F::BW;  // scale bytes per row

  if (threadIdx.x == 0) {
    for (int i = 0; i < RS; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 4);
    }
    for (int i = 0; i < CS; ++i) {
      mbar_init(&conv_full[i], 4);
      mbar_init(&conv_empty[i], 1);
    }
    for (int i = 0; i < TS; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(F::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int units = un.n_tiles * un.m_tiles * un.S;

  if (threadIdx.x == 0) pdl_trigger();
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer.  The codes do not depend on earlier
      // kernels: the first RS stages get their codes before the predecessor
      // grid is waited for, their activations after.
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      int u = blockIdx.x, nt = 0, mt = 0, s = 0, c = 0, c1 = 0;
      if (u < units) un.decode(u, nt, mt, s, c, c1);
      auto next = [&]() {
        if (++c >= c1) {
          u += gridDim.x;
          if (u < units) un.decode(u, nt, mt, s, c, c1);
        }
      };
      auto load_x = [&](uint8_t* dst, uint64_t* bar, int cc, int mm) {
#pragma unroll
        for (int q = 0; q < F::SUB; ++q)
          tma_load_2d(dst + RAW_A + q * (F::RAW_B / F::SUB), &mapX, bar, cc * F::CK + q * 64, mm * MT);
      };
      int pre_c[RS], pre_m[RS];
      int npre = 0;
      while (npre < RS && u < units) {
        mbar_expect_tx(&raw_full[npre], F::RAW_STAGE);
        tma_load_2d(raw + npre * F::RAW_STAGE, &mapQ, &raw_full[npre], c * 128, nt * BM);  // x in bytes
        pre_c[npre] = c;
        pre_m[npre++] = mt;
        next();
      }
      pdl_wait();
      for (int i = 0; i < npre; ++i) load_x(raw + i * F::RAW_STAGE, &raw_full[i], pre_c[i], pre_m[i]);
      issued = npre;
      stage = npre % RS;
      phase = npre == RS ? 1u : 0u;
      while (u < units) {
        if (!mbar_wait(&raw_empty[stage], phase ^ 1, abort_flag, err)) break;
        uint8_t* dst = raw + stage * F::RAW_STAGE;
        mbar_expect_tx(&raw_full[stage], F::RAW_STAGE);
        tma_load_2d(dst, &mapQ, &raw_full[stage], c * 128, nt * BM);
        load_x(dst, &raw_full[stage], c, mt);
        ++issued;
        if (++stage == RS) {
          stage = 0;
          phase ^= 1;
        }
        next();
      }
      // drain: every issued copy must land before this CTA may exit
      int st = stage;
      uint32_t ph = phase;
      for (int i = 0; i < RS && i < issued; ++i) {
        if (st == 0) {
          st = RS;
          ph ^= 1;
        }
        --st;
        mbar_wait_drain(&raw_full[st], ph);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: one TMEM slot (NB block accumulators) per chunk
      constexpr uint32_t IDESC = idesc_f16(BM, MT);
      int cst = 0, tsl = 0;
      uint32_t cph = 0, tph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int nt, mt, s, c0, c1;
        un.decode(u, nt, mt, s, c0, c1);
        for (int c = c0; c < c1; ++c) {
          if (!mbar_wait(&conv_full[cst], cph, abort_flag, err) || !mbar_wait(&tempty[tsl], tph ^ 1, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(conv + cst * F::CONV_STAGE), sb = sa + F::CONV_A;
#pragma unroll
          for (int b = 0; b < F::NB; ++b) {
            // block b covers columns b*BW .. b*BW + BW - 1: sub-tile (b*BW)/64, 16-column steps from there
            const int q = (b * F::BW) / 64, k0 = ((b * F::BW) % 64) / 16;
            const uint64_t ad = sw128_desc(sa + q * (F::CONV_A / F::SUB)), bd = sw128_desc(sb + q * (F::CONV_B / F::SUB));
#pragma unroll
            for (int k2 = 0; k2 < F::BW / 16; ++k2)
              umma(tmem_base + tsl * F::SLOT + b * MT, ad + 2 * (k0 + k2), bd + 2 * (k0 + k2), IDESC, k2);
          }
          umma_commit(&conv_empty[cst]);
          umma_commit(&tfull[tsl]);
          if (++cst == CS) {
            cst = 0;
            cph ^= 1;
          }
          if (++tsl == TS) {
            tsl = 0;
            tph ^= 1;
          }
        }
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else if (warp < 6) {
    // ---------------- epilogue: block accumulators -> scaled sums
    pdl_wait();
    const int lane_base = 32 * (warp & 3);
    const float g = FMT == 1 ? *gptr : 1.f;
    int tsl = 0;
    uint32_t tph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int nt, mt, s, c0, c1;
      un.decode(u, nt, mt, s, c0, c1);
      const int n = nt * BM + lane_base + lane;
      const uint8_t* srow = scales + (size_t)n * nsb;
      float acc[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[t] = 0.f;
      // the row's scale bytes are fetched kSA chunks ahead (a ring in
      // registers), so no chunk waits on a global load
      constexpr int kSA = 4;
      ChunkScales<FMT> ring[kSA];
#pragma unroll
      for (int j = 0; j < kSA; ++j)
        if (c0 + j < c1) ring[j] = load_scales<FMT>(srow, c0 + j);
      for (int c = c0; c < c1; c += kSA) {
#pragma unroll
        for (int j = 0; j < kSA; ++j) {
          if (c + j >= c1) break;
          const ChunkScales<FMT> cs = ring[j];
          if (c + j + kSA < c1) ring[j] = load_scales<FMT>(srow, c + j + kSA);
          if (!mbar_wait(&tfull[tsl], tph, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // the chunk's block accumulators, four blocks per wait
#pragma unroll
          for (int b0 = 0; b0 < F::NB; b0 += 4) {
            uint32_t v[4][16];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (b0 + q < F::NB)
                tmem_ld16_nowait(tmem_base + ((uint32_t)lane_base << 16) + tsl * F::SLOT + (b0 + q) * MT, v[q]);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (b0 + q >= F::NB) break;
              const float sc = block_scale<FMT>(cs, b0 + q, g);
#pragma unroll
              for (int t = 0; t < MT; ++t) acc[t] = __fmaf_rn(__uint_as_float(v[q][t]), sc, acc[t]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[tsl]);
          if (++tsl == TS) {
            tsl = 0;
            tph ^= 1;
          }
        }
        if (!ok) break;
      }
      if (!ok) break;
      float* out = Y + (size_t)s * part_stride + n;
#pragma unroll
      for (int t = 0; t < MT; ++t)
        if (mt * MT + t < M) out[(size_t)(mt * MT + t) * ldy] = acc[t];
    }
  } else {
    // ---------------- converters: raw codes -> f16 tiles (128-byte swizzle), bf16 x -> f16(x * 2^14)
    const int cw = warp - 6;
    int rst = 0, cst = 0;
    uint32_t rph = 0, cph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int nt, mt, s, c0, c1;
      un.decode(u, nt, mt, s, c0, c1);
      for (int c = c0; c < c1; ++c) {
        if (!mbar_wait(&raw_full[rst], rph, abort_flag, err) || !mbar_wait(&conv_empty[cst], cph ^ 1, abort_flag, err)) {
          ok = false;
          break;
        }
        const uint8_t* ra = raw + rst * F::RAW_STAGE;
        uint8_t* ca = conv + cst * F::CONV_STAGE;
        // A: this warp's 32 rows, 4 rows of 128 raw bytes per warp instruction;
        // lane j = l % 8 holds raw bytes 16j..16j+15 of its row
#pragma unroll 2
        for (int it = 0; it < 8; ++it) {
          const int r = 32 * cw + 4 * it + (lane >> 3), j = lane & 7;
          const uint4 w = *reinterpret_cast<const uint4*>(ra + r * 128 + j * 16);
          if constexpr (FMT == 0) {
            // 16 codes = columns 16j..16j+15: sub-tile j/4, 8-column chunks 2(j%4), 2(j%4)+1
            const uint4 lo = make_uint4(e4m3x2_f16x2(w.x), e4m3x2_f16x2(w.x >> 16), e4m3x2_f16x2(w.y),
                                        e4m3x2_f16x2(w.y >> 16));
            const uint4 hi = make_uint4(e4m3x2_f16x2(w.z), e4m3x2_f16x2(w.z >> 16), e4m3x2_f16x2(w.w),
                                        e4m3x2_f16x2(w.w >> 16));
            uint8_t* sub = ca + (j >> 2) * (F::CONV_A / F::SUB) + r * 128;
            const int ch = 2 * (j & 3);
            *reinterpret_cast<uint4*>(sub + ((ch ^ (r & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(sub + (((ch + 1) ^ (r & 7)) << 4)) = hi;
          } else {
            // 32 codes = columns 32j..32j+31: sub-tile j/2, 8-column chunks 4(j%2) .. 4(j%2)+3
            const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
            uint8_t* sub = ca + (j >> 1) * (F::CONV_A / F::SUB) + r * 128;
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // raw word i = 4 bytes = 8 codes = one 8-column chunk
              const uint4 o = make_uint4(e2m1x2_f16x2(wd[i]), e2m1x2_f16x2(wd[i] >> 8), e2m1x2_f16x2(wd[i] >> 16),
                                         e2m1x2_f16x2(wd[i] >> 24));
              const int ch = 4 * (j & 1) + i;
              *reinterpret_cast<uint4*>(sub + ((ch ^ (r & 7)) << 4)) = o;
            }
          }
        }
        // B: the swizzled bf16 tile, same chunk positions in f16
        bool bad = false;
#pragma unroll
        for (int i = 0; i < F::RAW_B / (16 * 128); ++i) {
          const int off = (cw * 32 + lane + 128 * i) * 16;
          const uint4 w = *reinterpret_cast<const uint4*>(ra + RAW_A + off);
          const uint32_t in[4] = {w.x, w.y, w.z, w.w};
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(in[q] << 16) * kXScale, b = __uint_as_float(in[q] & 0xFFFF0000u) * kXScale;
            bad |= !(fabsf(a) < 65504.f && fabsf(b) < 65504.f);
            const __half2 h = __floats2half2_rn(a, b);
            o[q] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(ca + F::CONV_A + off) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (bad) set_error(err, DEV_ERR_RANGE);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&raw_empty[rst]);
          mbar_arrive(&conv_full[cst]);
        }
        if (++rst == RS) {
          rst = 0;
          rph ^= 1;
        }
        if (++cst == CS) {
          cst = 0;
          cph ^= 1;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(F::TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeFn)p;
  }
  return fn;
}

int num_sms_tc() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// row_bytes: bytes of codes per weight row (K for MXFP8, K/2 for NVFP4)
template <int FMT>
cudaError_t run_lowbit(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* scales,
                       const float* g, float* Y, int ldy, size_t part_stride, int S, int* err, cudaStream_t st) {
  using F = Fmt<FMT>;
  const long long row_bytes = FMT == 0 ? K : K / 2;
  // the epilogue reads a chunk's scale bytes as one 4-byte (MXFP8) or 16-byte (NVFP4) word
  if (M < 1 || N % BM || K % F::CK || ((uintptr_t)q & 15) || ((uintptr_t)X & 15) || (ldx * 2) % 16 ||
      ((uintptr_t)scales & (FMT == 0 ? 3 : 15)))
    return cudaErrorNotSupported;
  EncodeFn fn = encode();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap mq, mx;
  {
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128, BM};
    cuuint32_t es[2] = {1, 1};
    if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    cuuint32_t box[2] = {64, MT};
    cuuint32_t es[2] = {1, 1};
    if (fn(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(X), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_lowbit_gemm<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int nch = K / F::CK;
  if (S < 1) S = 1;
  if (S > nch) S = nch;
  Units un{N / BM, (M + MT - 1) / MT, S, nch};
  const long long units = (long long)un.n_tiles * un.m_tiles * S;
  const int grid = (int)(units < num_sms_tc() ? units : num_sms_tc());
  return launch(k_lowbit_gemm<FMT>, grid, NTH, F::SMEM, st, mq, mx, scales, g, K, Y, ldy, part_stride, M, un, err);
}

}  // namespace

// Split count S in 1..min(8, chunks) with the shortest launch: units
// (tiles x S) run in ceil(units / SMs) rounds of 1/S of a tile's chunks each;
// ties go to the smaller S (fewer partial slices to add).  A count just above
// the SMs doubles the launch (160 units on 148 SMs: two rounds of one tile).
int lowbit_splits(int tiles, int nch) {
  if (tiles <= 0 || nch <= 0) return 1;
  const int sms = num_sms_tc();
  int best = 1;
  double best_t = 1e30;
  for (int S = 1; S <= 8 && S <= nch; ++S) {
    const double t = (double)((tiles * S + sms - 1) / sms) / S;
    if (t < best_t - 1e-9) {
      best_t = t;
      best = S;
    }
  }
  return best;
}

int mx_gemm_splits(int N, int K) { return lowbit_splits(N / BM, K / Fmt<0>::CK); }

int nv_gemm_splits(int N, int K) { return lowbit_splits(N / BM, K / Fmt<1>::CK); }

cudaError_t launch_mx_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* scales,
                              float* Y, int ldy, size_t part_stride, int S, int* err, cudaStream_t st) {
  return run_lowbit<0>(M, N, K, X, ldx, q, scales, nullptr, Y, ldy, part_stride, S, err, st);
}

cudaError_t launch_nv_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const uint8_t* q, const uint8_t* scales,
                              const float* g, float* Y, int ldy, size_t part_stride, int S, int* err,
                              cudaStream_t st) {
  if (!g) return cudaErrorNotSupported;
  return run_lowbit<1>(M, N, K, X, ldx, q, scales, g, Y, ldy, part_stride, S, err, st);
}

}  // namespace dory

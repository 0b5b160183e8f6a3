// bf16 GEMM on the sm_100a tensor cores: tcgen05.mma with fp32 accumulators
// in TMEM, operands staged in shared memory by TMA.
//
// Y[m, n] = sum_k X[m, k] W[n, k].  The weight matrix is the MMA's A operand
// (128-row tiles, K-major, 128-byte swizzle) and the tokens are the MMA's N
// dimension, so a decode step with one token still fills the 128-lane
// datapath with weights and the kernel streams W at HBM speed.
//
// A work unit is (128-row weight tile, token tile, K split).  Each CTA is
// persistent and takes units blockIdx.x, blockIdx.x + gridDim.x, ...:
//   warp 0 (one lane)  TMA producer: A and B tiles into a STAGES-deep ring
//   warp 1 (one lane)  MMA issuer: 4 K-steps of 16 per 64-wide k-block;
//                      accumulators double-buffered in TMEM
//   warps 2..5         epilogue: tcgen05.ld -> registers -> fp32 global
// Decode tiles use GN = 16 tokens per MMA instruction and loop over NG groups;
// the prefill tile uses one N = 256 instruction.
//
// Every mbarrier wait is bounded (about a second); on expiry the kernel sets
// the device error word, stops issuing work, waits (bounded) for its own
// copies in flight, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "addnorm.cuh"
#include "gemm_tc.cuh"
#include "umma.cuh"

namespace dory {

namespace {

using namespace tc;

constexpr int BK = 64;            // k elements per stage (128 bytes of bf16: one swizzle row)
constexpr int BM = 128;           // weight rows per tile (MMA M)
// Decode tiles: 64-column sub-tiles per stage and the shared-memory budget of
// the stage ring (a budget near 100 KB lets the next GEMM's CTA co-reside and
// prefetch its weights while this one drains).
constexpr int kDecodeKsub = 4;
constexpr int kDecodeBudget = 216 * 1024;

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// A TMA box of a 2-D tensor map, global -> L2 only.
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}

// Bytes at a 16-byte aligned address (a multiple of 16), global -> L2 only.
__device__ __forceinline__ void bulk_prefetch(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// KSUB 64-column sub-tiles per pipeline stage: a stage reads KSUB*128
// contiguous bytes of every weight row.
// GLU: a unit's A operand is two 128-row tiles of one matrix, rows
// [128 nt, +128) and [glu_rows + 128 nt, +128), with one accumulator each.
// PREP: the token operand is built in shared memory by the epilogue warps
// (see Prep) in a resident region of BSUB 64-column sub-tiles; stages then
// carry weights only.
template <int NG, int GN, int KSUB, int BUDGET = 216 * 1024, bool GLU = false, int PREP = 0, int BSUB = 0>
struct Tile {
  static constexpr int MT = NG * GN;                   // tokens per unit
  static constexpr int A_SUB = BM * BK * 2;            // 16 KB per sub-tile
  static constexpr int B_SUB = MT * BK * 2;
  static constexpr int NA = GLU ? 2 : 1;               // A tiles per unit
  static constexpr int A_BYTES = NA * KSUB * A_SUB;
  static constexpr int B_BYTES = PREP ? 0 : KSUB * B_SUB;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int B_RES = PREP ? BSUB * B_SUB : 0;  // resident token operand
  static constexpr int STAGES = (BUDGET - B_RES) / STAGE > 12 ? 12
                                : ((BUDGET - B_RES) / STAGE < 1 ? 1 : (BUDGET - B_RES) / STAGE);
  static constexpr int ACC = NA * MT;                  // TMEM columns per accumulator (pair)
  static constexpr int TMEM_COLS = 2 * ACC <= 32 ? 32 : 2 * ACC <= 64 ? 64 : 2 * ACC <= 128 ? 128 : 2 * ACC <= 256 ? 256 : 512;
  static constexpr int SMEM = STAGES * STAGE + B_RES + 1024 /*align*/ + 512 /*barriers*/;
};

// Units are (n tile, m tile, split).  Split boundaries are placed on groups
// of `gran` stages (KBg groups in all) so they fall on the same K columns
// whatever the stage width: a row's split-K grouping never depends on M.
struct UnitMap {
  int n_tiles, m_tiles, S, KBg, gran, units;
  __device__ __forceinline__ void decode(int u, int& nt, int& mt, int& s, int& kb0, int& kb1) const {
    s = u % S;
    int t = u / S;
    mt = t % m_tiles;
    nt = t / m_tiles;
    kb0 = (s * KBg / S) * gran;
    kb1 = ((s + 1) * KBg / S) * gran;
  }
};

// PACK: the weights are in the packed tile layout (see dory_pack_weight_bf16):
// 128 x 64 tiles stored as their 16 KB swizzled shared-memory image, tiles
// of one 128-row band consecutive along K, so a stage is one bulk copy.
//
// GLU (prefill, no split): the epilogue writes act[m, j] = silu(g) * u as
// bf16 (row stride ldy) from the pair of accumulators, where g and u are the
// products with weight rows j and glu_rows + j: the SwiGLU of a concatenated
// [gate; up] matrix, without its fp32 products ever reaching memory.
// The resident token operand of a PREP GEMM: the first CTA's units' K range
// as 64-column sub-tiles [lo, hi) (every CTA's units share one range when
// the host chose this path).
struct SubRange {
  int lo, hi;
};

__device__ __forceinline__ SubRange prep_range(const UnitMap& um, int ksub) {
  SubRange r{1 << 30, -1};
  for (int u = blockIdx.x; u < um.units; u += gridDim.x) {
    int nt, mt, s, kb0, kb1;
    um.decode(u, nt, mt, s, kb0, kb1);
    r.lo = min(r.lo, kb0 * ksub);
    r.hi = max(r.hi, kb1 * ksub);
  }
  return r;
}

__device__ __forceinline__ void bar_epi() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The operand stage (see Prep), run by the 128 epilogue threads (t = 0..127)
// into `breg`: sub-tile i of the region holds columns 64 (lo + i) .. + 63 of
// the MT token rows, 128-byte swizzled K-major (row m's 16-byte chunk c at
// m * 128 + (c ^ (m % 8)) * 16); rows >= M are zero.  K: the operand's width.
template <int PREP, int MT>
__device__ void prep_operand(const Prep& pp, int M, int K, SubRange rg, uint8_t* breg, float* red, int t) {
  const int nsub = rg.hi - rg.lo, c_lo = rg.lo * BK, c_hi = rg.hi * BK;
  // rows M..MT-1 of every sub-tile: bytes [M * 128, MT * 128)
  for (int i = t; i < nsub * (MT - M) * 8; i += 128) {
    const int sub = i / ((MT - M) * 8), off = i % ((MT - M) * 8);
    *reinterpret_cast<uint4*>(breg + sub * (MT * 128) + M * 128 + off * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  if constexpr (PREP == kPrepAddNorm) {
    // thread t runs virtual threads t + 128 j (j = 0..3): virtual warp
    // warp(t) + 4 j, the same lane
    for (int m = 0; m < M; ++m) {
      const float* hr = pp.h_in + (size_t)m * K;
      const float* yr = pp.y + (size_t)m * pp.ldy;
      float e[4][AN_CPT];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float ss = an_warp_tree(an_load(hr, yr, pp.S, pp.ps, K, t + 128 * j, e[j]));
        if ((t & 31) == 0) red[(t >> 5) + 4 * j] = ss;
      }
      bar_epi();
      const float inv = an_inv_from_warps(red);
      bar_epi();  // red is written again for the next row
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c = 0; c < AN_CPT; ++c) {
          const int i = t + 128 * j + c * AN_VT;
          if (i < K) {
            const float o = e[j][c] * inv;
            if (blockIdx.x == 0) pp.h_out[(size_t)m * K + i] = o;
            if (i >= c_lo && i < c_hi) {
              const int cc = i - c_lo, sub = cc / BK, ch = (cc % BK) / 8;
              *reinterpret_cast<bf16*>(breg + sub * (MT * 128) + m * 128 + ((ch ^ (m & 7)) << 4) + (cc % 8) * 2) =
                  __float2bfloat16_rn(o);
            }
          }
        }
    }
  } else {
    // SwiGLU: 16-byte chunks of 8 columns; gate columns j, up columns K + j
    const int nch = nsub * (BK / 8);
    for (int m = 0; m < M; ++m) {
      const float* yr = pp.y + (size_t)m * pp.ldy;
      for (int i = t; i < nch; i += 128) {
        const int col = c_lo + 8 * i;
        float g[8], u[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = u[e] = 0.f;
        for (int s = 0; s < pp.S; ++s) {
          const float4* gp = reinterpret_cast<const float4*>(yr + s * pp.ps + col);
          const float4* up = reinterpret_cast<const float4*>(yr + s * pp.ps + K + col);
          const float4 g0 = __ldcg(gp), g1 = __ldcg(gp + 1), u0 = __ldcg(up), u1 = __ldcg(up + 1);
          g[0] += g0.x; g[1] += g0.y; g[2] += g0.z; g[3] += g0.w;
          g[4] += g1.x; g[5] += g1.y; g[6] += g1.z; g[7] += g1.w;
          u[0] += u0.x; u[1] += u0.y; u[2] += u0.z; u[3] += u0.w;
          u[4] += u1.x; u[5] += u1.y; u[6] += u1.z; u[7] += u1.w;
        }
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a0 = g[2 * e] / (1.f + expf(-g[2 * e])) * u[2 * e];
          const float a1 = g[2 * e + 1] / (1.f + expf(-g[2 * e + 1])) * u[2 * e + 1];
          const __nv_bfloat162 p = __floats2bfloat162_rn(a0, a1);
          w[e] = *reinterpret_cast<const uint32_t*>(&p);
        }
        const int sub = i / (BK / 8), ch = i % (BK / 8);
        *reinterpret_cast<uint4*>(breg + sub * (MT * 128) + m * 128 + ((ch ^ (m & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  // generic-proxy writes -> visible to the tensor core's reads
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  bar_epi();
}

template <int NG, int GN, int KSUB, int BUDGET, bool PACK, bool GLU = false, int PREP = 0, int BSUB = 0>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, float* Y, int ldy,
              size_t part_stride, int M, UnitMap um, int* err, const uint8_t* Apack,
              int k_tiles, PfCtl pf, bf16* act, int glu_rows, Prep pp) {
  using TL = Tile<NG, GN, KSUB, BUDGET, GLU, PREP, BSUB>;
  constexpr int STAGES = TL::STAGES;
  auto load_a = [&](uint8_t* sa, uint64_t* bar, int nt, int kb, uint64_t pol) {
    if constexpr (PACK) {
      bulk_load(sa, Apack + ((size_t)nt * k_tiles + (size_t)kb * KSUB) * TL::A_SUB, TL::A_BYTES, bar, pol);
    } else {
#pragma unroll
      for (int q = 0; q < KSUB; ++q) tma_load_2d(sa + q * TL::A_SUB, &mapA, bar, (kb * KSUB + q) * BK, nt * BM, pol);
      if constexpr (GLU) {
#pragma unroll
        for (int q = 0; q < KSUB; ++q)
          tma_load_2d(sa + (KSUB + q) * TL::A_SUB, &mapA, bar, (kb * KSUB + q) * BK, glu_rows + nt * BM, pol);
      }
    }
  };
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* breg = smem + STAGES * TL::STAGE;  // PREP: resident token operand
  uint64_t* full = (uint64_t*)(breg + TL::B_RES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* b_ready = mma_done + 1;
  uint32_t* tmem_slot = (uint32_t*)(b_ready + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* red = (float*)(tmem_slot + 4);  // 16 floats (the operand stage's warp sums)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(mma_done, 1);
    mbar_init(b_ready, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    if (!PACK) asm volatile("prefetch.tensormap [%0];" ::"l"(&mapA) : "memory");
    if (!PREP) asm volatile("prefetch.tensormap [%0];" ::"l"(&mapB) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TL::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (threadIdx.x == 0) pdl_trigger();
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
      // (u, kb) items of this CTA in order
      int u = blockIdx.x, nt = 0, mt = 0, s = 0, kb = 0, kb1 = 0;
      if (u < um.units) um.decode(u, nt, mt, s, kb, kb1);
      auto next = [&]() {
        if (++kb >= kb1) {
          u += gridDim.x;
          if (u < um.units) um.decode(u, nt, mt, s, kb, kb1);
        }
      };
      // Weights do not depend on earlier kernels: fill the first stages with
      // A tiles before waiting for the predecessor grid, then add B.
      int pre_kb[STAGES], pre_mt[STAGES];
      int npre = 0;
      while (npre < STAGES && u < um.units) {
        uint8_t* sa = smem + npre * TL::STAGE;
        mbar_expect_tx(&full[npre], TL::STAGE);
        load_a(sa, &full[npre], nt, kb, pol_w);
        pre_kb[npre] = kb;
        pre_mt[npre] = mt;
        ++npre;
        next();
      }
      if (pf.own > 0) {
        // ask L2 for the CTA's next weight tiles while the previous kernel
        // still runs (the ring above holds the first STAGES of them)
        int u2 = u, nt2 = nt, mt2 = mt, s2 = s, kb2 = kb, kb12 = kb1;
        for (int c = 0; c < pf.own && u2 < um.units; ++c) {
          if constexpr (PACK) {
            bulk_prefetch(Apack + ((size_t)nt2 * k_tiles + (size_t)kb2 * KSUB) * TL::A_SUB, TL::A_BYTES);
          } else {
#pragma unroll
            for (int q = 0; q < KSUB; ++q) tma_prefetch_2d(&mapA, (kb2 * KSUB + q) * BK, nt2 * BM);
            if constexpr (GLU) {
#pragma unroll
              for (int q = 0; q < KSUB; ++q) tma_prefetch_2d(&mapA, (kb2 * KSUB + q) * BK, glu_rows + nt2 * BM);
            }
          }
          if (++kb2 >= kb12) {
            u2 += gridDim.x;
            if (u2 < um.units) um.decode(u2, nt2, mt2, s2, kb2, kb12);
          }
        }
      }
      if constexpr (!PREP) {
        pdl_wait();
        for (int i = 0; i < npre; ++i)
#pragma unroll
          for (int q = 0; q < KSUB; ++q)
            tma_load_2d(smem + i * TL::STAGE + TL::A_BYTES + q * TL::B_SUB, &mapB, &full[i],
                        (pre_kb[i] * KSUB + q) * BK, pre_mt[i] * TL::MT, pol_x);
      }
      int stage = npre % STAGES, issued = npre;
      uint32_t phase = npre == STAGES ? 1u : 0u;
      while (u < um.units) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err)) break;
        ++issued;
        uint8_t* sa = smem + stage * TL::STAGE;
        mbar_expect_tx(&full[stage], TL::STAGE);
        load_a(sa, &full[stage], nt, kb, pol_w);
        if constexpr (!PREP) {
#pragma unroll
          for (int q = 0; q < KSUB; ++q)
            tma_load_2d(sa + TL::A_BYTES + q * TL::B_SUB, &mapB, &full[stage], (kb * KSUB + q) * BK, mt * TL::MT,
                        pol_x);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
        next();
      }
      // drain: every issued copy must land before this CTA may exit.  The
      // last min(issued, STAGES) stages are the ones that can be in flight;
      // walk back over them and wait for their fill (bounded).
      int st = stage;
      uint32_t ph = phase;
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (st == 0) {
          st = STAGES;
          ph ^= 1;
        }
        --st;
        mbar_wait_drain(&full[st], ph);
      }
    }
    __syncwarp();
    if (!pf.early && pf.lo < pf.hi && !*abort_flag) l2_look_ahead(pf, lane, 32);
  } else if (warp == 1) {
    if (pf.early && pf.lo < pf.hi) l2_look_ahead(pf, lane, 32);
    pdl_wait();
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t IDESC = idesc_bf16(BM, GN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int sub_lo = 0;
      if constexpr (PREP != 0) {
        sub_lo = prep_range(um, KSUB).lo;
        ok = mbar_wait(b_ready, 0, abort_flag, err) && !*abort_flag;
        tc_fence_after();
      }
      for (int u = blockIdx.x; u < um.units && ok; u += gridDim.x) {
        int nt, mt, s, kb0, kb1;
        um.decode(u, nt, mt, s, kb0, kb1);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * TL::ACC;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * TL::STAGE);
#pragma unroll
          for (int q = 0; q < KSUB; ++q) {
            const uint64_t adesc = sw128_desc(sa + q * TL::A_SUB);
            const uint64_t bdesc =
                PREP ? sw128_desc(smem_u32(breg) + (uint32_t)((kb * KSUB + q - sub_lo) * TL::B_SUB))
                     : sw128_desc(sa + TL::A_BYTES + q * TL::B_SUB);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
#pragma unroll
              for (int g = 0; g < NG; ++g) {
                // +32 bytes per K-step of 16 inside the swizzled row; group g
                // starts GN rows (GN * 128 bytes) further into the B tile
                umma(d0 + g * GN, adesc + 2 * kk, bdesc + 2 * kk + (uint64_t)(g * GN * 128 >> 4), IDESC,
                     (kb > kb0 || q > 0 || kk > 0) ? 1u : 0u);
                if constexpr (GLU)  // the up tile: KSUB sub-tiles further, its accumulator MT columns on
                  umma(d0 + TL::MT + g * GN, adesc + 2 * kk + (uint64_t)(KSUB * TL::A_SUB >> 4),
                       bdesc + 2 * kk + (uint64_t)(g * GN * 128 >> 4), IDESC, (kb > kb0 || q > 0 || kk > 0) ? 1u : 0u);
              }
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // all MMAs issued by this thread have completed once mma_done fires
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ---------------- epilogue: warps 2..5 own TMEM lanes 32*(warp%4) ..
    pdl_wait();
    if constexpr (PREP != 0) {
      const int t = threadIdx.x - 64;
      const SubRange rg = prep_range(um, KSUB);
      if (rg.hi - rg.lo > BSUB || rg.hi <= rg.lo) {
        // the host sizes the region for every CTA; this cannot happen
        if (t == 0) {
          set_error(err, DEV_ERR_RANGE);
          *abort_flag = 1;
        }
      } else {
        prep_operand<PREP, TL::MT>(pp, M, k_tiles * BK, rg, breg, red, t);
      }
      if (t == 0) mbar_arrive(b_ready);
    }
    const int lane_base = 32 * (warp & 3);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < um.units; u += gridDim.x) {
      int nt, mt, s, kb0, kb1;
      um.decode(u, nt, mt, s, kb0, kb1);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, err)) break;
      tc_fence_after();
      const int n = nt * BM + lane_base + lane;
      float* out = Y + (size_t)s * part_stride + n;
      const int m_base = mt * TL::MT;
#pragma unroll 1
      for (int c = 0; c < TL::MT; c += 16) {
        if (m_base + c >= M) break;
        float v[16];
        tmem_ld16(tmem_base + ((uint32_t)lane_base << 16) + acc * TL::ACC + c, v);
        if constexpr (GLU) {
          float w[16];
          tmem_ld16(tmem_base + ((uint32_t)lane_base << 16) + acc * TL::ACC + TL::MT + c, w);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m_base + c + j;
            if (m < M) act[(size_t)m * ldy + n] = __float2bfloat16_rn(v[j] / (1.f + expf(-v[j])) * w[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m_base + c + j;
            if (m < M) out[(size_t)m * ldy] = v[j];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TL::TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// 2-D bf16 tensor map over rows x cols (row stride in elements), box of
// BK columns x box_rows rows, 128-byte swizzle; rows past the end read zeros.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t stride, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct MapKey {
  const void* p;
  int rows, cols;
  bool operator==(const MapKey& o) const { return p == o.p && rows == o.rows && cols == o.cols; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const { return std::hash<const void*>()(k.p) ^ ((size_t)k.rows << 20) ^ k.cols; }
};

std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_wmaps;

bool weight_map(CUtensorMap* m, const void* W, int N, int K) {
  std::lock_guard<std::mutex> lk(g_map_mu);
  MapKey key{W, N, K};
  auto it = g_wmaps.find(key);
  if (it != g_wmaps.end()) {
    *m = it->second;
    return true;
  }
  if (!make_map(m, W, N, K, K, BM)) return false;
  g_wmaps.emplace(key, *m);
  return true;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int NG, int GN, int KSUB, int BUDGET = kDecodeBudget, bool PACK = false, bool GLU = false, int PREP = 0,
          int BSUB = 0>
cudaError_t run(const CUtensorMap& ma, const bf16* X, int ldx, int M, int K, float* Y, int ldy, size_t ps,
                UnitMap um, int* err, cudaStream_t st, const void* Apack = nullptr,
                const PfCtl& pf = PfCtl{}, bf16* act = nullptr, int glu_rows = 0, const Prep& pp = Prep{}) {
  using TL = Tile<NG, GN, KSUB, BUDGET, GLU, PREP, BSUB>;
  auto kern = k_gemm_tc<NG, GN, KSUB, BUDGET, PACK, GLU, PREP, BSUB>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TL::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap mb;
  if (PREP)
    memset(&mb, 0, sizeof mb);  // the token operand is built in shared memory
  else if (!make_map(&mb, X, M, K, ldx, TL::MT))
    return cudaErrorInvalidValue;
  int grid = um.units < sm_count() ? um.units : sm_count();
  return launch(kern, dim3(grid), dim3(192), TL::SMEM, st, ma, mb, Y, ldy, ps, M, um, err, (const uint8_t*)Apack,
                K / BK, pf, act, glu_rows, pp);
}

// Split factor for the decode tiles: chosen from (N, K, batch) only, never
// from M, so a row's accumulation grouping is the same at every M.  Units are
// dealt round-robin to one CTA per SM; the model charges the larger of the
// whole GEMM at HBM speed and the busiest CTA at one SM's streaming rate,
// plus the partial sums' HBM traffic.
// cap > 0: prefer splits whose units fit in `cap` CTAs (see launch_gemm_tc).
int choose_split(int N, int K, int batch, int kstages, int cap = 0) {
  const double hbm = 6.5e12, sm_bw = 5.5e10;
  const int tiles = N / BM, sms = sm_count();
  if (cap > 0 && tiles <= cap) {
    int S = 1;
    while (S + 1 <= kMaxSplitK && S + 1 <= kstages && tiles * (S + 1) <= cap) ++S;
    return S;
  }
  // partial-sum traffic is charged for one row per sequence (plain decode);
  // a speculative verify chunk has gamma + 1 rows per sequence and pays more
  const double rows = batch;
  const double stage_bytes = (double)BM * (K / kstages) * 2;
  int best = 1;
  double best_t = 1e30;
  for (int S = 1; S <= kMaxSplitK && S <= kstages; ++S) {
    const int U = tiles * S;
    // busiest CTA: ceil(U / sms) units, the largest of which has ceil(KB / S) stages
    const int per_cta = (U + sms - 1) / sms;
    const double busiest = per_cta * (double)((kstages + S - 1) / S) * stage_bytes;
    double t = fmax(tiles * (double)kstages * stage_bytes / hbm, busiest / sm_bw);
    t += S * rows * N * 8.0 / hbm;
    if (t < best_t * 0.98) {
      best_t = t;
      best = S;
    }
  }
  return best;
}

__global__ void k_pack_weight(const bf16* __restrict__ src, uint8_t* __restrict__ dst, int N, int K) {
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;  // 16-byte chunk of the source
  if (i >= (size_t)N * K / 8) return;
  const int kc = K / 8;
  const int n = (int)(i / kc), c8 = (int)(i % kc);
  const int nt = n / BM, r = n % BM, kt = c8 / 8, c = c8 % 8;
  const size_t off = ((size_t)nt * (K / BK) + kt) * (BM * BK * 2) + r * 128 + ((c ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src + (size_t)n * K + (size_t)c8 * 8);
}

}  // namespace

cudaError_t launch_gemm_glu(int M, int dff, int K, const bf16* X, int ldx, const bf16* Wgu, bf16* act,
                            int* err, cudaStream_t st) {
  if (M <= 0 || dff % BM || K % BK || ldx % 8 || ((uintptr_t)X & 15) || ((uintptr_t)Wgu & 15))
    return cudaErrorNotSupported;
  CUtensorMap ma;
  if (!weight_map(&ma, Wgu, 2 * dff, K)) return cudaErrorNotSupported;
  // 128 x 128 token tiles: the gate/up accumulator pair fills 256 TMEM
  // columns, two pairs double-buffer the epilogue
  UnitMap um;
  um.n_tiles = dff / BM;
  um.KBg = K / BK;
  um.gran = 1;
  um.S = 1;
  um.m_tiles = (M + 127) / 128;
  um.units = um.n_tiles * um.m_tiles;
  return run<1, 128, 1, 200 * 1024, false, true>(ma, X, ldx, M, K, nullptr, dff, 0, um, err, st, nullptr,
                                                 PfCtl{}, act, dff);
}

cudaError_t launch_pack_weight(const bf16* W, void* dst, int N, int K, cudaStream_t st) {
  if (N % BM || K % BK || ((uintptr_t)W & 15) || ((uintptr_t)dst & 15)) return cudaErrorInvalidValue;
  const size_t chunks = (size_t)N * K / 8;
  k_pack_weight<<<(unsigned)((chunks + 255) / 256), 256, 0, st>>>(W, (uint8_t*)dst, N, K);
  return cudaGetLastError();
}

// Largest 64-column sub-tile range one CTA's units span (the resident token
// operand of an operand-stage GEMM), for a grid of min(units, SMs) CTAs.
static int prep_span(const UnitMap& um, int ksub) {
  const int grid = um.units < sm_count() ? um.units : sm_count();
  int span = 0;
  for (int b = 0; b < grid; ++b) {
    int lo = 1 << 30, hi = -1;
    for (int u = b; u < um.units; u += grid) {
      const int s = u % um.S;
      lo = std::min(lo, (s * um.KBg / um.S) * um.gran * ksub);
      hi = std::max(hi, ((s + 1) * um.KBg / um.S) * um.gran * ksub);
    }
    span = std::max(span, hi - lo);
  }
  return span;
}

// Decode GEMM with an operand stage: 16-token tiles, 2 sub-tiles per stage,
// the resident operand region sized for the widest CTA range.
static cudaError_t run_prep(const CUtensorMap& ma, int M, int K, float* Y, int ldy, size_t ps, UnitMap um, int* err,
                     cudaStream_t st, const PfCtl& pf, const Prep& pp) {
  constexpr int KS = 2;
  const int span = prep_span(um, KS);
#define DORY_PREP(P, B)                                                                                       \
  if (pp.mode == P && span <= B)                                                                             \
  return run<1, 16, KS, kDecodeBudget, false, false, P, B>(ma, nullptr, 0, M, K, Y, ldy, ps, um, err, st, nullptr, \
                                                           pf, nullptr, 0, pp)
  DORY_PREP(kPrepAddNorm, 8);
  DORY_PREP(kPrepAddNorm, 24);
  DORY_PREP(kPrepAddNorm, 40);
  DORY_PREP(kPrepSwiglu, 8);
  DORY_PREP(kPrepSwiglu, 24);
  DORY_PREP(kPrepSwiglu, 40);
#undef DORY_PREP
  return cudaErrorNotSupported;
}

bool gemm_tc_prep_ok(int M, int N, int K, int batch, const Prep& p) {
  if (p.mode == kPrepNone || M < 1 || M > 16 || N % BM || K % (4 * BK) || p.S < 1 || p.S > AN_MAXS || p.ldy % 4 ||
      p.ps % 4 || ((uintptr_t)p.y & 15))
    return false;
  if (p.mode == kPrepAddNorm && (K > AN_CPT * AN_VT || p.h_in == p.h_out ||
                                 ((uintptr_t)p.h_in & 15) || ((uintptr_t)p.h_out & 15) || p.ldy < K))
    return false;
  if (p.mode == kPrepSwiglu && p.ldy < 2 * K) return false;
  UnitMap um;
  um.n_tiles = N / BM;
  um.KBg = K / (4 * BK);
  um.gran = 2;
  um.S = choose_split(N, K, batch, um.KBg);
  if (um.S > um.KBg) return false;
  um.m_tiles = 1;
  um.units = um.n_tiles * um.S;
  return prep_span(um, 2) <= 40;
}

cudaError_t launch_gemm_tc(int M, int N, int K, const bf16* X, int ldx, const bf16* W, float* Y, int ldy,
                           size_t part_rows, int* err, int batch, bool invariant, int* S_out, size_t* ps_out,
                           cudaStream_t st, int variant, bool packed, const PfCtl* pf, const Prep* prep,
                           int cta_cap) {
  *S_out = 1;
  *ps_out = 0;
  const bool staged = prep && prep->mode != kPrepNone;
  if (staged) {
    // the operand stage: decode tiles of one 16-token group, weights by TMA
    if (!invariant || packed || variant != 0 || (size_t)M > part_rows || ((uintptr_t)W & 15) ||
        !gemm_tc_prep_ok(M, N, K, batch, *prep))
      return cudaErrorNotSupported;
  } else if (M <= 0 || N % BM || K % BK || ldx % 8 || (size_t)M > part_rows || ((uintptr_t)X & 15) ||
             ((uintptr_t)W & 15)) {
    return cudaErrorNotSupported;
  }
  CUtensorMap ma;
  if (packed)
    memset(&ma, 0, sizeof ma);
  else if (!weight_map(&ma, W, N, K))
    return cudaErrorNotSupported;
  UnitMap um;
  um.n_tiles = N / BM;
  if (invariant) {
    // decode / verify: 16-token MMA groups, split chosen from (N, K, batch).
    // Stages span 4 sub-tiles (512 contiguous bytes per weight row) when K
    // allows; variant 1 forces one sub-tile per stage.
    int NG = M <= 16 ? 1 : M <= 32 ? 2 : M <= 64 ? 4 : 8;
    const bool g256 = K % (4 * BK) == 0;  // split on 256-column groups
    const int ksub = (variant == 1 || !g256) ? 1 : (NG >= 8 ? 1 : (NG >= 2 ? 2 : kDecodeKsub));
    um.KBg = g256 ? K / (4 * BK) : K / BK;
    um.gran = g256 ? 4 / (staged ? 2 : ksub) : 1;
    const int S = choose_split(N, K, batch, um.KBg, staged ? 0 : cta_cap);
    if (S > um.KBg) return cudaErrorNotSupported;
    const size_t ps = part_rows * (size_t)ldy;
    um.S = S;
    const int MT = 16 * NG;
    um.m_tiles = (M + MT - 1) / MT;
    um.units = um.n_tiles * um.m_tiles * S;
    const PfCtl pfc = pf ? *pf : PfCtl{};
    if (staged) {
      const cudaError_t e = run_prep(ma, M, K, Y, ldy, ps, um, err, st, pfc, *prep);
      if (e == cudaSuccess) {
        *S_out = S;
        *ps_out = ps;
      }
      return e;
    }
    *S_out = S;
    *ps_out = ps;
#define DORY_RUN(NGV, KS)                                                                                 \
  return packed ? run<NGV, 16, KS, kDecodeBudget, true>(ma, X, ldx, M, K, Y, ldy, ps, um, err, st, W, pfc) \
                : run<NGV, 16, KS>(ma, X, ldx, M, K, Y, ldy, ps, um, err, st, nullptr, pfc)
    if (NG == 1) {
      if (ksub == 4) DORY_RUN(1, 4);
      if (ksub == 2) DORY_RUN(1, 2);
      DORY_RUN(1, 1);
    }
    if (NG == 2) {
      if (ksub == 2) DORY_RUN(2, 2);
      DORY_RUN(2, 1);
    }
    if (NG == 4) {
      if (ksub == 2) DORY_RUN(4, 2);
      DORY_RUN(4, 1);
    }
    DORY_RUN(8, 1);
#undef DORY_RUN
  }
  // prefill: 128 x 256 tiles, no split
  um.KBg = K / BK;
  um.gran = 1;
  um.S = 1;
  um.m_tiles = (M + 255) / 256;
  um.units = um.n_tiles * um.m_tiles;
  if (packed) return run<1, 256, 1, 200 * 1024, true>(ma, X, ldx, M, K, Y, ldy, 0, um, err, st, W);
  return run<1, 256, 1, 200 * 1024>(ma, X, ldx, M, K, Y, ldy, 0, um, err, st);
}

}  // namespace dory

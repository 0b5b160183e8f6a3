// Prefill attention, warp-specialised for the 5th-generation tensor cores
// (bf16, head_dim 128).  Each CTA runs two query slots of 128 rows that share
// one key/value stream: two query heads of one KV group on the same rows, or
// one head on two consecutive row tiles of the same sequence.
//
// What is computed: causal attention in sliding-window and full layers,
// three of the first to one of the second (Dory1.0-4B digest,
// onedev.kr/papers/1692, "How it works"); under last-loop caching (same
// digest, "Premises & limits") a recurrent-block query of loop t sees the
// loop-t keys of its own chunk and the final-loop keys cached by earlier
// calls.  The pages give neither the window rule nor the head layout; this
// library reads them as keys p - W < j <= p and as groups of query heads
// sharing one K/V head (20 query heads over 4 K/V heads at the 4B shape).
//
//   warps 0-3  softmax of slot 0, one query row per thread (= TMEM lane)
//   warps 4-7  softmax of slot 1
//   warp 8     allocates TMEM; one lane issues every MMA and commit
//   warp 9     loader: Q once, then K and V tiles of 128 keys into a
//              two-stage ring, by TMA when a tile is one run of rows of the
//              chunk scratch or of the cache, else by cp.async row by row
//   warps 10-11 idle (they complete the third warpgroup)
// The CTA launches with 168 registers a thread; the third warpgroup gives
// back all but 72 and the softmax warpgroups take them (216 each), enough to
// hold a row of S.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Per key tile j the MMA lane issues, for each slot q in turn,
//   O_q += P_q(j) V(j)      (P_q from TMEM, written over the first 64
//                            columns of S_q by the softmax as bf16 pairs)
//   S_q(j+1) = Q_q K(j+1)^T
// so one slot's softmax runs while the tensor core works on the other's
// products.  The commit after S_q(j+1) also covers O_q += P_q(j): when the
// softmax sees S_q(j+1) the slot's O is complete up to tile j and may be
// rescaled.  V stays as loaded (keys x head dims); the P V product reads it
// as an MN-major operand, so nothing is transposed.
//
// Softmax in base 2 (Q is pre-scaled by log2(e)/sqrt(head_dim)) with the
// lazy running maximum of the single-tile kernel: O and the row sum are
// rescaled only when a row maximum grows by more than 8.
//
// Every mbarrier wait is bounded; on expiry the CTA sets the device error
// word, every role stops, the loader waits (bounded) for its copies in flight
// and the MMA lane for its products, and TMEM is freed.
#include <cuda.h>
#include <climits>
#include <float.h>

#include <algorithm>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "attn_prefill.cuh"
#include "umma.cuh"

namespace dory {

namespace {

using namespace tc;

constexpr int HDT = 128;               // head dimensions
constexpr int TQ = 128;                // query rows per slot
constexpr int TK = 128;                // keys per tile
constexpr int NS = 2;                  // K/V ring stages
constexpr int NTH = 384;               // 12 warps, three warpgroups
constexpr int REG_SOFTMAX = 216, REG_OTHER = 72;  // 2 x 128 x 216 + 128 x 72 = 384 x 168
static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_OTHER <= NTH * 168, "register split exceeds the launch's registers");
constexpr int PANEL = 128 * 128;       // 64 head dims x 128 rows, bytes
constexpr int TILE = 2 * PANEL;        // one Q, K or V tile, bytes
constexpr float kLazy = 8.f;

constexpr int Q_OFF = 0;                       // 2 slots
constexpr int K_OFF = Q_OFF + 2 * TILE;        // NS stages
constexpr int V_OFF = K_OFF + NS * TILE;       // NS stages
constexpr int BAR_OFF = V_OFF + NS * TILE;     // mbarriers, TMEM slot, flags
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
constexpr int TMEM_COLS = 512;

__device__ __forceinline__ uint32_t sw(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 32 consecutive TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%"
      "18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D (TMEM) (+)= A (TMEM, M x 16 bf16 as 8 columns of pairs) * B (shared memory descriptor).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Shared-memory descriptor of an MN-major operand, 128-byte swizzle: rows of
// 64 elements (128 B) along N, consecutive K rows 128 B apart, 8-row groups
// 1024 B apart (stride offset), 64-element N panels `panel` bytes apart
// (leading offset).
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr, uint32_t panel) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)((panel >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Packed fp32 pairs (one instruction for two lanes of arithmetic):
// (x, y) = (a0 - b, a1 - b) and (x, y) += (a0, a1).
__device__ __forceinline__ void sub2(float& x, float& y, float a0, float a1, float b) {
  asm("{.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\tsub.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(x), "=f"(y)
      : "f"(a0), "f"(a1), "f"(b));
}
__device__ __forceinline__ void add2(float& x, float& y, float a0, float a1) {
  asm("{.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tadd.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(x), "=f"(y)
      : "f"(x), "f"(y), "f"(a0), "f"(a1));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Maximum of a row of 128 values held as bits, by three-input maxima.
__device__ __forceinline__ float row_max(const uint32_t (&r)[128]) {
  float m[43];
#pragma unroll
  for (int i = 0; i < 42; ++i)
    m[i] = max3(__uint_as_float(r[3 * i]), __uint_as_float(r[3 * i + 1]), __uint_as_float(r[3 * i + 2]));
  m[42] = fmaxf(__uint_as_float(r[126]), __uint_as_float(r[127]));
  float n[15];
#pragma unroll
  for (int i = 0; i < 14; ++i) n[i] = max3(m[3 * i], m[3 * i + 1], m[3 * i + 2]);
  n[14] = m[42];
  float p[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) p[i] = max3(n[3 * i], n[3 * i + 1], n[3 * i + 2]);
  return fmaxf(max3(p[0], p[1], p[2]), fmaxf(p[3], p[4]));
}

// A bounded wait taken by every lane of a warp, with one outcome for all of
// them (the warp-wide TMEM accesses and __syncwarp that follow need every lane).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err) {
  const bool ok = mbar_wait(bar, parity, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

constexpr uint32_t kIdescS = idesc_bf16(TQ, TK);                // Q K^T: both K-major
constexpr uint32_t kIdescO = idesc_bf16(TQ, HDT) | (1u << 16);  // P V: B (V) MN-major

// Per-slot geometry shared by every role (all computed from the row
// metadata, so each role takes the same decisions).
struct Slot {
  int r0, nrows, head, pf, pl, a, b;  // a..b: key tiles this slot reads (relative to kt0)
};

// 12 warps: three share a scheduler, whose 16K registers cap a thread at 168
// at launch.
__global__ void __launch_bounds__(NTH, 1)
    k_attn_prefill_ws(int KV, int G, const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_ks, const __grid_constant__ CUtensorMap map_vs,
                      const __grid_constant__ CUtensorMap map_kc, const __grid_constant__ CUtensorMap map_vc,
                      const bf16* __restrict__ kscr, const bf16* __restrict__ vscr, KVView kv, RowMeta m,
                      const int2* __restrict__ tiles, const int4* __restrict__ items, bf16* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = (uint64_t*)(smem + BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;            // [NS]
  uint64_t* v_full = k_full + NS;         // [NS]
  uint64_t* k_empty = v_full + NS;        // [NS]
  uint64_t* v_empty = k_empty + NS;       // [NS]
  uint64_t* s_full = v_empty + NS;        // [2]
  uint64_t* p_full = s_full + 2;          // [2]
  uint64_t* o_full = p_full + 2;
  uint32_t* tmem_slot = (uint32_t*)(o_full + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], TQ);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait();  // queries, chunk keys and row metadata come from earlier kernels
  pdl_trigger();

  // ---- the work item: one or two slots of one KV group and one sequence
  const int4 it = items[blockIdx.x];
  const int nslot = it.z >= 0 ? 2 : 1;
  const int H = KV * G, qd = H * HDT;
  const int g = it.y / G;
  Slot sl[2];
  int lo_t = INT_MAX, hi_t = 0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int2 tl = tiles[q == 0 ? it.x : (nslot == 2 ? it.z : it.x)];
    Slot& s = sl[q];
    s.r0 = tl.x;
    s.nrows = tl.y - tl.x;
    s.head = q == 0 ? it.y : it.w;
    s.pf = m.pos[tl.x];
    s.pl = m.pos[tl.y - 1];
    const int lo = kv.window > 0 ? max(0, s.pf - kv.window + 1) : 0;
    s.a = lo / TK;
    s.b = s.pl / TK;
    if (q < nslot) {
      lo_t = min(lo_t, s.a);
      hi_t = max(hi_t, s.b);
    }
  }
  const int n_tiles = hi_t - lo_t + 1;
  const int kt0 = lo_t * TK;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    sl[q].a -= lo_t;
    sl[q].b -= lo_t;
  }
  const int r_ref = sl[0].r0;
  const int seq = m.seq[r_ref], p0 = m.p0[r_ref], base = m.base[r_ref];
  const int k_last = max(sl[0].pl, nslot == 2 ? sl[1].pl : 0);  // last key position any slot reads

  if (warp >= 8) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_OTHER));
   if (warp == 9) {
    // ------------------------------------------------------------ loader
    const bf16* Kc = (const bf16*)kv.K;
    const bf16* Vc = (const bf16*)kv.V;
    const int page = kv.pt ? (1 << kv.page_shift) : 0;
    if (lane == 0) {
      mbar_expect_tx(q_full, (uint32_t)(nslot * TILE));
#pragma unroll
      for (int q = 0; q < 2; ++q)
        if (q < nslot)
          for (int p = 0; p < 2; ++p)
            tma2d(sb + Q_OFF + q * TILE + p * PANEL, &map_q, q_full, sl[q].head * HDT + p * 64, sl[q].r0);
    }
    int issued = 0;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int st = j % NS, use = j / NS;
      if (j >= NS) {
        ok = warp_wait(&k_empty[st], (use + 1) & 1, abort_flag, kv.err) &&
             warp_wait(&v_empty[st], (use + 1) & 1, abort_flag, kv.err);
        if (!ok) break;
      }
      const int kt = kt0 + j * TK;
      const uint32_t dk = sb + K_OFF + st * TILE, dv = sb + V_OFF + st * TILE;
      // one run of rows: the chunk scratch, or the cache without a ring wrap
      // or page change inside the tile
      const bool scr = kt >= p0;
      const bool cache_run = !scr && kt + TK - 1 < p0 &&
                             (kv.pt ? page >= TK : (kt % kv.cap) + TK <= kv.cap);
      if (scr || cache_run) {
        if (lane == 0) {
          const CUtensorMap* mk = scr ? &map_ks : &map_kc;
          const CUtensorMap* mv = scr ? &map_vs : &map_vc;
          const int y = scr ? base + (kt - p0) : (int)kv_row(kv, seq, KV, g, kt);
          const int x0 = scr ? g * HDT : 0;
          mbar_expect_tx(&k_full[st], TILE);
          tma2d(dk, mk, &k_full[st], x0, y);
          tma2d(dk + PANEL, mk, &k_full[st], x0 + 64, y);
          mbar_expect_tx(&v_full[st], TILE);
          tma2d(dv, mv, &v_full[st], x0, y);
          tma2d(dv + PANEL, mv, &v_full[st], x0 + 64, y);
        }
      } else {
        // row by row: positions past the last key any slot reads are zero
        const int kvd = KV * HDT;
        for (int i = lane; i < TK * 16; i += 32) {
          const int row = i >> 4, c = i & 15;
          const int jp = kt + row;
          const bool valid = jp <= k_last;
          const bf16 *ks = kscr, *vs = vscr;
          if (valid && jp >= p0) {
            const size_t o = (size_t)(base + jp - p0) * kvd + g * HDT + c * 8;
            ks = kscr + o;
            vs = vscr + o;
          } else if (valid) {
            const size_t o = kv_row(kv, seq, KV, g, jp) * HDT + c * 8;
            ks = Kc + o;
            vs = Vc + o;
          }
          const uint32_t off = (c >> 3) * PANEL + sw(row, c & 7);
          cp16(dk + off, ks, valid);
          cp16(dv + off, vs, valid);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&k_full[st]);
          mbar_arrive(&v_full[st]);
        }
      }
      issued = j + 1;
    }
    // copies still in flight land before the CTA can exit
    if (lane == 0) {
      mbar_wait_drain(q_full, 0);
      for (int j = max(0, issued - NS); j < issued; ++j) {
        mbar_wait_drain(&k_full[j % NS], (j / NS) & 1);
        mbar_wait_drain(&v_full[j % NS], (j / NS) & 1);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      auto s_mma = [&](int q, int st) {
        const uint32_t qa = sb + Q_OFF + q * TILE, ka = sb + K_OFF + st * TILE;
#pragma unroll
        for (int kk = 0; kk < HDT / 16; ++kk) {
          const uint64_t a = sw128_desc(qa + (kk >> 2) * PANEL) + 2 * (kk & 3);
          const uint64_t b = sw128_desc(ka + (kk >> 2) * PANEL) + 2 * (kk & 3);
          umma(tmem + q * 128, a, b, kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[q]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, kv.err) && mbar_wait(&k_full[0], 0, abort_flag, kv.err);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 2; ++q)
          if (q < nslot && sl[q].a == 0) s_mma(q, 0);
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st = j % NS;
        ok = mbar_wait(&v_full[st], (j / NS) & 1, abort_flag, kv.err);
        if (!ok) break;
        const int j1 = j + 1, st1 = j1 % NS;
        bool k_next = false;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q >= nslot || !ok) break;
          const Slot& s = sl[q];
          if (j >= s.a && j <= s.b) {
            ok = mbar_wait(&p_full[q], (j - s.a) & 1, abort_flag, kv.err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t va = sb + V_OFF + st * TILE;
#pragma unroll
            for (int kk = 0; kk < TK / 16; ++kk)
              umma_ts(tmem + 256 + q * 128, tmem + q * 128 + kk * 8, sw128_mn_desc(va + kk * 2048, PANEL),
                      kIdescO, (j > s.a || kk > 0) ? 1u : 0u);
          }
          if (j1 >= s.a && j1 <= s.b) {
            if (!k_next) {
              ok = mbar_wait(&k_full[st1], (j1 / NS) & 1, abort_flag, kv.err);
              if (!ok) break;
              tc_fence_after();
              k_next = true;
            }
            s_mma(q, st1);
          }
        }
        if (!ok) break;
        umma_commit(&v_empty[st]);
        if (j1 < n_tiles) umma_commit(&k_empty[st1]);
      }
      umma_commit(o_full);
      mbar_wait_drain(o_full, 0);  // no MMA may still write TMEM when it is freed
    }
    __syncwarp();
   }
  } else {
   asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_SOFTMAX));
   if (warp / 4 < nslot) {
    // ------------------------------------------------------------ softmax
    const int q = warp >> 2, row = tid & 127;
    const Slot s = q ? sl[1] : sl[0];
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = q * 128, o_col = 256 + q * 128;
    const int pr = s.pf + row;
    float m_used = -1e30f, l = 0.f;
    bool ok = true;
    for (int j = s.a; j <= s.b; ++j) {
      ok = warp_wait(&s_full[q], (j - s.a) & 1, abort_flag, kv.err);
      if (!ok) break;
      tc_fence_after();
      uint32_t r[TK];
#pragma unroll
      for (int c = 0; c < TK; c += 32) tmem_ld32(lane_addr + s_col + c, r + c);
      tmem_wait_ld();
      const int kt = kt0 + j * TK;
      // a tile every row of the slot sees whole needs no mask
      const bool open = kt + TK - 1 <= s.pf && (kv.window == 0 || kt >= s.pl - kv.window + 1);
      if (!open) {  // key kt + c is visible iff c_lo <= c <= c_hi
        const int c_hi = pr - kt, c_lo = kv.window > 0 ? pr - kv.window + 1 - kt : -1;
#pragma unroll
        for (int c = 0; c < TK; ++c)
          if (c > c_hi || c < c_lo) r[c] = __float_as_uint(-INFINITY);
      }
      const float mt = row_max(r);
      const bool grow = mt > m_used + kLazy;
      float factor = 1.f;
      if (grow) {
        factor = ex2(m_used - mt);
        m_used = mt;
      }
      if (j > s.a && __any_sync(0xffffffffu, grow)) {  // O holds earlier tiles: rescale this row
#pragma unroll 1
        for (int c = 0; c < HDT; c += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + o_col + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
          tmem_st32(lane_addr + o_col + c, o);
        }
      }
      l *= factor;
      // P = 2^(s - m) as bf16 pairs over the first 64 columns of S, 16
      // columns (32 keys) at a time; two running sums (even, odd keys)
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float x0, x1;
          sub2(x0, x1, __uint_as_float(r[32 * h + c]), __uint_as_float(r[32 * h + c + 1]), m_used);
          x0 = ex2(x0);
          x1 = ex2(x1);
          add2(rs0, rs1, x0, x1);
          pk[c / 2] = pack2(x0, x1);
        }
        tmem_st16(lane_addr + s_col + 16 * h, pk);
      }
      l += rs0 + rs1;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[q]);
    }
    // every product of this CTA complete: normalise and store this row of O
    if (ok && warp_wait(o_full, 0, abort_flag, kv.err)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* dst = out + (size_t)(s.r0 + row) * qd + s.head * HDT;
      uint32_t o[HDT];  // the whole row of O with one wait
#pragma unroll
      for (int c = 0; c < HDT; c += 32) tmem_ld32(lane_addr + o_col + c, o + c);
      tmem_wait_ld();
      if (row < s.nrows) {
#pragma unroll
        for (int e = 0; e < HDT; e += 8) {
          uint4 u;
          u.x = pack2(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
          u.y = pack2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
          u.z = pack2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
          u.w = pack2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + e) = u;
        }
      }
    }
   }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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

// bf16 rows x cols (row stride `stride` elements), box 64 columns x 128 rows,
// 128-byte swizzle; reads past the last row or column return zeros.
struct MapKey {
  const void* p;
  uint64_t rows, cols, stride;
  bool operator==(const MapKey& o) const { return p == o.p && rows == o.rows && cols == o.cols && stride == o.stride; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    return std::hash<const void*>()(k.p) ^ (k.rows * 0x9E3779B97F4A7C15ull) ^ (k.cols << 7) ^ (k.stride << 29);
  }
};
std::mutex g_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

bool map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t stride) {
  std::lock_guard<std::mutex> lk(g_mu);
  const MapKey key{ptr, rows, cols, stride};
  auto it = g_maps.find(key);
  if (it != g_maps.end()) {
    *m = it->second;
    return true;
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(key, *m);
  return true;
}

}  // namespace

int prefill_ws_items(int n_tiles, const int* tile_last_pos, const int* tile_seq, int H, int KV, int4* items,
                     int cap) {
  const int G = H / KV;
  struct Item {
    int4 v;
    int cost;
  };
  std::vector<Item> list;
  list.reserve((size_t)n_tiles * H);
  for (int g = 0; g < KV; ++g) {
    // head pairs on the same rows
    for (int t = 0; t < n_tiles; ++t)
      for (int h = g * G; h + 1 < (g + 1) * G; h += 2)
        list.push_back({make_int4(t, h, t, h + 1), tile_last_pos[t] / TK + 1});
    if (G % 2 == 0) continue;
    // the odd head: consecutive row tiles of one sequence
    const int h = (g + 1) * G - 1;
    for (int t = 0; t < n_tiles;) {
      if (t + 1 < n_tiles && tile_seq[t + 1] == tile_seq[t]) {
        list.push_back({make_int4(t, h, t + 1, h), tile_last_pos[t + 1] / TK + 1});
        t += 2;
      } else {
        list.push_back({make_int4(t, h, -1, -1), tile_last_pos[t] / TK + 1});
        t += 1;
      }
    }
  }
  if ((int)list.size() > cap) return -1;
  std::stable_sort(list.begin(), list.end(), [](const Item& a, const Item& b) { return a.cost > b.cost; });
  for (size_t i = 0; i < list.size(); ++i) items[i] = list[i].v;
  return (int)list.size();
}

cudaError_t launch_attn_prefill_ws(int n_items, const int4* items, const int2* tiles, int M, int H, int KV, int hd,
                                   const bf16* qh, const bf16* kscr, const bf16* vscr, KVView kv, size_t kv_rows,
                                   RowMeta m, bf16* out, cudaStream_t st) {
  if (hd != HDT || H % KV) return cudaErrorNotSupported;
  if (n_items == 0) return cudaSuccess;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_prefill_ws, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap mq, mks, mvs, mkc, mvc;
  const uint64_t kvd = (uint64_t)KV * HDT;
  if (!map_2d(&mq, qh, M, (uint64_t)H * HDT, (uint64_t)H * HDT) || !map_2d(&mks, kscr, M, kvd, kvd) ||
      !map_2d(&mvs, vscr, M, kvd, kvd) || !map_2d(&mkc, kv.K, kv_rows, HDT, HDT) ||
      !map_2d(&mvc, kv.V, kv_rows, HDT, HDT))
    return cudaErrorInvalidValue;
  return launch(k_attn_prefill_ws, dim3(n_items), dim3(NTH), SMEM_BYTES, st, KV, H / KV, mq, mks, mvs, mkc, mvc, kscr,
                vscr, kv, m, tiles, items, out);
}

}  // namespace dory

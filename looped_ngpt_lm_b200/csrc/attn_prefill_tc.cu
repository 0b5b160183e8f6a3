// Prefill attention on the 5th-generation tensor cores (bf16, head_dim 128):
// S = Q K^T and O += P V as tcgen05 MMAs with fp32 accumulators in TMEM.
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
// One CTA per (128 query rows of one sequence, query head); 6 warps.
//   warps 0-3  one query row per thread (= TMEM lane): read S from TMEM,
//              mask, online softmax in base 2 (Q is pre-scaled by
//              log2(e)/sqrt(head_dim)), write P as bf16 into shared memory,
//              finally read O, divide by the row sum and store
//   warp 4     allocates TMEM, issues the MMAs (one elected lane)
//   warps 4-5  transpose each V tile in shared memory (ldmatrix +
//              stmatrix.trans) so that both MMAs take K-major operands
//   all        cp.async loads of Q, K and V tiles (keys at or after the
//              chunk start from the chunk scratch, earlier keys from the
//              cache ring, positions outside [lo, p_last] zero-filled)
// Per 64-key tile: S (128 x 64) = Q K^T; softmax; O (128 x 128) += P V.
// The running max is updated lazily: O in TMEM and the row sum are
// rescaled only when a row's max grows by more than 8 (log2 units), so
// P = exp2(s - m) stays below 256.
//
// Shared memory operands use the canonical 128-byte-swizzled K-major layout
// (rows of 128 bytes, 16-byte chunk c of row r at (c ^ (r % 8)) * 16, 8-row
// groups 1024 bytes apart, 64-element panels stored one after another).
// Every mbarrier wait is bounded; on expiry the CTA sets the device error
// word, stops, waits (bounded) for its MMAs and frees its TMEM.
#include <float.h>

#include "attn_prefill.cuh"
#include "umma.cuh"

namespace dory {

namespace {

using namespace tc;

constexpr int TQ = 128;  // query rows per CTA (MMA M, TMEM lanes)
constexpr int TK = 64;   // keys per tile
constexpr int HDT = 128;
constexpr int NTH = 192;
constexpr float kLazy = 8.f;  // rescale O only when a row max grows by more than this

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr int Q_OFF = 0;                     // 2 panels x 128 rows x 128 B
constexpr int K_OFF = Q_OFF + 2 * TQ * 128;  // 2 panels x 64 keys x 128 B
constexpr int VS_OFF = K_OFF + 2 * TK * 128; // V as loaded: 64 keys x 256 B, chunks XOR-swizzled
constexpr int VT_OFF = VS_OFF + TK * 256;    // V^T: 128 rows (head dims) x 64 keys, one panel
constexpr int P_OFF = VT_OFF + HDT * 128;    // P: 128 rows x 64 keys, one panel
constexpr int BAR_OFF = P_OFF + TQ * 128;    // mbarriers, TMEM slot, flags
constexpr int SMEM_BYTES = BAR_OFF + 128 + 1024;
constexpr int TMEM_COLS = 256;               // S at columns [0, 64), O at [128, 256)
constexpr int S_COL = 0, O_COL = 128;

// byte offset of 16-byte chunk c (0..7) of row r inside one 128-byte-row panel
__device__ __forceinline__ uint32_t sw(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// generic-proxy shared-memory writes -> visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// V tile (64 keys x 128 dims, key rows of 256 B with chunks XOR-swizzled by
// key) -> V^T (128 dim rows x 64 keys, canonical panel).  One warp moves one
// 16 x 16 block per step: ldmatrix reads four 8 x 8 matrices (keys x dims),
// stmatrix.trans writes them transposed (dims x keys).  Warp `wi` of `nw`
// takes blocks wi, wi + nw, ... of the 4 x 8 blocks.
__device__ __forceinline__ void transpose_v(uint32_t vs, uint32_t vt, int wi, int nw, int lane) {
  const int i = lane >> 3, j = lane & 7;
  for (int b = wi; b < (TK / 16) * (HDT / 16); b += nw) {
    const int kb = b / (HDT / 16), db = b % (HDT / 16);
    const int key = kb * 16 + j + 8 * (i & 1), dch = 2 * db + (i >> 1);
    const uint32_t src = vs + key * 256 + ((dch ^ (key & 7)) << 4);
    uint32_t r0, r1, r2, r3;
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(src));
    const int row = db * 16 + 8 * (i >> 1) + j, kch = 2 * kb + (i & 1);
    const uint32_t dst = vt + sw(row, kch);
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
  }
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 64; c += 16) tmem_ld16(taddr + c, *reinterpret_cast<float(*)[16]>(&v[c]));
}

__global__ void __launch_bounds__(NTH, 2) k_attn_prefill_tc(int KV, int G, const bf16* __restrict__ qh,
                                                           const bf16* __restrict__ kscr,
                                                           const bf16* __restrict__ vscr, KVView kv, RowMeta m,
                                                           const int2* __restrict__ tiles, bf16* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + Q_OFF, sK = sb + K_OFF, sVS = sb + VS_OFF, sVT = sb + VT_OFF, sP = sb + P_OFF;
  uint64_t* s_bar = (uint64_t*)(smem + BAR_OFF);  // S of the current tile complete (and every earlier MMA)
  uint64_t* o_bar = s_bar + 1;                    // every MMA complete (after the loop)
  uint32_t* tmem_slot = (uint32_t*)(s_bar + 2);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(s_bar, 1);
    mbar_init(o_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 4) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait();  // queries and chunk keys come from the preceding kernel
  pdl_trigger();

  // heavy (late) tiles first: the grid walks the tile table backwards
  const int2 tile = tiles[gridDim.x - 1 - blockIdx.x];
  const int head = blockIdx.y, g = head / G;
  const int r0 = tile.x, nrows = tile.y - tile.x;
  const int H = KV * G, qd = H * HDT, kvd = KV * HDT;
  const int seq = m.seq[r0], p0 = m.p0[r0], base = m.base[r0];
  const int pf = m.pos[r0], pl = m.pos[tile.y - 1];
  const int lo_min = kv.window > 0 ? max(0, pf - kv.window + 1) : 0;
  const bf16* Kc = (const bf16*)kv.K;
  const bf16* Vc = (const bf16*)kv.V;

  // Q tile (rows past the tile are zero)
  for (int i = tid; i < TQ * 16; i += NTH) {
    const int row = i >> 4, c = i & 15;
    const bool ok = row < nrows;
    cp16(sQ + (c >> 3) * (TQ * 128) + sw(row, c & 7), qh + (size_t)(r0 + (ok ? row : 0)) * qd + head * HDT + c * 8,
         ok);
  }
  // K and V tiles: thread `tid` keeps 16-byte chunk column lc = tid % 16 and
  // rows tid / 16 + 12 n.  A tile that lies wholly inside the chunk scratch
  // and [lo_min, p_last] is a run of rows kvd elements apart; other tiles
  // take the per-row path.
  const int lc = tid & 15, lr = tid >> 4;  // lr in 0..11
  const uint32_t dK0 = sK + (lc >> 3) * (TK * 128);
  auto load_kv = [&](int kt) {
    const bool run = kt >= lo_min && kt >= p0 && kt + TK - 1 <= pl;
    const size_t off0 = (size_t)(base + kt - p0 + lr) * kvd + g * HDT + lc * 8;
#pragma unroll 1
    for (int row = lr, n = 0; row < TK; row += NTH / 16, ++n) {
      const uint32_t dk = dK0 + sw(row, lc & 7), dv = sVS + row * 256 + ((lc ^ (row & 7)) << 4);
      if (run) {
        const size_t o = off0 + (size_t)n * (NTH / 16) * kvd;
        cp16(dk, kscr + o, true);
        cp16(dv, vscr + o, true);
      } else {
        const int j = kt + row;
        const bool ok = j >= lo_min && j <= pl;
        const bf16 *ks = qh, *vs = qh;
        if (ok && j >= p0) {
          const size_t o = (size_t)(base + j - p0) * kvd + g * HDT + lc * 8;
          ks = kscr + o;
          vs = vscr + o;
        } else if (ok) {
          const size_t o = kv_row(kv, seq, KV, g, j) * HDT + lc * 8;
          ks = Kc + o;
          vs = Vc + o;
        }
        cp16(dk, ks, ok);
        cp16(dv, vs, ok);
      }
    }
  };
  const int kt0 = (lo_min / TK) * TK;
  load_kv(kt0);
  cp_commit();
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  fence_async_smem();
  __syncthreads();

  // softmax state of row `tid` (warps 0-3)
  const int pr = pf + tid;
  const int lo_r = kv.window > 0 ? pr - kv.window + 1 : 0;
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  float m_used = -1e30f, l = 0.f;
  uint32_t s_phase = 0;
  int t = 0;
  for (int kt = kt0; kt <= pl; kt += TK, ++t) {
    // S = Q K^T
    if (warp == 4 && lane == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < HDT / 16; ++kk) {
        const uint64_t a = sw128_desc(sQ + (kk >> 2) * (TQ * 128)) + 2 * (kk & 3);
        const uint64_t b = sw128_desc(sK + (kk >> 2) * (TK * 128)) + 2 * (kk & 3);
        umma(tmem + S_COL, a, b, idesc_bf16(TQ, TK), kk > 0 ? 1u : 0u);
      }
      umma_commit(s_bar);
    }
    // S is ready, and so is every earlier MMA (the previous P V included)
    mbar_wait(s_bar, s_phase, abort_flag, kv.err);
    s_phase ^= 1;
    tc_fence_after();
    __syncthreads();
    if (*abort_flag) break;
    if (warp >= 4) {
      transpose_v(sVS, sVT, warp - 4, 2, lane);
      fence_async_smem();
    } else {
      float sv[TK];
      tmem_ld64(lane_addr + S_COL, sv);
      // a tile visible to every row of the CTA needs no mask
      const bool open = kt + TK - 1 <= pf && (kv.window == 0 || kt >= pl - kv.window + 1);
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < TK; ++c) {
        if (!open) {
          const int j = kt + c;
          if (!(j <= pr && j >= lo_r)) sv[c] = -INFINITY;
        }
        mt = fmaxf(mt, sv[c]);
      }
      const bool grow = mt > m_used + kLazy;
      float factor = 1.f;
      if (grow) {
        factor = ex2(m_used - mt);
        m_used = mt;
      }
      if (t > 0 && __any_sync(0xffffffffu, grow)) {  // O holds earlier tiles: rescale its rows
#pragma unroll 1
        for (int c = 0; c < HDT; c += 16) {
          float o[16];
          tmem_ld16(lane_addr + O_COL + c, o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= factor;
          tmem_st16(lane_addr + O_COL + c, o);
        }
      }
      l *= factor;
      uint32_t pk[TK / 2];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < TK; c += 2) {
        const float a = ex2(sv[c] - m_used), b = ex2(sv[c + 1] - m_used);
        rs += a + b;
        pk[c / 2] = pack2(a, b);
      }
      l += rs;
#pragma unroll
      for (int ch = 0; ch < TK / 8; ++ch)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sP + sw(tid, ch)), "r"(pk[4 * ch]),
                     "r"(pk[4 * ch + 1]), "r"(pk[4 * ch + 2]), "r"(pk[4 * ch + 3])
                     : "memory");
      fence_async_smem();
      tc_fence_before();
    }
    __syncthreads();  // P and V^T written, S consumed, O rescaled; K and V staging free
    if (kt + TK <= pl) load_kv(kt + TK);
    cp_commit();
    // O += P V
    if (warp == 4 && lane == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < TK / 16; ++kk)
        umma(tmem + O_COL, sw128_desc(sP) + 2 * kk, sw128_desc(sVT) + 2 * kk, idesc_bf16(TQ, HDT),
             (t > 0 || kk > 0) ? 1u : 0u);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    fence_async_smem();
    __syncthreads();
  }
  // every MMA of this CTA complete
  if (warp == 4 && lane == 0) umma_commit(o_bar);
  if (warp < 4) {
    const bool done = !*abort_flag && mbar_wait(o_bar, 0, abort_flag, kv.err);
    tc_fence_after();
    if (done) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* dst = out + (size_t)(r0 + tid) * qd + head * HDT;
#pragma unroll 1
      for (int c = 0; c < HDT; c += 16) {
        float o[16];
        tmem_ld16(lane_addr + O_COL + c, o);
        if (tid < nrows) {
          uint4 u0, u1;
          u0.x = pack2(o[0] * inv, o[1] * inv);
          u0.y = pack2(o[2] * inv, o[3] * inv);
          u0.z = pack2(o[4] * inv, o[5] * inv);
          u0.w = pack2(o[6] * inv, o[7] * inv);
          u1.x = pack2(o[8] * inv, o[9] * inv);
          u1.y = pack2(o[10] * inv, o[11] * inv);
          u1.z = pack2(o[12] * inv, o[13] * inv);
          u1.w = pack2(o[14] * inv, o[15] * inv);
          *reinterpret_cast<uint4*>(dst + c) = u0;
          *reinterpret_cast<uint4*>(dst + c + 8) = u1;
        }
      }
    }
  } else if (warp == 4 && lane == 0) {
    mbar_wait_drain(o_bar, 0);  // no MMA may still write TMEM when it is freed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace

bool attn_prefill_tc_supported(int hd) { return hd == HDT; }

cudaError_t launch_attn_prefill_tc(int n_tiles, const int2* tiles, int H, int KV, int hd, const bf16* qh,
                                   const bf16* kscr, const bf16* vscr, KVView kv, RowMeta m, bf16* out,
                                   cudaStream_t st) {
  if (hd != HDT || H % KV) return cudaErrorNotSupported;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_prefill_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch(k_attn_prefill_tc, dim3(n_tiles, H), dim3(NTH), SMEM_BYTES, st, KV, H / KV, qh, kscr, vscr, kv, m,
                tiles, out);
}

}  // namespace dory

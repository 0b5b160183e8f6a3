// Prefill attention on the tensor cores (bf16 mma.sync, fp32 accumulate),
// flash-attention style, for chunks whose K/V sit in the chunk scratch.
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
// One 128-thread block per (64-row query tile of one sequence, query head).
// Each warp owns 16 query rows; Q fragments stay in registers.  Key tiles of
// 64 absolute positions stream through a double-buffered shared-memory ring
// (cp.async, 16-byte chunks XOR-swizzled by row); keys at or after the chunk
// start come from the scratch rows, earlier keys from the cache (ring index
// j % cap).  Per key tile: S = Q K^T (m16n8k16), causal / sliding-window mask,
// base-2 online softmax (Q is pre-scaled by log2(e)/sqrt(head_dim)), then
// O += P V with P rounded to bf16.  Tiles wholly outside every row's window
// are skipped.  Keys outside [lo, p_last] are zero-filled so unwritten memory
// never reaches the products.
#include <float.h>

#include "attn_prefill.cuh"

namespace dory {

namespace {

constexpr int QT = 64;  // query rows per block
constexpr int KT = 64;  // keys per tile

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// byte offset of (row, 16-byte chunk) in a [rows][HD] bf16 tile, chunks
// XOR-swizzled by row so ldmatrix reads of 8 rows hit 8 different banks
template <int HD>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * HD * 2 + ((chunk ^ (row & 7)) << 4));
}

// Base-2 exponential on the special-function unit (PTX ex2.approx.ftz:
// subnormal results flush to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared memory: two K and two V tiles; the Q tile is staged in the second
// K tile and moved to registers before the first prefetch lands there.
template <int HD>
__global__ void __launch_bounds__(128, 3) k_attn_prefill(int KV, int G, const bf16* __restrict__ qh,
                                                      const bf16* __restrict__ kscr, const bf16* __restrict__ vscr,
                                                      KVView kv, RowMeta m, const int2* __restrict__ tiles,
                                                      bf16* __restrict__ out) {
  constexpr int CH = HD / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  static_assert(QT == KT, "the Q tile is staged in a K tile");
  uint8_t* sK = smem;
  uint8_t* sV = sK + 2 * KT * HD * 2;
  uint8_t* sQ = sK + KT * HD * 2;
  pdl_wait();
  pdl_trigger();

  // heavy (late) tiles first: the grid walks the tile table backwards
  const int2 tile = tiles[gridDim.x - 1 - blockIdx.x];
  const int head = blockIdx.y, g = head / G;
  const int r0 = tile.x, r1 = tile.y;  // rows [r0, r1) of one sequence
  const int H = KV * G, qd = H * HD, kvd = KV * HD;
  const int seq = m.seq[r0], p0 = m.p0[r0], base = m.base[r0];
  const int pf = m.pos[r0], pl = m.pos[r1 - 1];
  const int lo_min = kv.window > 0 ? max(0, pf - kv.window + 1) : 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bf16* Kc = (const bf16*)kv.K;
  const bf16* Vc = (const bf16*)kv.V;

  // Q tile -> shared memory (rows past r1 are zero)
  for (int i = tid; i < QT * CH; i += 128) {
    const int row = i / CH, ch = i % CH;
    const int r = r0 + row;
    const bool ok = r < r1;
    cp_async16(smem_addr(sQ + swz<HD>(row, ch)), qh + (size_t)(ok ? r : r0) * qd + head * HD + ch * 8, ok);
  }
  auto load_kv = [&](int kt, int buf) {
    uint8_t* dk = sK + buf * KT * HD * 2;
    uint8_t* dv = sV + buf * KT * HD * 2;
    for (int i = tid; i < KT * CH; i += 128) {
      const int row = i / CH, ch = i % CH;
      const int j = kt + row;
      const bool ok = j >= lo_min && j <= pl;
      const bf16 *ks, *vs;
      if (j >= p0) {
        const size_t o = (size_t)(base + (ok ? j - p0 : 0)) * kvd + g * HD + ch * 8;
        ks = kscr + o;
        vs = vscr + o;
      } else {
        const size_t o = (ok ? kv_row(kv, seq, KV, g, j) : 0) * HD + ch * 8;
        ks = Kc + o;
        vs = Vc + o;
      }
      cp_async16(smem_addr(dk + swz<HD>(row, ch)), ks, ok);
      cp_async16(smem_addr(dv + swz<HD>(row, ch)), vs, ok);
    }
  };
  const int kt0 = (lo_min / KT) * KT;
  load_kv(kt0, 0);
  cp_async_commit();

  // Q fragments: this warp's 16 rows, HD/16 k-chunks
  cp_async_wait<0>();
  __syncthreads();
  uint32_t qa[HD / 16][4];
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const int row = warp * 16 + (lane % 16), ch = kk * 2 + lane / 16;
    ldsm_x4(smem_addr(sQ + swz<HD>(row, ch)), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
  }
  __syncthreads();  // every warp holds its Q fragments: the tile may be overwritten
  const int gq = lane >> 2, tig = lane & 3;
  // positions of this thread's two rows
  const int pr0 = pf + warp * 16 + gq, pr1 = pr0 + 8;
  const int lo0 = kv.window > 0 ? pr0 - kv.window + 1 : 0, lo1 = kv.window > 0 ? pr1 - kv.window + 1 : 0;

  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-1e30f, -1e30f}, lrow[2] = {0.f, 0.f};

  int buf = 0;
  for (int kt = kt0; kt <= pl; kt += KT) {
    if (kt + KT <= pl) load_kv(kt + KT, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* k_s = sK + buf * KT * HD * 2;
    const uint8_t* v_s = sV + buf * KT * HD * 2;
    // S = Q K^T : 16 x 64 per warp
    float s[KT / 8][4];
#pragma unroll
    for (int i = 0; i < KT / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
      for (int n = 0; n < KT / 16; ++n) {
        uint32_t b0, b1, b2, b3;
        const int key = n * 16 + (lane % 8) + (lane / 16) * 8, ch = kk * 2 + (lane / 8) % 2;
        ldsm_x4(smem_addr(k_s + swz<HD>(key, ch)), b0, b1, b2, b3);
        mma_bf16(s[2 * n], qa[kk], b0, b1);
        mma_bf16(s[2 * n + 1], qa[kk], b2, b3);
      }
    }
    // mask and online softmax (two rows per thread).  A tile whose keys are
    // all visible to all 16 rows of this warp (causal and window) skips the
    // per-element mask.
    const int wr0 = pf + warp * 16;  // positions of this warp's first and last rows
    const bool open = kt + KT - 1 <= wr0 && (kv.window == 0 || kt >= wr0 + 15 - kv.window + 1);
    float mx[2] = {mrow[0], mrow[1]};
    if (!open) {
#pragma unroll
      for (int n = 0; n < KT / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = kt + n * 8 + 2 * tig + (e & 1);
          const int pr = e < 2 ? pr0 : pr1, lo = e < 2 ? lo0 : lo1;
          const bool ok = j <= pr && j >= lo && j >= 0;
          s[n][e] = ok ? s[n][e] : -FLT_MAX;
        }
      }
    }
#pragma unroll
    for (int n = 0; n < KT / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) mx[e >> 1] = fmaxf(mx[e >> 1], s[n][e]);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
    }
    float corr[2], rs[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 2; ++i) corr[i] = ex2(mrow[i] - mx[i]);
    uint32_t pa[KT / 16][4];
#pragma unroll
    for (int n = 0; n < KT / 8; ++n) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = (open || s[n][e] != -FLT_MAX) ? ex2(s[n][e] - mx[e >> 1]) : 0.f;
        rs[e >> 1] += p[e];
      }
      // C fragments of key tiles 2c, 2c+1 form the A fragment of k-chunk c
      const int c = n >> 1, hi = n & 1;
      pa[c][hi * 2 + 0] = pack_bf16(p[0], p[1]);
      pa[c][hi * 2 + 1] = pack_bf16(p[2], p[3]);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 1);
      rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 2);
      lrow[i] = lrow[i] * corr[i] + rs[i];
      mrow[i] = mx[i];
    }
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      o[i][0] *= corr[0];
      o[i][1] *= corr[0];
      o[i][2] *= corr[1];
      o[i][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int c = 0; c < KT / 16; ++c) {
      const uint32_t a[4] = {pa[c][0], pa[c][1], pa[c][2], pa[c][3]};
#pragma unroll
      for (int d = 0; d < HD / 16; ++d) {
        uint32_t b0, b1, b2, b3;
        const int key = c * 16 + (lane % 8) + ((lane / 8) % 2) * 8, ch = d * 2 + lane / 16;
        ldsm_x4_t(smem_addr(v_s + swz<HD>(key, ch)), b0, b1, b2, b3);
        mma_bf16(o[2 * d], a, b0, b1);
        mma_bf16(o[2 * d + 1], a, b2, b3);
      }
    }
    __syncthreads();
    buf ^= 1;
  }
  // normalise and store this thread's two rows
  const float inv0 = lrow[0] > 0.f ? 1.f / lrow[0] : 0.f, inv1 = lrow[1] > 0.f ? 1.f / lrow[1] : 0.f;
  const int ra = r0 + warp * 16 + gq, rb = ra + 8;
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) {
    const int d = i * 8 + 2 * tig;
    if (ra < r1)
      *reinterpret_cast<__nv_bfloat162*>(out + (size_t)ra * qd + head * HD + d) =
          __floats2bfloat162_rn(o[i][0] * inv0, o[i][1] * inv0);
    if (rb < r1)
      *reinterpret_cast<__nv_bfloat162*>(out + (size_t)rb * qd + head * HD + d) =
          __floats2bfloat162_rn(o[i][2] * inv1, o[i][3] * inv1);
  }
}

}  // namespace

int prefill_tiles(int n_seq, const int* cu, int2* tiles, int cap, int rows) {
  int n = 0;
  for (int b = 0; b < n_seq; ++b)
    for (int r = cu[b]; r < cu[b + 1]; r += rows) {
      if (n >= cap) return -1;
      tiles[n++] = make_int2(r, r + rows < cu[b + 1] ? r + rows : cu[b + 1]);
    }
  return n;
}

bool attn_prefill_supported(int hd) { return hd == 64 || hd == 128; }

cudaError_t launch_attn_prefill(int n_tiles, const int2* tiles, int H, int KV, int hd, const bf16* qh,
                                const bf16* kscr, const bf16* vscr, KVView kv, RowMeta m, bf16* out,
                                cudaStream_t st) {
  const int G = H / KV;
  if (hd == 128) {
    constexpr int SM = 4 * KT * 128 * 2;
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_attn_prefill<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    return launch(k_attn_prefill<128>, dim3(n_tiles, H), dim3(128), SM, st, KV, G, qh, kscr, vscr, kv, m, tiles, out);
  }
  if (hd == 64) {
    constexpr int SM = 4 * KT * 64 * 2;
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_attn_prefill<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    return launch(k_attn_prefill<64>, dim3(n_tiles, H), dim3(128), SM, st, KV, G, qh, kscr, vscr, kv, m, tiles, out);
  }
  return cudaErrorNotSupported;
}

}  // namespace dory

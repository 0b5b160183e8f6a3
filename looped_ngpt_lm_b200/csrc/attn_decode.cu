// Fused GQA attention for decode and speculative chunks (K/V written straight
// into the cache).
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
// One 256-thread block per (row, KV head g, absolute key block of DEC_BK
// positions):
//   1. stage the block's cached keys and values in shared memory with cp.async
//      (every byte in flight at once from a short rolled loop); keys of this
//      chunk are rebuilt from the QKV projection's split-K partials with the
//      same in-order sums and rounding the cache write uses;
//   2. q of the G query heads sharing KV head g = in-order partial sums,
//      scaled by log2(e)/sqrt(head_dim); the block holding the row's own
//      position writes the row's K and V into the cache slot;
//   3. base-2 online softmax over the block's keys: 8 warps x 4 groups of 8
//      lanes, one key per group, head_dim/8 dimensions per lane; groups merge
//      by a fixed xor tree, warps in index order;
//   4. the block stores (m, l, -, -, acc[head_dim]) per head (rows padded to
//      16 bytes); the last block of the (row, g) pair to finish (device
//      counter) merges every block's partial in block order, after copying
//      them into shared memory when they fit.
// Loops stay rolled: each block runs its code once, so a compact body keeps
// the instruction cache warm.  Block boundaries are absolute positions, so a
// row computes the same bits whether it is decoded alone or verified inside a
// speculative chunk.
#include <float.h>

#include "attn_decode.cuh"
#include "gemm_tc.cuh"
#include "warp_mma.cuh"

namespace dory {

namespace {

constexpr int NW = 8;  // warps per block

}  // namespace

int g_attn_cluster = 1;

namespace {

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// In-order sum of a value's S split-K slices.
__device__ __forceinline__ float sum_splits(const float* p, int S, size_t ps) {
  float v[kMaxSplitK];
#pragma unroll
  for (int s = 0; s < kMaxSplitK; ++s) v[s] = s < S ? __ldcg(p + s * ps) : 0.f;
  float a = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxSplitK; ++s)
    if (s < S) a += v[s];
  return a;
}

template <typename T, int HD, int G>
struct DecSmem {
  T k[DEC_BK][HD];
  T v[DEC_BK][HD];
  float q[G][HD];
  float wm[NW][G], wl[NW][G];
  float wacc[NW][G][HD];
  int last;
};

template <typename T, int HD, int G>
__global__ void __launch_bounds__(256) k_attn_decode(int KV, const float* __restrict__ qkv, int S, size_t ps,
                                                     KVView kv, RowMeta m, float* __restrict__ part, int nb_max,
                                                     unsigned* __restrict__ counters, T* __restrict__ out,
                                                     float scale_log2) {
  constexpr int DL = HD / 8;                    // dimensions per lane
  constexpr int CH = HD * (int)sizeof(T) / 16;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem<T, HD, G>& sm = *reinterpret_cast<DecSmem<T, HD, G>*>(smem_raw);

  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x / KV, g = blockIdx.x % KV;
  const int pos = m.pos[r], seq = m.seq[r], p0 = m.p0[r], base = m.base[r];
  if (pos < 0 || pos >= kv.limit) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
    return;
  }
  const int lo = kv.window > 0 ? max(0, pos - kv.window + 1) : 0;
  const int nb_row = pos / DEC_BK - lo / DEC_BK + 1;
  if (nb_row > nb_max) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
    return;
  }
  if ((int)blockIdx.y >= nb_row) return;
  const int kb = (lo / DEC_BK + blockIdx.y) * DEC_BK;
  const int klo = max(lo, kb), khi = min(pos, kb + DEC_BK - 1);
  const int H = KV * G, qd = H * HD, kvd = KV * HD, ld = qd + 2 * kvd;
  const int tid = threadIdx.x;
  T* Kc = (T*)kv.K;
  T* Vc = (T*)kv.V;

  // 1. cached keys -> shared memory (all copies in flight), chunk keys rebuilt
  const int cache_hi = min(khi, p0 - 1);  // last cached key of this block
  for (int i = tid; i < (cache_hi - klo + 1) * CH; i += blockDim.x) {
    const int jj = i / CH, c = i % CH;
    const size_t src = kv_row(kv, seq, KV, g, klo + jj) * HD;
    cp16(saddr(&sm.k[klo - kb + jj][0]) + c * 16, (const uint8_t*)(Kc + src) + c * 16);
    cp16(saddr(&sm.v[klo - kb + jj][0]) + c * 16, (const uint8_t*)(Vc + src) + c * 16);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  const int jc0 = max(klo, p0);  // first key of this chunk in the block
  for (int i = tid; i < (khi - jc0 + 1) * HD; i += blockDim.x) {
    const int jj = i / HD, d = i % HD;
    const float* src = qkv + (size_t)(base + (jc0 + jj - p0)) * ld + qd + g * HD + d;
    sm.k[jc0 - kb + jj][d] = from_f<T>(sum_splits(src, S, ps));
    sm.v[jc0 - kb + jj][d] = from_f<T>(sum_splits(src + kvd, S, ps));
  }
  // 2. q for the G heads; the own key goes to the cache
  for (int i = tid; i < G * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    sm.q[h][d] = sum_splits(qkv + (size_t)r * ld + (g * G + h) * HD + d, S, ps) * scale_log2;
  }
  if (khi == pos) {
    const size_t slot = kv_row(kv, seq, KV, g, pos) * HD;
    for (int i = tid; i < 2 * HD; i += blockDim.x) {
      const int d = i % HD;
      const bool is_v = i >= HD;
      const float a = sum_splits(qkv + (size_t)r * ld + qd + (is_v ? kvd : 0) + g * HD + d, S, ps);
      (is_v ? Vc : Kc)[slot + d] = from_f<T>(a);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // 3. online softmax over the block's keys
  const int w = tid >> 5, lane = tid & 31, sg = lane >> 3, dl = lane & 7;
  float qv[G][DL], mx[G], ls[G], acc[G][DL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mx[h] = -FLT_MAX;
    ls[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) {
      qv[h][e] = sm.q[h][dl * DL + e];
      acc[h][e] = 0.f;
    }
  }
#pragma unroll 1
  for (int jq = kb + 4 * w; jq <= khi; jq += 4 * NW) {
    const int j = jq + sg;
    const bool valid = j >= klo && j <= khi;
    const int row = valid ? j - kb : 0;
    float kf[DL], vf[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) {
      kf[e] = to_f(sm.k[row][dl * DL + e]);
      vf[e] = to_f(sm.v[row][dl * DL + e]);
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) sdot += qv[h][e] * kf[e];
      sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
      sdot += __shfl_xor_sync(0xffffffffu, sdot, 2);
      sdot += __shfl_xor_sync(0xffffffffu, sdot, 4);
      if (valid) {
        const float mn = fmaxf(mx[h], sdot);
        const float corr = exp2f(mx[h] - mn);
        const float p = exp2f(sdot - mn);
        ls[h] = ls[h] * corr + p;
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[h][e] = acc[h][e] * corr + p * vf[e];
        mx[h] = mn;
      }
    }
  }
#pragma unroll 1
  for (int off = 8; off <= 16; off <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float om = __shfl_xor_sync(0xffffffffu, mx[h], off);
      const float ol = __shfl_xor_sync(0xffffffffu, ls[h], off);
      const float mn = fmaxf(mx[h], om);
      const float ca = (mx[h] == -FLT_MAX) ? 0.f : exp2f(mx[h] - mn);
      const float cb = (om == -FLT_MAX) ? 0.f : exp2f(om - mn);
      ls[h] = ls[h] * ca + ol * cb;
#pragma unroll
      for (int e = 0; e < DL; ++e) {
        const float oa = __shfl_xor_sync(0xffffffffu, acc[h][e], off);
        acc[h][e] = acc[h][e] * ca + oa * cb;
      }
      mx[h] = mn;
    }
  }
  if (sg == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (dl == 0) {
        sm.wm[w][h] = mx[h];
        sm.wl[w][h] = ls[h];
      }
#pragma unroll
      for (int e = 0; e < DL; ++e) sm.wacc[w][h][dl * DL + e] = acc[h][e];
    }
  }
  __syncthreads();
  constexpr int PE = HD + 4;  // partial entry: m, l, 2 pad, acc[HD]
  const size_t hstride = (size_t)nb_max * PE;
  float* pr0 = part + ((size_t)r * H + g * G) * hstride;
  for (int i = tid; i < G * (HD + 2); i += blockDim.x) {
    const int h = i / (HD + 2), c = i % (HD + 2);
    float M = -FLT_MAX;
    for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, sm.wm[ww][h]);
    float val = M;
    if (c > 0) {
      val = 0.f;
      for (int ww = 0; ww < NW; ++ww) {
        const float sc = sm.wm[ww][h] == -FLT_MAX ? 0.f : exp2f(sm.wm[ww][h] - M);
        val += (c == 1 ? sm.wl[ww][h] : sm.wacc[ww][h][c - 2]) * sc;
      }
    }
    pr0[h * hstride + blockIdx.y * PE + (c < 2 ? c : c + 2)] = val;
  }

  // 4. the last block of this (row, g) merges all blocks in order
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = atomicAdd(&counters[r * KV + g], 1u) == (unsigned)(nb_row - 1);
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  // every block's partial -> shared memory (reusing the key/value buffers)
  // when they fit, else read them from L2
  const bool in_smem = (size_t)G * nb_row * PE * 4 <= sizeof(sm.k) + sizeof(sm.v);
  const float* pb = pr0;
  size_t pstride = hstride;
  if (in_smem) {
    float* dst = reinterpret_cast<float*>(&sm.k[0][0]);  // [G][nb_row][PE]
    const int nrow4 = nb_row * PE / 4;                   // 16-byte pieces per head
    for (int i = tid; i < G * nrow4; i += blockDim.x) {
      const int h = i / nrow4, c = i % nrow4;
      cp16(saddr(dst + (size_t)h * nb_row * PE) + c * 16, pr0 + h * hstride + c * 4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    pb = dst;
    pstride = (size_t)nb_row * PE;
  }
  __syncthreads();
  // shared memory: plain loads; global (other blocks' writes): L2 loads
  auto ldp = [&](const float* p) { return in_smem ? *p : __ldcg(p); };
  for (int i = tid; i < G * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    const float* ph = pb + h * pstride;
    float M = -FLT_MAX;
    for (int b = 0; b < nb_row; ++b) M = fmaxf(M, ldp(ph + b * PE));
    float L = 0.f, a = 0.f;
    for (int b = 0; b < nb_row; ++b) {
      const float wgt = exp2f(ldp(ph + b * PE) - M);
      L += ldp(ph + b * PE + 1) * wgt;
      a += ldp(ph + b * PE + 4 + d) * wgt;
    }
    out[(size_t)r * qd + (g * G + h) * HD + d] = from_f<T>(a / L);
  }
  if (tid == 0) counters[r * KV + g] = 0u;
}

// ---------------------------------------------------------------------------
// Cluster variant: one cluster of CS blocks per (row, KV head).  The row's key
// range [lo, pos] is cut into CS equal parts (a function of the row's own
// positions only, so decode and verify rows get identical partitions); each
// block streams its part through shared memory in sub-chunks of DEC_BK keys;
// the blocks' partials are merged in rank order by rank 0 through
// distributed shared memory.  No global partials, fences or counters.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float dsmem_ld(const float* local, int rank) {
  uint32_t a = saddr(local), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

template <typename T, int HD, int G>
struct ClSmem {
  T k[DEC_BK][HD];
  T v[DEC_BK][HD];
  float q[G][HD];
  float wm[NW][G], wl[NW][G];
  float wacc[NW][G][HD];
  float part[G][HD + 2];   // this block's (m, l, acc) -- read by rank 0
  float rw[16][G];         // rank 0: per-rank weights
  float rinv[G];
};

template <typename T, int HD, int G, int CS>
__global__ void __launch_bounds__(256) k_attn_decode_cl(int KV, const float* __restrict__ qkv, int S, size_t ps,
                                                        KVView kv, RowMeta m, T* __restrict__ out,
                                                        float scale_log2) {
  constexpr int DL = HD / 8;
  constexpr int CH = HD * (int)sizeof(T) / 16;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  ClSmem<T, HD, G>& sm = *reinterpret_cast<ClSmem<T, HD, G>*>(smem_raw);

  pdl_wait();
  pdl_trigger();
  const int pair = blockIdx.x / CS, rank = blockIdx.x % CS;
  const int r = pair / KV, g = pair % KV;
  const int pos = m.pos[r], seq = m.seq[r], p0 = m.p0[r], base = m.base[r];
  const bool row_ok = pos >= 0 && pos < kv.limit;
  if (!row_ok && threadIdx.x == 0 && rank == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
  const int lo = kv.window > 0 ? max(0, pos - kv.window + 1) : 0;
  const int nk = pos - lo + 1, per = (nk + CS - 1) / CS;
  const int klo = lo + rank * per, khi = row_ok ? min(pos, klo + per - 1) : klo - 1;  // empty when klo > khi
  const int H = KV * G, qd = H * HD, kvd = KV * HD, ld = qd + 2 * kvd;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, sg = lane >> 3, dl = lane & 7;
  T* Kc = (T*)kv.K;
  T* Vc = (T*)kv.V;

  if (row_ok) {
    for (int i = tid; i < G * HD; i += blockDim.x) {
      const int h = i / HD, d = i % HD;
      sm.q[h][d] = sum_splits(qkv + (size_t)r * ld + (g * G + h) * HD + d, S, ps) * scale_log2;
    }
    if (klo <= pos && pos <= khi) {  // this block holds the row's own key
      const size_t slot = kv_row(kv, seq, KV, g, pos) * HD;
      for (int i = tid; i < 2 * HD; i += blockDim.x) {
        const int d = i % HD;
        const bool is_v = i >= HD;
        const float a = sum_splits(qkv + (size_t)r * ld + qd + (is_v ? kvd : 0) + g * HD + d, S, ps);
        (is_v ? Vc : Kc)[slot + d] = from_f<T>(a);
      }
    }
  }
  __syncthreads();
  float qv[G][DL], mx[G], ls[G], acc[G][DL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mx[h] = -FLT_MAX;
    ls[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) {
      qv[h][e] = sm.q[h][dl * DL + e];
      acc[h][e] = 0.f;
    }
  }
#pragma unroll 1
  for (int c0 = klo; c0 <= khi; c0 += DEC_BK) {
    const int c1 = min(khi, c0 + DEC_BK - 1);
    const int cache_hi = min(c1, p0 - 1);
    for (int i = tid; i < (cache_hi - c0 + 1) * CH; i += blockDim.x) {
      const int jj = i / CH, c = i % CH;
      const size_t src = kv_row(kv, seq, KV, g, c0 + jj) * HD;
      cp16(saddr(&sm.k[jj][0]) + c * 16, (const uint8_t*)(Kc + src) + c * 16);
      cp16(saddr(&sm.v[jj][0]) + c * 16, (const uint8_t*)(Vc + src) + c * 16);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const int jc0 = max(c0, p0);
    for (int i = tid; i < (c1 - jc0 + 1) * HD; i += blockDim.x) {
      const int jj = i / HD, d = i % HD;
      const float* src = qkv + (size_t)(base + (jc0 + jj - p0)) * ld + qd + g * HD + d;
      sm.k[jc0 - c0 + jj][d] = from_f<T>(sum_splits(src, S, ps));
      sm.v[jc0 - c0 + jj][d] = from_f<T>(sum_splits(src + kvd, S, ps));
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
#pragma unroll 1
    for (int jq = c0 + 4 * w; jq <= c1; jq += 4 * NW) {
      const int j = jq + sg;
      const bool valid = j <= c1;
      const int row = valid ? j - c0 : 0;
      float kf[DL], vf[DL];
#pragma unroll
      for (int e = 0; e < DL; ++e) {
        kf[e] = to_f(sm.k[row][dl * DL + e]);
        vf[e] = to_f(sm.v[row][dl * DL + e]);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float sdot = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) sdot += qv[h][e] * kf[e];
        sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
        sdot += __shfl_xor_sync(0xffffffffu, sdot, 2);
        sdot += __shfl_xor_sync(0xffffffffu, sdot, 4);
        if (valid) {
          const float mn = fmaxf(mx[h], sdot);
          const float corr = exp2f(mx[h] - mn);
          const float p = exp2f(sdot - mn);
          ls[h] = ls[h] * corr + p;
#pragma unroll
          for (int e = 0; e < DL; ++e) acc[h][e] = acc[h][e] * corr + p * vf[e];
          mx[h] = mn;
        }
      }
    }
    __syncthreads();
  }
#pragma unroll 1
  for (int off = 8; off <= 16; off <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float om = __shfl_xor_sync(0xffffffffu, mx[h], off);
      const float ol = __shfl_xor_sync(0xffffffffu, ls[h], off);
      const float mn = fmaxf(mx[h], om);
      const float ca = (mx[h] == -FLT_MAX) ? 0.f : exp2f(mx[h] - mn);
      const float cb = (om == -FLT_MAX) ? 0.f : exp2f(om - mn);
      ls[h] = ls[h] * ca + ol * cb;
#pragma unroll
      for (int e = 0; e < DL; ++e) {
        const float oa = __shfl_xor_sync(0xffffffffu, acc[h][e], off);
        acc[h][e] = acc[h][e] * ca + oa * cb;
      }
      mx[h] = mn;
    }
  }
  if (sg == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (dl == 0) {
        sm.wm[w][h] = mx[h];
        sm.wl[w][h] = ls[h];
      }
#pragma unroll
      for (int e = 0; e < DL; ++e) sm.wacc[w][h][dl * DL + e] = acc[h][e];
    }
  }
  __syncthreads();
  // warps -> this block's partial (per-warp weights computed once per head)
  if (tid < G) {
    float M = -FLT_MAX;
    for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, sm.wm[ww][tid]);
    float L = 0.f;
    for (int ww = 0; ww < NW; ++ww) {
      const float sc = sm.wm[ww][tid] == -FLT_MAX ? 0.f : exp2f(sm.wm[ww][tid] - M);
      sm.wm[ww][tid] = sc;  // now the warp's weight
      L += sm.wl[ww][tid] * sc;
    }
    sm.part[tid][0] = M;
    sm.part[tid][1] = L;
  }
  __syncthreads();
  for (int i = tid; i < G * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    float a = 0.f;
    for (int ww = 0; ww < NW; ++ww) a += sm.wacc[ww][h][d] * sm.wm[ww][h];
    sm.part[h][2 + d] = a;
  }
  cluster_sync();  // every block's partial is ready
  if (rank == 0 && row_ok) {
    if (tid < G) {
      float M = -FLT_MAX;
      for (int q = 0; q < CS; ++q) M = fmaxf(M, dsmem_ld(&sm.part[tid][0], q));
      float L = 0.f;
      for (int q = 0; q < CS; ++q) {
        const float mq = dsmem_ld(&sm.part[tid][0], q);
        const float wq = mq == -FLT_MAX ? 0.f : exp2f(mq - M);
        sm.rw[q][tid] = wq;
        L += dsmem_ld(&sm.part[tid][1], q) * wq;
      }
      sm.rinv[tid] = 1.f / L;
    }
    __syncthreads();
    for (int i = tid; i < G * HD; i += blockDim.x) {
      const int h = i / HD, d = i % HD;
      float a = 0.f;
      for (int q = 0; q < CS; ++q) a += dsmem_ld(&sm.part[h][2 + d], q) * sm.rw[q][h];
      out[(size_t)r * qd + (g * G + h) * HD + d] = from_f<T>(a * sm.rinv[h]);
    }
  }
  cluster_sync();  // rank 0 has read every partial; blocks may exit
}

// ---------------------------------------------------------------------------
// Tensor-core variant (bf16, head_dim 64 or 128): the cluster layout above,
// with each warp running 16-key steps on mma.sync.  The G query heads that
// share the KV head are rows 0..G-1 of a 16-row A tile (rows G..15 are zero),
// so S = Q K^T and O += P V cost 2 * head_dim / 8 MMAs per 16 keys.  Warps
// take steps w, w + 8, ...; their states merge in warp order, then the
// cluster's blocks merge in rank order through distributed shared memory.
// A block's keys stream through two shared-memory chunks of TC_KC keys: the
// first two are requested at once, and chunk i + 2 is requested as soon as
// chunk i has been consumed.
constexpr int TC_KC = 128;  // keys per shared-memory chunk (two chunks)

// Base-2 exponential on the special-function unit (PTX ex2.approx.ftz).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void dsmem_st(float* local, int rank, float v) {
  uint32_t a = saddr(local), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

template <int HD, int G, int CS>
struct TcSmem {
  uint8_t q[16 * HD * 2];
  uint8_t k[2][TC_KC * HD * 2];
  uint8_t v[2][TC_KC * HD * 2];
  float wm[NW][G], wl[NW][G];
  float wacc[NW][G][HD];
  float part[G][HD + 2];
  float all[CS][G][HD + 2];  // every rank's (max, sum) and this rank's dimensions of its accumulator
  float rw[CS][G];
  float rinv[G];
};

// Cluster size of the tensor-core decode attention: the largest of 16, 8, 4
// whose grid for `batch` sequences stays within about four waves of one
// block per SM.  It depends on the number of sequences only (never on rows
// per sequence), so plain decode and a speculative verify of the same
// sequences split every row's keys identically.
constexpr int kDecodeBlockBudget = 4 * 148;
inline int decode_cluster_size(int batch, int KV) {
  const int pairs = batch * KV;
  if (pairs * 16 <= kDecodeBlockBudget) return 16;
  if (pairs * 8 <= kDecodeBlockBudget) return 8;
  return 4;
}

template <int HD, int G, int CS>
__global__ void __launch_bounds__(256) k_attn_decode_tc(int KV, const float* __restrict__ qkv, int S, size_t ps,
                                                        KVView kv, RowMeta m, bf16* __restrict__ out,
                                                        float scale_log2) {
  using namespace wm;
  constexpr int CH = HD / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem_raw[];
  TcSmem<HD, G, CS>& sm = *reinterpret_cast<TcSmem<HD, G, CS>*>(smem_raw);

  const int pair = blockIdx.x / CS, rank = blockIdx.x % CS;
  const int r = pair / KV, g = pair % KV;
  const int pos = m.pos[r], seq = m.seq[r], p0 = m.p0[r], base = m.base[r];
  const bool row_ok = pos >= 0 && pos < kv.limit;
  if (!row_ok && threadIdx.x == 0 && rank == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
  const int lo = kv.window > 0 ? max(0, pos - kv.window + 1) : 0;
  const int nk = pos - lo + 1, per = (nk + CS - 1) / CS;
  const int klo = lo + rank * per, khi = row_ok ? min(pos, klo + per - 1) : klo - 1;
  const int H = KV * G, qd = H * HD, kvd = KV * HD, ld = qd + 2 * kvd;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, tig = lane & 3;
  // linear or ring cache: this (sequence, KV head)'s rows; paged: the pools
  const bf16* Kc = (const bf16*)kv.K + (kv.pt ? 0 : ((size_t)seq * KV + g) * kv.cap * HD);
  const bf16* Vc = (const bf16*)kv.V + (kv.pt ? 0 : ((size_t)seq * KV + g) * kv.cap * HD);

  // chunk ci holds keys klo + ci * TC_KC .. in buffer ci & 1.  Cached keys
  // (positions < p0) and the zero padding up to 16 keys come by cp.async;
  // they were written by earlier calls and nothing in flight rewrites them
  // (this chunk's positions map to ring slots no row here reads), so the
  // first two chunks are requested before waiting for the QKV projection.
  const int nchunk = khi >= klo ? (khi - klo) / TC_KC + 1 : 0;
  // thread `tid` keeps chunk column tid % CH and rows tid / CH + RS * n; the
  // ring slot of its row advances by RS (a division only when it wraps)
  constexpr int RS = 256 / CH;
  auto issue_cached = [&](int ci) {
    const int c0 = klo + ci * TC_KC, c1 = min(khi, c0 + TC_KC - 1), n = c1 - c0 + 1, n16 = (n + 15) & ~15;
    const int cache_hi = min(c1, p0 - 1);
    uint8_t* kb = sm.k[ci & 1];
    uint8_t* vb = sm.v[ci & 1];
    const int c = tid % CH;
    int jj = tid / CH;
    if (kv.pt) {
      for (; jj < n16; jj += RS) {
        if (c0 + jj <= cache_hi || jj >= n) {  // cached key, or zero padding up to 16 keys
          const size_t src = (jj < n ? kv_row(kv, seq, KV, g, c0 + jj) : 0) * HD + c * 8;
          cp_async16(smem_addr(kb + swz<HD>(jj, c)), Kc + src, jj < n);
          cp_async16(smem_addr(vb + swz<HD>(jj, c)), Vc + src, jj < n);
        }
      }
    } else {
      int slot = (c0 + jj) % kv.cap;
      for (; jj < n16; jj += RS) {
        if (c0 + jj <= cache_hi || jj >= n) {  // cached key, or zero padding up to 16 keys
          const size_t src = (size_t)slot * HD + c * 8;
          cp_async16(smem_addr(kb + swz<HD>(jj, c)), Kc + src, jj < n);
          cp_async16(smem_addr(vb + swz<HD>(jj, c)), Vc + src, jj < n);
        }
        slot += RS;
        if (slot >= kv.cap) slot %= kv.cap;  // rare: only when the row wraps around the ring
      }
    }
    cp_async_commit();
  };
  // the chunk's own keys (positions >= p0), summed from the QKV partials
  auto fill_new = [&](int ci) {
    const int c0 = klo + ci * TC_KC, c1 = min(khi, c0 + TC_KC - 1);
    const int jc0 = max(c0, p0);
    uint8_t* kb = sm.k[ci & 1];
    uint8_t* vb = sm.v[ci & 1];
#pragma unroll 4
    for (int i = tid; i < (c1 - jc0 + 1) * HD; i += blockDim.x) {
      const int jj = i / HD, d = i % HD, row = jc0 - c0 + jj;
      const float* src = qkv + (size_t)(base + (jc0 + jj - p0)) * ld + qd + g * HD + d;
      *reinterpret_cast<bf16*>(kb + swz<HD>(row, d / 8) + (d % 8) * 2) = __float2bfloat16_rn(sum_splits(src, S, ps));
      *reinterpret_cast<bf16*>(vb + swz<HD>(row, d / 8) + (d % 8) * 2) =
          __float2bfloat16_rn(sum_splits(src + kvd, S, ps));
    }
  };
  if (nchunk > 0) issue_cached(0);
  if (nchunk > 1) issue_cached(1);
  pdl_wait();

  // Q tile: rows 0..G-1 = the G heads (pre-scaled, bf16), rows G..15 zero;
  // the block holding the row's own position also writes the row's K and V
  // into the cache.  Every split-K partial these need is requested before
  // any is summed (one round trip to L2); each sum runs in slice order.
  constexpr int QIT = (G * HD + 255) / 256;  // passes of the 256 threads that hold query elements
  const bool own = row_ok && klo <= pos && pos <= khi;
  float qp[QIT][kMaxSplitK], kp[kMaxSplitK];
#pragma unroll
  for (int it = 0; it < QIT; ++it) {
    const int i = tid + it * 256, h = i / HD, d = i % HD;
    const bool live = h < G && row_ok;
    const float* src = qkv + (size_t)r * ld + (live ? (g * G + h) * HD + d : 0);
#pragma unroll
    for (int s = 0; s < kMaxSplitK; ++s) qp[it][s] = live && s < S ? __ldcg(src + s * ps) : 0.f;
  }
  {
    const int d = tid % HD;
    const bool live = own && tid < 2 * HD;
    const float* src = qkv + (size_t)r * ld + (live ? qd + (tid >= HD ? kvd : 0) + g * HD + d : 0);
#pragma unroll
    for (int s = 0; s < kMaxSplitK; ++s) kp[s] = live && s < S ? __ldcg(src + s * ps) : 0.f;
  }
#pragma unroll
  for (int it = 0; it < 16 * HD / 256; ++it) {
    const int i = tid + it * 256, h = i / HD, d = i % HD;
    float val = 0.f;
    if (it < QIT && h < G && row_ok) {
      float a = 0.f;
#pragma unroll
      for (int s = 0; s < kMaxSplitK; ++s)
        if (s < S) a += qp[it < QIT ? it : 0][s];
      val = a * scale_log2;
    }
    *reinterpret_cast<bf16*>(sm.q + swz<HD>(h, d / 8) + (d % 8) * 2) = __float2bfloat16_rn(val);
  }
  // a decode row's chunk holds one new key, its own: when that chunk sits in
  // one of the first two buffers it is written from these sums (the same
  // bits the cache gets) instead of being summed again by fill_new
  const int ci_own = own ? (pos - klo) / TC_KC : -1;
  const bool own_direct = own && p0 == pos && ci_own < 2;
  if (own && tid < 2 * HD) {  // this block holds the row's own key
    float a = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxSplitK; ++s)
      if (s < S) a += kp[s];
    const bf16 b = __float2bfloat16_rn(a);
    const int d = tid % HD;
    bf16* dst = (bf16*)(tid >= HD ? kv.V : kv.K);
    dst[kv_row(kv, seq, KV, g, pos) * HD + d] = b;
    if (own_direct) {
      uint8_t* buf = tid >= HD ? sm.v[ci_own & 1] : sm.k[ci_own & 1];
      *reinterpret_cast<bf16*>(buf + swz<HD>(pos - klo - ci_own * TC_KC, d / 8) + (d % 8) * 2) = b;
    }
  }
  __syncthreads();
  uint32_t qa[HD / 16][4];
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk)
    ldsm_x4(smem_addr(sm.q + swz<HD>(lane % 16, kk * 2 + lane / 16)), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);

  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-FLT_MAX, -FLT_MAX}, lrow[2] = {0.f, 0.f};

  if (nchunk > 0 && !(own_direct && ci_own == 0)) fill_new(0);
  if (nchunk > 1 && !(own_direct && ci_own == 1)) fill_new(1);

#pragma unroll 1
  for (int ci = 0; ci < nchunk; ++ci) {
    const int c0 = klo + ci * TC_KC, n = min(khi, c0 + TC_KC - 1) - c0 + 1;
    if (ci + 1 < nchunk)
      cp_async_wait<1>();  // chunk ci landed; ci + 1 may be in flight
    else
      cp_async_wait<0>();
    __syncthreads();
    // the O projection that follows may launch (and stream its weights)
    // once this block's first keys have arrived, not before
    if (ci == 0) pdl_trigger();
    const uint8_t* kbuf = sm.k[ci & 1];
    const uint8_t* vbuf = sm.v[ci & 1];
#pragma unroll 1
    for (int st = w; st * 16 < n; st += NW) {
      float sc[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t) sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_addr(kbuf + swz<HD>(st * 16 + (lane % 8) + (lane / 16) * 8, kk * 2 + (lane / 8) % 2)), b0, b1,
                b2, b3);
        mma_bf16(sc[0], qa[kk], b0, b1);
        mma_bf16(sc[1], qa[kk], b2, b3);
      }
      float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int jl = st * 16 + t * 8 + 2 * tig + (e & 1);
          if (jl >= n) sc[t][e] = -FLT_MAX;
          mx[e >> 1] = fmaxf(mx[e >> 1], sc[t][e]);
        }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      }
      float corr[2], rs[2] = {0.f, 0.f}, pv[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i) corr[i] = mrow[i] == -FLT_MAX ? 0.f : ex2(mrow[i] - mx[i]);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pv[t][e] = sc[t][e] == -FLT_MAX ? 0.f : ex2(sc[t][e] - mx[e >> 1]);
          rs[e >> 1] += pv[t][e];
        }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 1);
        rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 2);
        lrow[i] = lrow[i] * corr[i] + rs[i];
        mrow[i] = mx[i];
      }
      const uint32_t pa[4] = {pack_bf16(pv[0][0], pv[0][1]), pack_bf16(pv[0][2], pv[0][3]),
                              pack_bf16(pv[1][0], pv[1][1]), pack_bf16(pv[1][2], pv[1][3])};
      if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {  // a row max moved
#pragma unroll
        for (int i = 0; i < HD / 8; ++i) {
          o[i][0] *= corr[0];
          o[i][1] *= corr[0];
          o[i][2] *= corr[1];
          o[i][3] *= corr[1];
        }
      }
#pragma unroll
      for (int d = 0; d < HD / 16; ++d) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_addr(vbuf + swz<HD>(st * 16 + (lane % 8) + ((lane / 8) % 2) * 8, d * 2 + lane / 16)), b0, b1,
                  b2, b3);
        mma_bf16(o[2 * d], pa, b0, b1);
        mma_bf16(o[2 * d + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // buffer ci & 1 is free
    if (ci + 2 < nchunk) {
      issue_cached(ci + 2);
      fill_new(ci + 2);
    }
  }
  if (nchunk == 0) pdl_trigger();
  // this warp's rows 0..G-1 (held by lanes with gq < G, row gq) -> shared memory
  if (gq < G) {
    if (tig == 0) {
      sm.wm[w][gq] = mrow[0];
      sm.wl[w][gq] = lrow[0];
    }
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      sm.wacc[w][gq][i * 8 + 2 * tig] = o[i][0];
      sm.wacc[w][gq][i * 8 + 2 * tig + 1] = o[i][1];
    }
  }
  __syncthreads();
  if (tid < G) {
    float M = -FLT_MAX;
    for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, sm.wm[ww][tid]);
    float L = 0.f;
    for (int ww = 0; ww < NW; ++ww) {
      const float scw = sm.wm[ww][tid] == -FLT_MAX ? 0.f : exp2f(sm.wm[ww][tid] - M);
      sm.wm[ww][tid] = scw;
      L += sm.wl[ww][tid] * scw;
    }
    sm.part[tid][0] = M;
    sm.part[tid][1] = L;
  }
  __syncthreads();
  for (int i = tid; i < G * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    float a = 0.f;
    for (int ww = 0; ww < NW; ++ww) a += sm.wacc[ww][h][d] * sm.wm[ww][h];
    sm.part[h][2 + d] = a;
  }
  __syncthreads();
  // every rank merges HD / CS of the head dimensions: each block pushes its
  // (max, sum) pair to every rank and each of its accumulator elements to
  // the rank that owns that dimension (stores only), then, after one cluster
  // barrier, each rank reads only its own shared memory and writes its slice
  // of the output.  The merge runs in rank order, the same sums as a single
  // merging block.
  static_assert(HD % CS == 0, "head dimensions split evenly over the cluster");
  constexpr int DS = HD / CS;  // head dimensions per rank
  for (int i = tid; i < CS * G * 2; i += blockDim.x) {
    const int q = i / (G * 2), e = i % (G * 2);
    dsmem_st(&sm.all[rank][e >> 1][e & 1], q, sm.part[e >> 1][e & 1]);
  }
  for (int i = tid; i < G * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    dsmem_st(&sm.all[rank][h][2 + d], d / DS, sm.part[h][2 + d]);
  }
  cluster_sync();  // every partial has landed where it is merged
  if (row_ok) {
    if (tid < G) {
      float M = -FLT_MAX;
      for (int q = 0; q < CS; ++q) M = fmaxf(M, sm.all[q][tid][0]);
      float L = 0.f;
      for (int q = 0; q < CS; ++q) {
        const float mq = sm.all[q][tid][0];
        const float wq = mq == -FLT_MAX ? 0.f : exp2f(mq - M);
        sm.rw[q][tid] = wq;
        L += sm.all[q][tid][1] * wq;
      }
      sm.rinv[tid] = 1.f / L;
    }
    __syncthreads();
    for (int i = tid; i < G * DS; i += blockDim.x) {
      const int h = i / DS, d = rank * DS + i % DS;
      float a = 0.f;
      for (int q = 0; q < CS; ++q) a += sm.all[q][h][2 + d] * sm.rw[q][h];
      out[(size_t)r * qd + (g * G + h) * HD + d] = __float2bfloat16_rn(a * sm.rinv[h]);
    }
  }
}

template <int HD, int G, int CS>
cudaError_t dispatch_tc(int M, int KV, const float* qkv, int S, size_t ps, KVView kv, RowMeta m, bf16* out,
                        cudaStream_t st) {
  constexpr int SMEM = (int)sizeof(TcSmem<HD, G, CS>);
  auto kern = k_attn_decode_tc<HD, G, CS>;
  static int state = 0;
  if (state == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      cudaGetLastError();
      state = -1;
    } else {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(CS);
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = SMEM;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = CS;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      state = (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) ? 1 : -1;
      cudaGetLastError();
    }
  }
  if (state < 0) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M * KV * CS);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  return cudaLaunchKernelEx(&cfg, kern, KV, qkv, S, ps, kv, m, out, scale_log2);
}

template <typename T, int HD, int G>
cudaError_t dispatch_cl(int M, int KV, const float* qkv, int S, size_t ps, KVView kv, RowMeta m, T* out,
                        cudaStream_t st) {
  constexpr int CS = 16;
  constexpr int SMEM = (int)sizeof(ClSmem<T, HD, G>);
  static int state = 0;  // 0 unknown, 1 usable, -1 not schedulable here
  if (state == 0) {
    auto kern = k_attn_decode_cl<T, HD, G, CS>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      cudaGetLastError();
      state = -1;
    } else {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(CS);
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = SMEM;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = CS;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      state = (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) ? 1 : -1;
      cudaGetLastError();
    }
  }
  if (state < 0) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M * KV * CS);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  return cudaLaunchKernelEx(&cfg, k_attn_decode_cl<T, HD, G, CS>, KV, qkv, S, ps, kv, m, out, scale_log2);
}

template <typename T, int HD, int G>
cudaError_t dispatch(int M, int KV, const float* qkv, int S, size_t ps, KVView kv, RowMeta m, int max_ctx,
                     float* part, int nb_cap, int part_rows, unsigned* counters, T* out, int batch,
                     cudaStream_t st) {
  if constexpr (sizeof(T) == 2 && HD >= 64 && G <= 16) {
    if (g_attn_cluster) {
      const int cs = g_attn_cluster >= 4 ? g_attn_cluster : decode_cluster_size(batch, KV);
      cudaError_t e = cs == 16  ? dispatch_tc<HD, G, 16>(M, KV, qkv, S, ps, kv, m, (bf16*)out, st)
                      : cs == 8 ? dispatch_tc<HD, G, 8>(M, KV, qkv, S, ps, kv, m, (bf16*)out, st)
                                : dispatch_tc<HD, G, 4>(M, KV, qkv, S, ps, kv, m, (bf16*)out, st);
      if (e != cudaErrorNotSupported) return e;
    }
  }
  if (g_attn_cluster) {
    cudaError_t e = dispatch_cl<T, HD, G>(M, KV, qkv, S, ps, kv, m, out, st);
    if (e != cudaErrorNotSupported) return e;
  }
  const int span = kv.window > 0 ? min(max_ctx, kv.window) : max_ctx;
  const int nb = (span + DEC_BK - 1) / DEC_BK + 1;
  constexpr int SMEM = (int)sizeof(DecSmem<T, HD, G>);
  if (nb > nb_cap || M > part_rows) return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_decode<T, HD, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  return launch(k_attn_decode<T, HD, G>, dim3(M * KV, nb), dim3(256), SMEM, st, KV, qkv, S, ps, kv, m, part, nb,
                counters, out, scale_log2);
}

}  // namespace

template <typename T>
cudaError_t launch_attn_decode(int M, int H, int KV, int hd, const float* qkv, int S, size_t ps, KVView kv,
                               RowMeta m, int max_ctx, float* part, int nb_cap, int part_rows, unsigned* counters,
                               T* out, int batch, cudaStream_t st) {
  const int G = H / KV;
#define DORY_DEC_CASE(HDV, GV)                                                                                   \
  if (hd == HDV && G == GV)                                                                                      \
    return dispatch<T, HDV, GV>(M, KV, qkv, S, ps, kv, m, max_ctx, part, nb_cap, part_rows, counters, out, batch, \
                                st);
  DORY_DEC_CASE(32, 1) DORY_DEC_CASE(32, 2) DORY_DEC_CASE(32, 4) DORY_DEC_CASE(32, 5) DORY_DEC_CASE(32, 8)
  DORY_DEC_CASE(64, 1) DORY_DEC_CASE(64, 2) DORY_DEC_CASE(64, 4) DORY_DEC_CASE(64, 5) DORY_DEC_CASE(64, 8)
  DORY_DEC_CASE(128, 1) DORY_DEC_CASE(128, 2) DORY_DEC_CASE(128, 4) DORY_DEC_CASE(128, 5)
#undef DORY_DEC_CASE
  return cudaErrorInvalidValue;
}

template cudaError_t launch_attn_decode<float>(int, int, int, int, const float*, int, size_t, KVView, RowMeta, int,
                                               float*, int, int, unsigned*, float*, int, cudaStream_t);
template cudaError_t launch_attn_decode<bf16>(int, int, int, int, const float*, int, size_t, KVView, RowMeta, int,
                                              float*, int, int, unsigned*, bf16*, int, cudaStream_t);

int attn_decode_ctas(int batch, int KV, int hd, int G) {
  if (!g_attn_cluster || hd < 64 || G > 16) return 0;
  const int cs = g_attn_cluster >= 4 ? g_attn_cluster : decode_cluster_size(batch, KV);
  return batch * KV * cs;
}

}  // namespace dory

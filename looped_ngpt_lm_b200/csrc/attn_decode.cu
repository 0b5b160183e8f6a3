// Fused GQA attention for decode and speculative chunks (K/V written straight
// into the cache).
//
// One block per (row, KV head g, absolute key block of DEC_BK positions):
//   1. q of the G query heads that share KV head g = in-order sum of the QKV
//      projection's split-K partials (scaled by log2(e)/sqrt(head_dim));
//   2. the block holding the row's own position writes the row's K and V
//      (same partial sums, rounded to the storage type) into the cache slot;
//   3. keys of earlier calls come from the cache (ring index j % cap); keys of
//      this chunk are rebuilt from the partials with the same arithmetic, so
//      they equal what the cache will hold;
//   4. base-2 online softmax over the block's keys: 8 warps x 4 groups of 8
//      lanes, one key per group, head_dim/8 dimensions per lane; groups merge
//      by a fixed xor tree, warps in index order;
//   5. the block stores (m, l, acc[head_dim]) per head; the last block of the
//      (row, g) pair to finish (device counter) merges all blocks in block
//      order and writes the attention output.
// Block boundaries are absolute positions, so a row computes the same bits
// whether it is decoded alone or verified inside a speculative chunk.
#include <float.h>

#include "attn_decode.cuh"
#include "gemm_tc.cuh"

namespace dory {

namespace {

// A row slice of DL elements kept in the storage type until it is used.
template <typename T, int DL>
struct RowBuf {
  T v[DL];
};

// Vector load of DL consecutive elements (16-byte pieces; 8 bytes for 4 bf16).
template <typename T, int DL>
__device__ __forceinline__ void load_raw(const T* p, RowBuf<T, DL>& b) {
  constexpr int BYTES = DL * (int)sizeof(T);
  if constexpr (BYTES % 16 == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(p);
    uint4* dst = reinterpret_cast<uint4*>(b.v);
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i) dst[i] = src[i];
  } else {
    static_assert(BYTES == 8, "row slice must be 8 or a multiple of 16 bytes");
    *reinterpret_cast<uint2*>(b.v) = *reinterpret_cast<const uint2*>(p);
  }
}

// In-order sum of a value's S split-K slices (independent, predicated loads).
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
__global__ void __launch_bounds__(256) k_attn_decode(int KV, const float* __restrict__ qkv, int S, size_t ps,
                                                     KVView kv, RowMeta m, float* __restrict__ part, int nb_max,
                                                     unsigned* __restrict__ counters, T* __restrict__ out,
                                                     float scale_log2) {
  constexpr int DL = HD / 8;
  constexpr int NW = 8;
  constexpr int KPI = NW * 4;  // keys per iteration
  __shared__ float q_sm[G][HD];
  __shared__ float sm_m[NW][G], sm_l[NW][G];
  __shared__ float sm_acc[NW][G][HD];
  __shared__ int s_last;

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
  const int ab = lo / DEC_BK + blockIdx.y;
  const int kb = ab * DEC_BK;
  const int klo = max(lo, kb), khi = min(pos, kb + DEC_BK - 1);
  const int H = KV * G, qd = H * HD, kvd = KV * HD, ld = qd + 2 * kvd;
  const int tid = threadIdx.x;

  constexpr int QPT = (G * HD + 255) / 256;  // q values per thread
#pragma unroll
  for (int c = 0; c < QPT; ++c) {
    const int idx = tid + c * 256;
    if (idx < G * HD) {
      const int h = idx / HD, d = idx % HD;
      q_sm[h][d] = sum_splits(qkv + (size_t)r * ld + (g * G + h) * HD + d, S, ps) * scale_log2;
    }
  }
  T* Kc = (T*)kv.K + ((size_t)seq * KV + g) * kv.cap * HD;
  T* Vc = (T*)kv.V + ((size_t)seq * KV + g) * kv.cap * HD;
  if (khi == pos) {  // this block holds the row's own key: write it to the cache
    const size_t slot = (size_t)(pos % kv.cap) * HD;
    for (int idx = tid; idx < 2 * HD; idx += blockDim.x) {
      const int d = idx % HD;
      const bool is_v = idx >= HD;
      const float a = sum_splits(qkv + (size_t)r * ld + qd + (is_v ? kvd : 0) + g * HD + d, S, ps);
      (is_v ? Vc : Kc)[slot + d] = from_f<T>(a);
    }
  }
  __syncthreads();

  const int w = tid >> 5, lane = tid & 31, sg = lane >> 3, dl = lane & 7;
  float qv[G][DL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DL; ++e) qv[h][e] = q_sm[h][dl * DL + e];
  float mx[G], ls[G], acc[G][DL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mx[h] = -FLT_MAX;
    ls[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[h][e] = 0.f;
  }
  constexpr int ITER = DEC_BK / KPI;
  RowBuf<T, DL> kr[ITER], vr[ITER];
  bool valid[ITER];
#pragma unroll
  for (int it = 0; it < ITER; ++it) {
    const int j = kb + it * KPI + w * 4 + sg;
    valid[it] = j >= klo && j <= khi;
    if (valid[it]) {
      if (j < p0) {
        const size_t idx = (size_t)(j % kv.cap) * HD + dl * DL;
        load_raw<T, DL>(Kc + idx, kr[it]);
        load_raw<T, DL>(Vc + idx, vr[it]);
      } else {  // key of this chunk: rebuild it from the projection partials
        const float* src = qkv + (size_t)(base + (j - p0)) * ld + qd + g * HD + dl * DL;
#pragma unroll
        for (int e = 0; e < DL; ++e) {
          kr[it].v[e] = from_f<T>(sum_splits(src + e, S, ps));
          vr[it].v[e] = from_f<T>(sum_splits(src + kvd + e, S, ps));
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < DL; ++e) kr[it].v[e] = vr[it].v[e] = from_f<T>(0.f);
    }
  }
#pragma unroll
  for (int it = 0; it < ITER; ++it) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) sdot += qv[h][e] * to_f(kr[it].v[e]);
      sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
      sdot += __shfl_xor_sync(0xffffffffu, sdot, 2);
      sdot += __shfl_xor_sync(0xffffffffu, sdot, 4);
      if (valid[it]) {
        const float mn = fmaxf(mx[h], sdot);
        const float corr = exp2f(mx[h] - mn);
        const float p = exp2f(sdot - mn);
        ls[h] = ls[h] * corr + p;
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[h][e] = acc[h][e] * corr + p * to_f(vr[it].v[e]);
        mx[h] = mn;
      }
    }
  }
#pragma unroll
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
        sm_m[w][h] = mx[h];
        sm_l[w][h] = ls[h];
      }
#pragma unroll
      for (int e = 0; e < DL; ++e) sm_acc[w][h][dl * DL + e] = acc[h][e];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * (HD + 2); idx += blockDim.x) {
    const int h = idx / (HD + 2), c = idx % (HD + 2);
    float M = -FLT_MAX;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, sm_m[ww][h]);
    float val = 0.f;
    if (c == 0) {
      val = M;
    } else {
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) {
        const float sc = sm_m[ww][h] == -FLT_MAX ? 0.f : exp2f(sm_m[ww][h] - M);
        val += (c == 1 ? sm_l[ww][h] : sm_acc[ww][h][c - 2]) * sc;
      }
    }
    part[(((size_t)r * H + g * G + h) * nb_max + blockIdx.y) * (HD + 2) + c] = val;
  }
  // last block of this (row, g) merges every block in order
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(&counters[r * KV + g], 1u);
    s_last = prev == (unsigned)(nb_row - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge: (1) all threads fetch every block's (m, l) into shared memory;
  // (2) per head, the max M and 1/L = 1 / sum_b l_b 2^(m_b - M); (3) block
  // weights 2^(m_b - M); (4) every (head, dim) output sums its blocks with
  // independent loads.  Block order fixes the summation order.
  float* sm_mb = &sm_acc[0][0][0];  // reused: [G][nb_row] m, then weights
  float* sm_lb = sm_mb + G * nb_row;  // [G][nb_row] l
  float* sm_hd = sm_lb + G * nb_row;  // [G] M, then [G] 1/L
  const size_t hstride = (size_t)nb_max * (HD + 2);
  const float* pr0 = part + ((size_t)r * H + g * G) * hstride;
  for (int idx = tid; idx < G * nb_row; idx += blockDim.x) {
    const int h = idx / nb_row, b = idx % nb_row;
    sm_mb[idx] = __ldcg(pr0 + h * hstride + b * (HD + 2));
    sm_lb[idx] = __ldcg(pr0 + h * hstride + b * (HD + 2) + 1);
  }
  __syncthreads();
  if (tid < G) {
    float M = -FLT_MAX;
    for (int b = 0; b < nb_row; ++b) M = fmaxf(M, sm_mb[tid * nb_row + b]);
    float L = 0.f;
    for (int b = 0; b < nb_row; ++b) L += sm_lb[tid * nb_row + b] * exp2f(sm_mb[tid * nb_row + b] - M);
    sm_hd[tid] = M;
    sm_hd[G + tid] = 1.f / L;
  }
  __syncthreads();
  for (int idx = tid; idx < G * nb_row; idx += blockDim.x) sm_mb[idx] = exp2f(sm_mb[idx] - sm_hd[idx / nb_row]);
  __syncthreads();
  const float* wts = sm_mb;
  constexpr int OPT = (G * HD + 255) / 256;  // outputs per thread
  constexpr int BB = 8;                      // blocks per batch of loads
  float o[OPT];
#pragma unroll
  for (int c = 0; c < OPT; ++c) o[c] = 0.f;
  for (int b0 = 0; b0 < nb_row; b0 += BB) {
    float v[OPT][BB];
#pragma unroll
    for (int c = 0; c < OPT; ++c) {
      const int idx = tid + c * 256;
      const int h = idx / HD, d = idx % HD;
#pragma unroll
      for (int j = 0; j < BB; ++j)
        v[c][j] = (idx < G * HD && b0 + j < nb_row) ? __ldcg(pr0 + h * hstride + (b0 + j) * (HD + 2) + 2 + d) : 0.f;
    }
#pragma unroll
    for (int c = 0; c < OPT; ++c) {
      const int h = min((tid + c * 256) / HD, G - 1);
#pragma unroll
      for (int j = 0; j < BB; ++j)
        if (b0 + j < nb_row) o[c] += v[c][j] * wts[h * nb_row + b0 + j];
    }
  }
#pragma unroll
  for (int c = 0; c < OPT; ++c) {
    const int idx = tid + c * 256;
    if (idx < G * HD) {
      const int h = idx / HD, d = idx % HD;
      out[(size_t)r * qd + (g * G + h) * HD + d] = from_f<T>(o[c] * sm_hd[G + h]);
    }
  }
  if (tid == 0) counters[r * KV + g] = 0u;
}

template <typename T, int HD, int G>
cudaError_t dispatch(int M, int KV, const float* qkv, int S, size_t ps, KVView kv, RowMeta m, int max_ctx,
                     float* part, int nb_cap, unsigned* counters, T* out, cudaStream_t st) {
  const int span = kv.window > 0 ? min(max_ctx, kv.window) : max_ctx;
  const int nb = (span + DEC_BK - 1) / DEC_BK + 1;
  // the merge keeps 2 * G * nb + 2 * G floats in the 8 * G * HD float buffer
  if (nb > nb_cap || 2 * nb + 2 > 8 * HD) return cudaErrorInvalidValue;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  return launch(k_attn_decode<T, HD, G>, dim3(M * KV, nb), dim3(256), 0, st, KV, qkv, S, ps, kv, m, part, nb,
                counters, out, scale_log2);
}

}  // namespace

template <typename T>
cudaError_t launch_attn_decode(int M, int H, int KV, int hd, const float* qkv, int S, size_t ps, KVView kv,
                               RowMeta m, int max_ctx, float* part, int nb_cap, unsigned* counters, T* out,
                               cudaStream_t st) {
  const int G = H / KV;
#define DORY_DEC_CASE(HDV, GV) \
  if (hd == HDV && G == GV) return dispatch<T, HDV, GV>(M, KV, qkv, S, ps, kv, m, max_ctx, part, nb_cap, counters, out, st);
  DORY_DEC_CASE(32, 1) DORY_DEC_CASE(32, 2) DORY_DEC_CASE(32, 4) DORY_DEC_CASE(32, 5) DORY_DEC_CASE(32, 8)
  DORY_DEC_CASE(64, 1) DORY_DEC_CASE(64, 2) DORY_DEC_CASE(64, 4) DORY_DEC_CASE(64, 5) DORY_DEC_CASE(64, 8)
  DORY_DEC_CASE(128, 1) DORY_DEC_CASE(128, 2) DORY_DEC_CASE(128, 4) DORY_DEC_CASE(128, 5)
#undef DORY_DEC_CASE
  return cudaErrorInvalidValue;
}

template cudaError_t launch_attn_decode<float>(int, int, int, int, const float*, int, size_t, KVView, RowMeta, int,
                                               float*, int, unsigned*, float*, cudaStream_t);
template cudaError_t launch_attn_decode<bf16>(int, int, int, int, const float*, int, size_t, KVView, RowMeta, int,
                                              float*, int, unsigned*, bf16*, cudaStream_t);

}  // namespace dory

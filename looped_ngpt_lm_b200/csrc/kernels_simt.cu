// CUDA-core kernels of the looped nGPT forward: planning, embedding, the nGPT
// residual+L2-norm, loop re-injection, QKV split and KV-cache writes, GQA
// attention over ring/linear caches, SwiGLU, argmax, speculative acceptance,
// and a reference SIMT GEMM (fp32 storage, or bf16 before the tensor-core
// path takes over).
//
// What is computed: the layer update h <- N(h + sublayer(h)) with N the L2
// normalisation of the nGPT backbone (review of "Dory1.0-4B: A Looped
// Normalized-GPT", blog.secrett2633.cloud, "1. Key Terms"; the update rule
// itself is this library's reading), and
// the loop boundary u_t = N(s_{t-1} + x), s_0 = x, of the shared recurrent
// block (Dory1.0-4B digest, onedev.kr/papers/1692, "How it works").
//
// Every reduction here runs in a fixed order that depends only on the row's
// own data and absolute positions, never on how many rows share a launch, so
// a row computes bit-identical results alone or inside a larger chunk.
#include <float.h>

#include "addnorm.cuh"
#include "common.cuh"
#include "kernels.cuh"
#include "gemm_tc.cuh"

namespace dory {


// ------------------------------------------------------------------ planning
__global__ void k_plan_uniform(int n_rows, int rps, int pos_offset, const int* seq_ids, const int* seq_len,
                               RowMeta m) {
  pdl_wait();
  pdl_trigger();
  int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= n_rows) return;
  int b = r / rps, i = r % rps;
  int seq = seq_ids[b];
  int p0 = seq_len[seq] + pos_offset;
  m.seq[r] = seq;
  m.pos[r] = p0 + i;
  m.p0[r] = p0;
  m.base[r] = b * rps;
  m.pend[r] = p0 + rps;
}

cudaError_t launch_plan_uniform(int n_seq, int rps, int pos_offset, const int* seq_ids, const int* seq_len,
                                RowMeta m, cudaStream_t st) {
  int n = n_seq * rps;
  launch(k_plan_uniform, (n + 127) / 128, 128, 0, st, n, rps, pos_offset, seq_ids, seq_len, m);
  return cudaGetLastError();
}

__global__ void k_plan_ragged(int n_seq, const int* cu, const int* seq_ids, const int* seq_len, RowMeta m) {
  pdl_wait();
  pdl_trigger();
  int b = blockIdx.x;
  int seq = seq_ids[b];
  int r0 = cu[b], r1 = cu[b + 1];
  int p0 = seq_len[seq];
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    m.seq[r] = seq;
    m.pos[r] = p0 + (r - r0);
    m.p0[r] = p0;
    m.base[r] = r0;
    m.pend[r] = p0 + (r1 - r0);
  }
}

cudaError_t launch_plan_ragged(int n_seq, int n_rows, const int* cu, const int* seq_ids, const int* seq_len,
                               RowMeta m, cudaStream_t st) {
  (void)n_rows;
  launch(k_plan_ragged, n_seq, 128, 0, st, n_seq, cu, seq_ids, seq_len, m);
  return cudaGetLastError();
}

__global__ void k_advance(int n_seq, const int* seq_ids, int* seq_len, int delta) {
  pdl_wait();
  pdl_trigger();
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < n_seq) seq_len[seq_ids[b]] += delta;
}

cudaError_t launch_advance(int n_seq, const int* seq_ids, int* seq_len, int delta, cudaStream_t st) {
  launch(k_advance, (n_seq + 127) / 128, 128, 0, st, n_seq, seq_ids, seq_len, delta);
  return cudaGetLastError();
}

__global__ void k_advance_ragged(int n_seq, const int* seq_ids, const int* cu, int* seq_len) {
  pdl_wait();
  pdl_trigger();
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < n_seq) seq_len[seq_ids[b]] += cu[b + 1] - cu[b];
}

cudaError_t launch_advance_ragged(int n_seq, const int* seq_ids, const int* cu, int* seq_len, cudaStream_t st) {
  launch(k_advance_ragged, (n_seq + 127) / 128, 128, 0, st, n_seq, seq_ids, cu, seq_len);
  return cudaGetLastError();
}

__global__ void k_fill_i32(int n, int* p, int v) {
  pdl_wait();
  pdl_trigger();
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

cudaError_t launch_fill_i32(int n, int* p, int v, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  launch(k_fill_i32, (n + 255) / 256, 256, 0, st, n, p, v);
  return cudaGetLastError();
}

__global__ void k_split_reduce(size_t total, const float* part, int S, size_t ps, float* out) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < S; ++s) a += part[s * ps + i];
    out[i] = a;
  }
}

cudaError_t launch_split_reduce(int M, int N, const float* part, int S, size_t ps, float* out, cudaStream_t st) {
  size_t total = (size_t)M * N;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  launch(k_split_reduce, blocks, 256, 0, st, total, part, S, ps, out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ embedding
template <typename T>
__global__ void k_embed(int d, int vocab, const int* tokens, const T* E, float* h, T* hop, float* x, int* err) {
  pdl_wait();
  pdl_trigger();
  int r = blockIdx.x;
  int tok = tokens[r];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) set_error(err, DEV_ERR_BAD_TOKEN);
    tok = 0;
  }
  const T* src = E + (size_t)tok * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    T v = src[i];
    h[(size_t)r * d + i] = to_f(v);
    hop[(size_t)r * d + i] = v;
    if (x) x[(size_t)r * d + i] = to_f(v);
  }
}

template <typename T>
cudaError_t launch_embed(int M, int d, int vocab, const int* tokens, const T* E, float* h, T* hop, float* x,
                         int* err, cudaStream_t st) {
  launch(k_embed<T>, M, 256, 0, st, d, vocab, tokens, E, h, hop, x, err);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ add + norm
// One 512-thread block per row, one thread per virtual thread of the
// arithmetic in addnorm.cuh (shared with the decode GEMM's operand stage).
template <typename T>
__global__ void __launch_bounds__(AN_VT) k_addnorm(int d, const float* h_in, float* h_out,
                                                   const float* __restrict__ y, int S, size_t ps, int ldy, T* hop,
                                                   float* copy_out) {
  pdl_trigger();  // see common.cuh: the next GEMM may take SMs as the last one drains
  pdl_wait();
  __shared__ float red[AN_VT / 32];
  const int r = blockIdx.x, v = threadIdx.x;
  float e[AN_CPT];
  const float ss = an_warp_tree(an_load(h_in + (size_t)r * d, y + (size_t)r * ldy, S, ps, d, v, e));
  if ((v & 31) == 0) red[v >> 5] = ss;
  __syncthreads();
  const float inv = an_inv_from_warps(red);
#pragma unroll
  for (int c = 0; c < AN_CPT; ++c) {
    const int i = v + c * AN_VT;
    if (i < d) {
      const float o = e[c] * inv;
      h_out[(size_t)r * d + i] = o;
      hop[(size_t)r * d + i] = from_f<T>(o);
      if (copy_out) copy_out[(size_t)r * d + i] = o;
    }
  }
}

// Long prefill chunks: one warp per row, 16-byte loads and stores.  The same
// mathematics (v = h + sum_s y_s in slice order, h <- v / max(||v||, 1e-12))
// in another summation order: prefill rows never have to match the bits of
// decode rows (those take the 512-virtual-thread arithmetic above).
constexpr int ANR_ROWS = 8;   // rows (warps) per block
constexpr int ANR_V4 = 24;    // float4 per lane: d <= 3072

template <typename T>
__global__ void __launch_bounds__(ANR_ROWS * 32) k_addnorm_rows(int M, int d, const float* h_in, float* h_out,
                                                               const float* __restrict__ y, int S, size_t ps,
                                                               int ldy, T* hop, float* copy_out) {
  pdl_trigger();  // see common.cuh
  pdl_wait();
  const int r = blockIdx.x * ANR_ROWS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= M) return;
  const int d4 = d >> 2;
  const float4* hr = reinterpret_cast<const float4*>(h_in + (size_t)r * d);
  // every load of a slice is issued before any is used
  float4 v[ANR_V4];
#pragma unroll
  for (int c = 0; c < ANR_V4; ++c) {
    const int i = lane + 32 * c;
    v[c] = i < d4 ? __ldcg(hr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int sl = 0; sl < S; ++sl) {
    const float4* yr = reinterpret_cast<const float4*>(y + sl * ps + (size_t)r * ldy);
    float4 b[ANR_V4];
#pragma unroll
    for (int c = 0; c < ANR_V4; ++c) {
      const int i = lane + 32 * c;
      b[c] = i < d4 ? __ldcg(yr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int c = 0; c < ANR_V4; ++c) {
      v[c].x += b[c].x;
      v[c].y += b[c].y;
      v[c].z += b[c].z;
      v[c].w += b[c].w;
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < ANR_V4; ++c) {
    ss = __fmaf_rn(v[c].x, v[c].x, ss);
    ss = __fmaf_rn(v[c].y, v[c].y, ss);
    ss = __fmaf_rn(v[c].z, v[c].z, ss);
    ss = __fmaf_rn(v[c].w, v[c].w, ss);
  }
  ss = warp_sum(ss);
  const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
  float4* ho = reinterpret_cast<float4*>(h_out + (size_t)r * d);
  float4* co = copy_out ? reinterpret_cast<float4*>(copy_out + (size_t)r * d) : nullptr;
#pragma unroll
  for (int c = 0; c < ANR_V4; ++c) {
    const int i = lane + 32 * c;
    if (i < d4) {
      const float4 o = make_float4(v[c].x * inv, v[c].y * inv, v[c].z * inv, v[c].w * inv);
      ho[i] = o;
      if (co) co[i] = o;
      if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(o.x, o.y), b = __floats2bfloat162_rn(o.z, o.w);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&a);
        u.y = *reinterpret_cast<const uint32_t*>(&b);
        reinterpret_cast<uint2*>(hop + (size_t)r * d)[i] = u;
      } else {
        reinterpret_cast<float4*>(hop + (size_t)r * d)[i] = o;
      }
    }
  }
}

// The same arithmetic spread over a cluster of AN_CL blocks per row: block
// rank q runs virtual threads 64q .. 64q + 63, so each SM reads an eighth
// of the row's split-K slices (a lone block reading all of them competes on
// its SM with the next GEMM's weight stream, which starts while it runs).
// Every warp pushes its sum into all ranks' shared memory; after the
// cluster barrier each rank adds the 16 sums in order.
constexpr int AN_CL = 8;
constexpr int AN_CL_T = AN_VT / AN_CL;

__device__ __forceinline__ void an_push(float* local, unsigned rank, float v) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(local), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

template <typename T>
__global__ void __cluster_dims__(AN_CL, 1, 1) __launch_bounds__(AN_CL_T)
    k_addnorm_cl(int d, const float* h_in, float* h_out, const float* __restrict__ y, int S, size_t ps, int ldy,
                 T* hop, float* copy_out) {
  pdl_trigger();  // see common.cuh
  pdl_wait();
  __shared__ float red[AN_VT / 32];
  unsigned rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int r = blockIdx.x / AN_CL, v = (int)rank * AN_CL_T + threadIdx.x;
  float e[AN_CPT];
  const float ss = an_warp_tree(an_load(h_in + (size_t)r * d, y + (size_t)r * ldy, S, ps, d, v, e));
  if ((threadIdx.x & 31) == 0)
    for (unsigned q = 0; q < AN_CL; ++q) an_push(&red[v >> 5], q, ss);
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  const float inv = an_inv_from_warps(red);
#pragma unroll
  for (int c = 0; c < AN_CPT; ++c) {
    const int i = v + c * AN_VT;
    if (i < d) {
      const float o = e[c] * inv;
      h_out[(size_t)r * d + i] = o;
      hop[(size_t)r * d + i] = from_f<T>(o);
      if (copy_out) copy_out[(size_t)r * d + i] = o;
    }
  }
}

template <typename T>
cudaError_t launch_addnorm(int M, int d, const float* h_in, float* h_out, const float* y, int S, size_t ps, int ldy,
                           T* hop, float* copy_out, cudaStream_t st, bool any_order) {
  if (d > AN_CPT * AN_VT || S > AN_MAXS) return cudaErrorInvalidValue;
  // prefill rows: a warp per row with 16-byte accesses
  if (any_order && M > 64 && d % 4 == 0 && d <= 4 * 32 * ANR_V4 && ldy % 4 == 0 && ps % 4 == 0)
    return launch(k_addnorm_rows<T>, dim3((M + ANR_ROWS - 1) / ANR_ROWS), dim3(ANR_ROWS * 32), 0, st, M, d, h_in,
                  h_out, y, S, ps, ldy, hop, copy_out);
  // decode-sized batches: a cluster per row; long chunks: one block per row
  if (M <= 64) return launch(k_addnorm_cl<T>, dim3(M * AN_CL), dim3(AN_CL_T), 0, st, d, h_in, h_out, y, S, ps, ldy,
                             hop, copy_out);
  return launch(k_addnorm<T>, dim3(M), dim3(AN_VT), 0, st, d, h_in, h_out, y, S, ps, ldy, hop, copy_out);
}

// ------------------------------------------------------------------ loop boundary
template <typename T>
__global__ void k_reinject(int d, float* h, const float* x, int s_src, const float* s_in, bool make_u, T* hop,
                           float* stash_s, int rps, int scols, int col0) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[33];
  const int r = blockIdx.x;
  float* hr = h + (size_t)r * d;
  const float* xr = x + (size_t)r * d;
  float sv[16];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    int i = threadIdx.x + c * 256;
    sv[c] = 0.f;
    if (i < d) {
      sv[c] = s_src == 0 ? xr[i] : (s_src == 1 ? hr[i] : s_in[(size_t)r * d + i]);
      ss += sv[c] * sv[c];
    }
  }
  if (s_src == 1) {  // s = N(h)
    ss = block_sum(ss, red);
    const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
    for (int c = 0; c < 16; ++c) sv[c] *= inv;
  }
  if (stash_s) {
    size_t srow = (size_t)((r / rps) * scols + r % rps + col0) * d;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      int i = threadIdx.x + c * 256;
      if (i < d) stash_s[srow + i] = sv[c];
    }
  }
  if (make_u) {  // u = N(s + x)
    float uu = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      int i = threadIdx.x + c * 256;
      if (i < d) {
        sv[c] += xr[i];
        uu += sv[c] * sv[c];
      }
    }
    uu = block_sum(uu, red);
    const float inv = 1.f / fmaxf(sqrtf(uu), 1e-12f);
#pragma unroll
    for (int c = 0; c < 16; ++c) sv[c] *= inv;
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    int i = threadIdx.x + c * 256;
    if (i < d) {
      hr[i] = sv[c];
      hop[(size_t)r * d + i] = from_f<T>(sv[c]);
    }
  }
}

template <typename T>
cudaError_t launch_reinject(int M, int d, float* h, const float* x, int s_src, const float* s_in, bool make_u,
                            T* hop, float* stash_s, int rps, int scols, int col0, cudaStream_t st) {
  if (d > 16 * 256) return cudaErrorInvalidValue;
  launch(k_reinject<T>, M, 256, 0, st, d, h, x, s_src, s_in, make_u, hop, stash_s, rps, scols, col0);
  return cudaGetLastError();
}

__global__ void k_stash_copy(int d, float* state, float* stash, int rps, int scols, int col0, int dir) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  size_t srow = (size_t)((r / rps) * scols + r % rps + col0) * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    if (dir == 0)
      stash[srow + i] = state[(size_t)r * d + i];
    else
      state[(size_t)r * d + i] = stash[srow + i];
  }
}

cudaError_t launch_stash_copy(int M, int d, float* state, float* stash, int rps, int scols, int col0, int dir,
                              cudaStream_t st) {
  launch(k_stash_copy, M, 256, 0, st, d, state, stash, rps, scols, col0, dir);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ QKV split
template <typename T>
__global__ void k_qkv_post(int H, int KV, int hd, const float* qkv, int S, size_t ps, float* q_out, T* kscr,
                           T* vscr, bool direct, KVView kv, RowMeta m, int max_batch, bf16* qh, float qscale) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int qd = H * hd, kvd = KV * hd, ld = qd + 2 * kvd;
  const float* src = qkv + (size_t)r * ld;
  const int seq = m.seq[r], pos = m.pos[r];
  if (pos < 0 || pos >= kv.limit) {
    if (threadIdx.x == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
    return;
  }
  // four consecutive elements per thread (hd, and so every segment of the
  // row, is a multiple of 4; the row and slice strides keep 16-byte alignment)
  for (int i = 4 * threadIdx.x; i < ld; i += 4 * blockDim.x) {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
      const float4 b = *reinterpret_cast<const float4*>(src + s * ps + i);
      a[0] += b.x;
      a[1] += b.y;
      a[2] += b.z;
      a[3] += b.w;
    }
    if (i < qd) {
      if (qh) {  // the tensor-core attention reads only the scaled bf16 copy
        const __nv_bfloat162 lo = __floats2bfloat162_rn(a[0] * qscale, a[1] * qscale);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(a[2] * qscale, a[3] * qscale);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&lo);
        u.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(qh + (size_t)r * qd + i) = u;
      } else {
        *reinterpret_cast<float4*>(q_out + (size_t)r * qd + i) = make_float4(a[0], a[1], a[2], a[3]);
      }
    } else {
      int j = i - qd;
      const bool is_v = j >= kvd;
      if (is_v) j -= kvd;
      T* dst;
      if (direct) {
        const int g = j / hd, e = j % hd;
        dst = (is_v ? (T*)kv.V : (T*)kv.K) + kv_row(kv, seq, KV, g, pos) * hd + e;
      } else {
        dst = (is_v ? vscr : kscr) + (size_t)r * kvd + j;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = from_f<T>(a[e]);
    }
  }
  (void)max_batch;
}

template <typename T>
cudaError_t launch_qkv_post(int M, int H, int KV, int hd, const float* qkv, int S, size_t ps, float* q_out,
                            T* kscr, T* vscr, bool direct, KVView kv, RowMeta m, int max_batch, bf16* qh,
                            cudaStream_t st) {
  const float qscale = 1.4426950408889634f / sqrtf((float)hd);
  if (hd % 4 || ps % 4) return cudaErrorInvalidValue;
  launch(k_qkv_post<T>, M, 256, 0, st, H, KV, hd, qkv, S, ps, q_out, kscr, vscr, direct, kv, m, max_batch, qh,
         qscale);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ attention
// Block (row r, kv head g, key block b): 4 warps; each warp is 4 groups of 8
// lanes; group s of warp w takes keys kb + 4w + s + 16i; each lane of a group
// holds hd/8 dimensions.  Per group: online softmax (base-2) over its keys for
// the G query heads that share kv head g; groups are merged by a fixed xor
// tree, warps in index order.  Partial result: m, l, acc[hd] per head.
template <typename T, int HD, int G>
__global__ void __launch_bounds__(128) k_attn_partial(int KV, const float* __restrict__ q, const T* kscr,
                                                      const T* vscr, bool inchunk_scratch, KVView kv, RowMeta m,
                                                      float* __restrict__ part, int nb_max, float scale_log2) {
  pdl_wait();
  pdl_trigger();
  constexpr int DL = HD / 8;  // dims per lane
  __shared__ float sm_m[4][G], sm_l[4][G];
  __shared__ float sm_acc[4][G][HD];
  const int r = blockIdx.x / KV, g = blockIdx.x % KV;
  const int pos = m.pos[r], seq = m.seq[r], p0 = m.p0[r], base = m.base[r];
  if (pos < 0 || pos >= kv.limit) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
    return;
  }
  const int lo = kv.window > 0 ? max(0, pos - kv.window + 1) : 0;
  const int nb_row = pos / ATTN_BK - lo / ATTN_BK + 1;
  if (nb_row > nb_max) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
    return;
  }
  if ((int)blockIdx.y >= nb_row) return;
  const int ab = lo / ATTN_BK + blockIdx.y;
  const int klo = max(lo, ab * ATTN_BK), khi = min(pos, ab * ATTN_BK + ATTN_BK - 1);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, sg = lane >> 3, dl = lane & 7;
  const int H = KV * G;
  const int qd = H * HD, kvd = KV * HD;

  float qv[G][DL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DL; ++e) qv[h][e] = q[(size_t)r * qd + (g * G + h) * HD + dl * DL + e] * scale_log2;

  float mx[G], ls[G], acc[G][DL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mx[h] = -FLT_MAX;
    ls[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[h][e] = 0.f;
  }
  const T* Kc = (const T*)kv.K;
  const T* Vc = (const T*)kv.V;
  const int kb = ab * ATTN_BK;
  for (int jq = kb + 4 * w; jq <= khi; jq += 16) {
    const int j = jq + sg;
    const bool valid = j >= klo && j <= khi;
    float kf[DL], vf[DL];
    if (valid) {
      const T *kp, *vp;
      if (inchunk_scratch && j >= p0) {
        size_t row = (size_t)(base + (j - p0));
        kp = kscr + row * kvd + g * HD;
        vp = vscr + row * kvd + g * HD;
      } else {
        size_t idx = kv_row(kv, seq, KV, g, j) * HD;
        kp = Kc + idx;
        vp = Vc + idx;
      }
#pragma unroll
      for (int e = 0; e < DL; ++e) {
        kf[e] = to_f(kp[dl * DL + e]);
        vf[e] = to_f(vp[dl * DL + e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < DL; ++e) kf[e] = vf[e] = 0.f;
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
        float mn = fmaxf(mx[h], sdot);
        float corr = exp2f(mx[h] - mn);
        float p = exp2f(sdot - mn);
        ls[h] = ls[h] * corr + p;
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[h][e] = acc[h][e] * corr + p * vf[e];
        mx[h] = mn;
      }
    }
  }
  // merge the 4 groups of the warp (xor 8, then 16)
#pragma unroll
  for (int off = 8; off <= 16; off <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float om = __shfl_xor_sync(0xffffffffu, mx[h], off);
      float ol = __shfl_xor_sync(0xffffffffu, ls[h], off);
      float mn = fmaxf(mx[h], om);
      float ca = (mx[h] == -FLT_MAX) ? 0.f : exp2f(mx[h] - mn);
      float cb = (om == -FLT_MAX) ? 0.f : exp2f(om - mn);
      ls[h] = ls[h] * ca + ol * cb;
#pragma unroll
      for (int e = 0; e < DL; ++e) {
        float oa = __shfl_xor_sync(0xffffffffu, acc[h][e], off);
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
  // merge warps 0..3 in order; thread t handles (head, dim) pairs
  for (int idx = threadIdx.x; idx < G * (HD + 2); idx += blockDim.x) {
    const int h = idx / (HD + 2), c = idx % (HD + 2);
    float M = -FLT_MAX;
#pragma unroll
    for (int ww = 0; ww < 4; ++ww) M = fmaxf(M, sm_m[ww][h]);
    float val = 0.f;
    if (c == 0) {
      val = M;
    } else {
#pragma unroll
      for (int ww = 0; ww < 4; ++ww) {
        float sc = sm_m[ww][h] == -FLT_MAX ? 0.f : exp2f(sm_m[ww][h] - M);
        val += (c == 1 ? sm_l[ww][h] : sm_acc[ww][h][c - 2]) * sc;
      }
    }
    const int head = g * G + h;
    part[(((size_t)r * H + head) * nb_max + blockIdx.y) * (HD + 2) + c] = val;
  }
}

// One warp per (row, head): merge the row's key blocks in order.
template <typename T, int HD>
__global__ void k_attn_combine(int H, const float* __restrict__ part, int nb_max, KVView kv, RowMeta m, T* out) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x, head = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (head >= H) return;
  const int lane = threadIdx.x & 31;
  const int pos = m.pos[r];
  const int lo = kv.window > 0 ? max(0, pos - kv.window + 1) : 0;
  const int nb = pos / ATTN_BK - lo / ATTN_BK + 1;
  constexpr int DPL0 = HD / 32;
  if (pos < 0 || pos >= kv.limit || nb > nb_max) {  // rejected by the partial kernel
#pragma unroll
    for (int e = 0; e < DPL0; ++e) out[(size_t)r * H * HD + head * HD + lane * DPL0 + e] = from_f<T>(0.f);
    return;
  }
  const float* pr = part + ((size_t)r * H + head) * nb_max * (HD + 2);
  float M = -FLT_MAX;
  for (int b = 0; b < nb; ++b) M = fmaxf(M, pr[b * (HD + 2)]);
  constexpr int DPL = HD / 32;
  float L = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int b = 0; b < nb; ++b) {
    const float* pb = pr + b * (HD + 2);
    float sc = exp2f(pb[0] - M);
    L += pb[1] * sc;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] += pb[2 + lane * DPL + e] * sc;
  }
  const float inv = 1.f / L;
#pragma unroll
  for (int e = 0; e < DPL; ++e) out[(size_t)r * H * HD + head * HD + lane * DPL + e] = from_f<T>(acc[e] * inv);
}

template <typename T, int HD, int G>
static cudaError_t attn_dispatch(int M, int KV, const float* q, const T* kscr, const T* vscr, bool sc, KVView kv,
                                 RowMeta m, int nb, float* part, T* out, cudaStream_t st) {
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  dim3 grid(M * KV, nb);
  launch(k_attn_partial<T, HD, G>, grid, 128, 0, st, KV, q, kscr, vscr, sc, kv, m, part, nb, scale_log2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int H = KV * G;
  dim3 g2(M, (H + 3) / 4);
  launch(k_attn_combine<T, HD>, g2, 128, 0, st, H, part, nb, kv, m, out);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_attention(int M, int H, int KV, int hd, const float* q, const T* kscr, const T* vscr,
                             bool sc, KVView kv, RowMeta m, int max_ctx, float* part, int part_rows, T* out,
                             cudaStream_t st) {
  int span = kv.window > 0 ? min(max_ctx, kv.window) : max_ctx;
  int nb = (span + ATTN_BK - 1) / ATTN_BK + 1;
  const int G = H / KV;
  if (part_rows <= 0) return cudaErrorInvalidValue;
  // rows are independent: long chunks run in slices of part_rows rows that
  // reuse the partial buffer (chunk keys are addressed by m.base, absolute)
  for (int r0 = 0; r0 < M; r0 += part_rows) {
    const int n = min(part_rows, M - r0);
    RowMeta ms{m.seq + r0, m.pos + r0, m.p0 + r0, m.base + r0, m.pend + r0};
    const float* qs = q + (size_t)r0 * H * hd;
    T* os = out + (size_t)r0 * H * hd;
    cudaError_t e = cudaErrorInvalidValue;
#define DORY_ATTN_CASE(HDV, GV) \
  if (hd == HDV && G == GV) e = attn_dispatch<T, HDV, GV>(n, KV, qs, kscr, vscr, sc, kv, ms, nb, part, os, st);
    DORY_ATTN_CASE(32, 1) DORY_ATTN_CASE(32, 2) DORY_ATTN_CASE(32, 4) DORY_ATTN_CASE(32, 5) DORY_ATTN_CASE(32, 8)
    DORY_ATTN_CASE(64, 1) DORY_ATTN_CASE(64, 2) DORY_ATTN_CASE(64, 4) DORY_ATTN_CASE(64, 5) DORY_ATTN_CASE(64, 8)
    DORY_ATTN_CASE(128, 1) DORY_ATTN_CASE(128, 2) DORY_ATTN_CASE(128, 4) DORY_ATTN_CASE(128, 5)
#undef DORY_ATTN_CASE
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T>
__global__ void k_kv_commit(int KV, int hd, const T* kscr, const T* vscr, KVView kv, RowMeta m) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int pos = m.pos[r], pend = m.pend[r], seq = m.seq[r];
  if (pos < pend - kv.cap) return;  // overwritten later in this chunk
  if (pos < 0 || pos >= kv.limit) {
    if (threadIdx.x == 0) set_error(kv.err, DEV_ERR_BAD_INDEX);
    return;
  }
  const int kvd = KV * hd;
  for (int j = threadIdx.x; j < kvd; j += blockDim.x) {
    int g = j / hd, e = j % hd;
    size_t off = kv_row(kv, seq, KV, g, pos) * hd + e;
    ((T*)kv.K)[off] = kscr[(size_t)r * kvd + j];
    ((T*)kv.V)[off] = vscr[(size_t)r * kvd + j];
  }
}

template <typename T>
cudaError_t launch_kv_commit(int M, int KV, int hd, const T* kscr, const T* vscr, KVView kv, RowMeta m,
                             cudaStream_t st) {
  launch(k_kv_commit<T>, M, 128, 0, st, KV, hd, kscr, vscr, kv, m);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ SwiGLU
template <typename T>
__global__ void k_swiglu(int dff, const float* gu, int S, size_t ps, T* act) {
  pdl_trigger();  // see common.cuh
  pdl_wait();
  const int r = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= dff) return;
  const float* row = gu + (size_t)r * 2 * dff;
  float g = 0.f, u = 0.f;
  for (int s = 0; s < S; ++s) {
    g += row[s * ps + i];
    u += row[s * ps + dff + i];
  }
  float a = g / (1.f + expf(-g)) * u;
  act[(size_t)r * dff + i] = from_f<T>(a);
}

template <typename T>
cudaError_t launch_swiglu(int M, int dff, const float* gu, int S, size_t ps, T* act, cudaStream_t st) {
  dim3 grid((dff + 255) / 256, M);
  launch(k_swiglu<T>, grid, 256, 0, st, dff, gu, S, ps, act);
  return cudaGetLastError();
}

template <typename T>
__global__ void k_gather_rows(int d, const int* rows, const T* src, T* dst) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const T* s = src + (size_t)rows[r] * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) dst[(size_t)r * d + i] = s[i];
}

template <typename T>
cudaError_t launch_gather_rows(int R, int d, const int* rows, const T* src, T* dst, cudaStream_t st) {
  launch(k_gather_rows<T>, R, 256, 0, st, d, rows, src, dst);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ SIMT GEMM
// 64 (m) x 64 (n) tile per 256-thread block, k tile 16; each thread 4x4
// outputs accumulated in increasing k.
template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(int M, int N, int K, const T* __restrict__ X, int ldx,
                                                   const T* __restrict__ W, float* __restrict__ Y, int ldy) {
  pdl_wait();
  pdl_trigger();
  __shared__ float xs[16][64 + 4];
  __shared__ float ws[16][64 + 4];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      int rr = i / 16, kk = i % 16;
      int gm = m0 + rr, gn = n0 + rr, gk = k0 + kk;
      xs[kk][rr] = (gm < M && gk < K) ? to_f(X[(size_t)gm * ldx + gk]) : 0.f;
      ws[kk][rr] = (gn < N && gk < K) ? to_f(W[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn < N) Y[(size_t)gm * ldy + gn] = acc[i][j];
    }
  }
}

template <typename T>
cudaError_t launch_gemm_simt(int M, int N, int K, const T* X, int ldx, const T* W, float* Y, int ldy,
                             cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  launch(k_gemm_simt<T>, grid, 256, 0, st, M, N, K, X, ldx, W, Y, ldy);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ argmax
// One block per row; per-thread running (max, lowest index) over 16-byte
// loads (8 in flight per thread) when every row starts 16-byte aligned, then
// a fixed tree.  max with lowest-index ties is order independent.
constexpr int AM_THREADS = 1024;

__device__ __forceinline__ void am_take(float v, int i, float& best, int& bi) {
  if (v > best || (v == best && i < bi)) {
    best = v;
    bi = i;
  }
}

__global__ void __launch_bounds__(AM_THREADS) k_argmax(int V, const float* logits, int* out, bool vec) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sv[AM_THREADS / 32];
  __shared__ int si[AM_THREADS / 32];
  const float* x = logits + (size_t)blockIdx.x * V;
  float best = -FLT_MAX;
  int bi = 0x7fffffff;
  if (vec) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int n4 = V / 4;
#pragma unroll 8
    for (int i = threadIdx.x; i < n4; i += AM_THREADS) {
      const float4 v = x4[i];
      am_take(v.x, 4 * i, best, bi);
      am_take(v.y, 4 * i + 1, best, bi);
      am_take(v.z, 4 * i + 2, best, bi);
      am_take(v.w, 4 * i + 3, best, bi);
    }
  } else {
    for (int i = threadIdx.x; i < V; i += AM_THREADS) am_take(x[i], i, best, bi);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    am_take(ov, oi, best, bi);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sv[w] = best;
    si[w] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < AM_THREADS / 32; ++i) am_take(sv[i], si[i], best, bi);
    out[blockIdx.x] = bi;
  }
}

cudaError_t launch_argmax(int R, int V, const float* logits, int* out, cudaStream_t st) {
  const bool vec = (V & 3) == 0 && ((uintptr_t)logits & 15) == 0;
  launch(k_argmax, R, AM_THREADS, 0, st, V, logits, out, vec);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ speculative acceptance
__global__ void k_spec_accept(int B, int gamma, int dstride, const int* seq_ids, int* seq_len, const int* drafts,
                              const int* vtok, int* pending, const SpecIo* io, unsigned long long* accepted,
                              int* flags, const int* err, cudaGraphConditionalHandle cond, int use_cond) {
  pdl_wait();
  pdl_trigger();
  __shared__ int n_unfinished;
  if (threadIdx.x == 0) n_unfinished = 0;
  __syncthreads();
  int* out = io->out;
  int* out_len = io->out_len;
  const int max_new = io->max_new;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    int ol = out_len[b];
    if (ol >= max_new) continue;  // finished: cache and length stay frozen
    const int* a = vtok + b * (gamma + 1);
    int n = 0;
    while (n < gamma && a[n] == drafts[n * dstride + b]) ++n;
    for (int i = 0; i < n && ol < max_new; ++i) out[b * max_new + ol++] = drafts[i * dstride + b];
    if (ol < max_new) out[b * max_new + ol++] = a[n];
    out_len[b] = ol;
    seq_len[seq_ids[b]] += n + 1;
    pending[b] = a[n];
    atomicAdd(accepted, (unsigned long long)n);
    if (ol < max_new) atomicAdd(&n_unfinished, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // every step gives each unfinished sequence at least one token, so
    // max_new steps finish every sequence; one more means something is wrong
    const int done = n_unfinished == 0, steps = flags[1] + 1;
    const int overrun = !done && steps > max_new;
    flags[0] = done;
    flags[1] = steps;
    if (overrun) flags[2] = 1;
    if (use_cond) cudaGraphSetConditional(cond, (done || overrun || *(volatile const int*)err != 0) ? 0u : 1u);
  }
}

cudaError_t launch_spec_accept(int B, int gamma, int dstride, const int* seq_ids, int* seq_len, const int* drafts,
                               const int* vtok, int* pending, const SpecIo* io, unsigned long long* accepted,
                               int* flags, const int* err, unsigned long long cond, bool use_cond,
                               cudaStream_t st) {
  launch(k_spec_accept, 1, 256, 0, st, B, gamma, dstride, seq_ids, seq_len, drafts, vtok, pending, io, accepted,
         flags, err, (cudaGraphConditionalHandle)cond, use_cond ? 1 : 0);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ instantiations
#define DORY_INST(T)                                                                                              \
  template cudaError_t launch_embed<T>(int, int, int, const int*, const T*, float*, T*, float*, int*,            \
                                       cudaStream_t);                                                             \
  template cudaError_t launch_addnorm<T>(int, int, const float*, float*, const float*, int, size_t, int, T*,      \
                                         float*, cudaStream_t, bool);                                             \
  template cudaError_t launch_reinject<T>(int, int, float*, const float*, int, const float*, bool, T*, float*,    \
                                          int, int, int, cudaStream_t);                                           \
  template cudaError_t launch_qkv_post<T>(int, int, int, int, const float*, int, size_t, float*, T*, T*, bool,    \
                                          KVView, RowMeta, int, bf16*, cudaStream_t);                             \
  template cudaError_t launch_attention<T>(int, int, int, int, const float*, const T*, const T*, bool, KVView,    \
                                           RowMeta, int, float*, int, T*, cudaStream_t);                          \
  template cudaError_t launch_kv_commit<T>(int, int, int, const T*, const T*, KVView, RowMeta, cudaStream_t);     \
  template cudaError_t launch_swiglu<T>(int, int, const float*, int, size_t, T*, cudaStream_t);                   \
  template cudaError_t launch_gather_rows<T>(int, int, const int*, const T*, T*, cudaStream_t);                   \
  template cudaError_t launch_gemm_simt<T>(int, int, int, const T*, int, const T*, float*, int, cudaStream_t);
DORY_INST(float)
DORY_INST(bf16)
#undef DORY_INST

}  // namespace dory

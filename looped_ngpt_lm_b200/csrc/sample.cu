// Temperature / top-p sampling, one 1024-thread block per row.  The released
// model's settings are temperature 1.0 and top-p 0.95 (lucasainews.com,
// "NVIDIA, 루프 구조 4B 모델 Dory1.0-4B 4가지 정밀도로 공개", "How to run");
// the pages give no procedure, and the one below is this library's reading.
//
// The draw for a row is Philox4x32 with 10 rounds (Salmon, Moraes, Dror and
// Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011), key = the
// 64-bit seed, counter = (sequence id, position of the new token, 0, 0):
// u = (first word >> 8) / 2^24.  The masses are integers,
// q_i = floor(exp2((l_i - max) * log2(e) / T) * 2^31); the nucleus is every
// token with q_i >= tau, tau the largest value whose tail mass reaches
// ceil(top_p * sum q); the token is the first index (in token order) at which
// the running nucleus mass exceeds floor(u * M), M the nucleus mass.  Every
// sum is an integer sum, so the result does not depend on the order of the
// parallel reductions.
#include <float.h>

#include "kernels.cuh"

namespace dory {

namespace {

constexpr int SP_T = 1024;  // threads per row
constexpr int SP_W = SP_T / 32;

__device__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;  // key increments: golden ratio and sqrt(3) - 1 in 32-bit fixed point
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// block-wide sum of an unsigned 64-bit value (every thread gets the total)
__device__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long* red) {
  v = warp_sum_u64(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  v = lane < SP_W ? red[lane] : 0ull;
  return warp_sum_u64(v);
}

// seq[row], pos[row] (+ pos_add): the draw's counter; rows (optional) maps a
// row to its index in seq / pos.
__global__ void __launch_bounds__(SP_T) k_sample(int V, const float* logits, uint32_t* qbuf, const int* rows,
                                                 const int* seq, const int* pos, int pos_add, float scale,
                                                 double top_p, uint32_t k0, uint32_t k1, int* out, bool vec) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ unsigned long long hist[];  // [SP_W][256] per-warp histograms
  __shared__ unsigned long long red[SP_W];
  __shared__ float redf[SP_W];
  __shared__ unsigned long long s_above;
  __shared__ uint32_t s_prefix;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x, mr = rows ? rows[row] : row;
  const float* l = logits + (size_t)row * V;
  uint32_t* q = qbuf + (size_t)row * V;

  // Passes over the row read 16 bytes per thread and keep 8 loads in flight
  // (vec: V % 4 == 0 and 16-byte aligned rows); the single block per row is
  // otherwise bound by L2 latency.
  const int V4 = vec ? V / 4 : 0;
  const float4* l4 = reinterpret_cast<const float4*>(l);
  uint4* q4 = reinterpret_cast<uint4*>(q);

  // 1. max
  float mx = -FLT_MAX;
#pragma unroll 8
  for (int i = tid; i < V4; i += SP_T) {
    const float4 v = l4[i];
    mx = fmaxf(fmaxf(mx, v.x), fmaxf(v.y, fmaxf(v.z, v.w)));
  }
  for (int i = 4 * V4 + tid; i < V; i += SP_T) mx = fmaxf(mx, l[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) redf[w] = mx;
  __syncthreads();
  mx = lane < SP_W ? redf[lane] : -FLT_MAX;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));

  // 2. integer masses (in place when q aliases the logits: each element is
  // read and written by the same thread)
  unsigned long long Q = 0;
  auto mass = [&](float x) { return (uint32_t)floorf(exp2f((x - mx) * scale) * 2147483648.f); };
#pragma unroll 4
  for (int i = tid; i < V4; i += SP_T) {
    const float4 v = l4[i];
    const uint4 o = make_uint4(mass(v.x), mass(v.y), mass(v.z), mass(v.w));
    q4[i] = o;
    Q += (unsigned long long)o.x + o.y + o.z + o.w;
  }
  for (int i = 4 * V4 + tid; i < V; i += SP_T) {
    const uint32_t qi = mass(l[i]);
    q[i] = qi;
    Q += qi;
  }
  Q = block_sum_u64(Q, red);
  const unsigned long long P = (unsigned long long)ceil(top_p * (double)Q);

  // 3. tau: a byte at a time from the top, within the elements that share the
  // bytes chosen so far; `above` is the mass of the elements above that range
  uint32_t prefix = 0;
  unsigned long long above = 0;
  unsigned long long* h = hist + w * 256;
  for (int b = 3; b >= 0; --b) {
    for (int i = lane; i < 256; i += 32) h[i] = 0ull;
    __syncthreads();
    // digit 0 is the crowded bin (most masses are small): it is summed in a
    // register and reduced once instead of serialising shared atomics
    unsigned long long z = 0;
    auto take = [&](uint32_t qi) {
      if (qi != 0u && ((unsigned long long)qi >> (8 * b + 8)) == prefix) {
        const uint32_t dg = (qi >> (8 * b)) & 255u;
        if (dg == 0u)
          z += qi;
        else
          atomicAdd(&h[dg], (unsigned long long)qi);
      }
    };
#pragma unroll 8
    for (int i = tid; i < V4; i += SP_T) {
      const uint4 v = q4[i];
      take(v.x);
      take(v.y);
      take(v.z);
      take(v.w);
    }
    for (int i = 4 * V4 + tid; i < V; i += SP_T) take(q[i]);
    z = block_sum_u64(z, red);  // includes a barrier: every histogram is complete
    if (tid == 0) h[0] += z;   // warp 0's table, digit 0
    // merge the per-warp histograms into warp 0's
    for (int d = tid; d < 256; d += SP_T) {
      unsigned long long s = 0;
      for (int ww = 0; ww < SP_W; ++ww) s += hist[ww * 256 + d];
      hist[d] = s;
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long acc = above;
      int d = 255;
      for (; d > 0; --d) {
        if (acc + hist[d] >= P) break;
        acc += hist[d];
      }
      s_above = acc;
      s_prefix = (prefix << 8) | (uint32_t)d;
    }
    __syncthreads();
    prefix = s_prefix;
    above = s_above;
  }
  const uint32_t tau = prefix;

  // 4. nucleus mass, one contiguous range of tokens per thread
  const int C = ((V + SP_T - 1) / SP_T + 3) & ~3, i0 = min(V, tid * C), i1 = min(V, i0 + C);
  unsigned long long local = 0;
  if (vec) {
#pragma unroll 8
    for (int i = i0; i < i1; i += 4) {  // i0, i1 multiples of 4 when vec
      const uint4 v = q4[i / 4];
      local += (v.x >= tau ? v.x : 0u) + (unsigned long long)(v.y >= tau ? v.y : 0u) +
               (v.z >= tau ? v.z : 0u) + (unsigned long long)(v.w >= tau ? v.w : 0u);
    }
  } else {
    for (int i = i0; i < i1; ++i) {
      const uint32_t qi = q[i];
      if (qi >= tau) local += qi;
    }
  }
  // exclusive prefix of `local` over the threads (warp scan, then warp totals)
  unsigned long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  __syncthreads();
  if (lane == 31) red[w] = incl;
  __syncthreads();
  if (w == 0) {
    unsigned long long t = red[lane], ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long v = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += v;
    }
    red[lane] = ti - t;  // exclusive prefix of the warp totals
  }
  __syncthreads();
  const unsigned long long base = red[w] + incl - local;

  // 5. the draw and the token: the thread whose range holds the target scans it
  __shared__ unsigned long long s_total;  // M, the nucleus mass
  if (tid == SP_T - 1) s_total = base + local;
  __syncthreads();
  const unsigned long long total = s_total;
  const uint32_t word = philox_word0((uint32_t)seq[mr], (uint32_t)(pos[mr] + pos_add), 0u, 0u, k0, k1);
  const unsigned long long r = (unsigned long long)(((unsigned __int128)(word >> 8) * total) >> 24);
  if (local > 0 && base <= r && r < base + local) {
    // the owner walks its range in batches of 32 values loaded at once
    unsigned long long run = base;
    bool found = false;
    for (int j0 = i0; j0 < i1 && !found; j0 += 32) {
      uint32_t buf[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) buf[t] = j0 + t < i1 ? q[j0 + t] : 0u;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        if (!found && buf[t] >= tau && buf[t] != 0u) {
          run += buf[t];
          if (run > r) {
            out[row] = j0 + t;
            found = true;
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_sample(int R, int V, const float* logits, uint32_t* qbuf, const int* rows, const int* seq,
                          const int* pos, int pos_add, float temperature, float top_p, unsigned long long seed,
                          int* out, cudaStream_t st) {
  if (R <= 0 || V <= 0 || !(temperature > 0.f) || !(top_p > 0.f) || top_p > 1.f) return cudaErrorInvalidValue;
  const float scale = (float)(1.4426950408889634 / (double)temperature);
  constexpr int SMEM = SP_W * 256 * 8;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_sample, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const bool vec = V % 4 == 0 && ((uintptr_t)logits & 15) == 0 && ((uintptr_t)qbuf & 15) == 0;
  launch(k_sample, R, SP_T, SMEM, st, V, logits, qbuf, rows, seq, pos, pos_add, scale, (double)top_p,
         (uint32_t)(seed & 0xFFFFFFFFull), (uint32_t)(seed >> 32), out, vec);
  return cudaGetLastError();
}

}  // namespace dory

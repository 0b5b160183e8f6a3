// Launchers of the looped nGPT kernels.  Every launcher queues work on
// `stream` and returns the launch status; none allocates memory.
#pragma once

#include "common.cuh"

namespace dory {

// Per-row metadata of one forward chunk (device arrays of n_rows entries).
//   seq  : sequence slot of the row
//   pos  : absolute position of the row's token
//   p0   : first position of this sequence's rows in the chunk
//   base : chunk row index of this sequence's first row
//   pend : p0 + (rows of this sequence in the chunk)
struct RowMeta {
  int* seq;
  int* pos;
  int* p0;
  int* base;
  int* pend;
};

// One attention layer's cache for one slot: K, V of shape
// [max_batch][n_kv][cap][head_dim] in the storage type.  window == 0 means
// full causal attention, otherwise keys p-window < j <= p.  Position j lives
// at index j % cap (a ring for sliding-window layers, cap >= max_seq for full).
//
// Paged full-attention layers (pt != NULL): positions come in pages of
// 2^page_shift; page table pt[seq * pt_stride + j >> page_shift] names the
// page holding position j, and K, V are [pages][n_kv][2^page_shift][head_dim].
struct KVView {
  void* K;
  void* V;
  int cap;
  int window;
  int limit;  // max_seq: positions >= limit are rejected (error word set)
  int* err;   // device error word
  const int* pt = nullptr;
  int pt_stride = 0;
  int page_shift = 0;
};

// Row index (in head_dim-element rows) of position j of sequence seq, KV
// head g, in K or V of the layer.
__device__ __forceinline__ size_t kv_row(const KVView& kv, int seq, int n_kv, int g, int j) {
  if (kv.pt) {
    const int page = kv.pt[(size_t)seq * kv.pt_stride + (j >> kv.page_shift)];
    return (((size_t)page * n_kv + g) << kv.page_shift) + (size_t)(j & ((1 << kv.page_shift) - 1));
  }
  return ((size_t)seq * n_kv + g) * kv.cap + (size_t)(j % kv.cap);
}

// ---- chunk planning (device-side row metadata) ---------------------------
cudaError_t launch_plan_uniform(int n_seq, int rows_per_seq, int pos_offset, const int* seq_ids,
                                const int* seq_len, RowMeta m, cudaStream_t st);
cudaError_t launch_plan_ragged(int n_seq, int n_rows, const int* cu_rows, const int* seq_ids,
                               const int* seq_len, RowMeta m, cudaStream_t st);
cudaError_t launch_advance(int n_seq, const int* seq_ids, int* seq_len, int delta, cudaStream_t st);
// seq_len[seq_ids[b]] += cu[b+1] - cu[b]
cudaError_t launch_advance_ragged(int n_seq, const int* seq_ids, const int* cu, int* seq_len, cudaStream_t st);

// ---- elementwise / normalisation -----------------------------------------
// h <- E[token] (fp32), hop <- E[token]; x (if not NULL) <- the same rows.
template <typename T>
cudaError_t launch_embed(int M, int d, int vocab, const int* tokens, const T* E, float* h, T* hop, float* x,
                         int* err, cudaStream_t st);
// h_out <- N(h_in + sum_{s<S} y[s]) ; hop <- (T)h_out ; copy_out (if not NULL)
// <- h_out (h_out may equal h_in).  y[s] = y + s*part_stride, rows of ldy.
// S <= kMaxSplitK; d, ldy and part_stride multiples of 4.  Rows take the
// 512-virtual-thread arithmetic of addnorm.cuh (the bits a decode row and
// the same row of a speculative chunk share) unless any_order: then long
// batches of rows (prefill chunks) may use a faster summation order.
template <typename T>
cudaError_t launch_addnorm(int M, int d, const float* h_in, float* h_out, const float* y, int S,
                           size_t part_stride, int ldy, T* hop, float* copy_out, cudaStream_t st,
                           bool any_order = false);
// Loop boundary.  s_src: 0 -> s = x ; 1 -> s = N(h) ; 2 -> s = s_in.
// If make_u: out = N(s + x), else out = s.  h <- out, hop <- (T)out.
// If s_save: s_save <- s.  stash rows: when stash_x/stash_s are given, row r
// also copies x / s into stash[(r / rps) * stash_cols + r % rps + col0].
template <typename T>
cudaError_t launch_reinject(int M, int d, float* h, const float* x, int s_src, const float* s_in,
                            bool make_u, T* hop, float* stash_s, int rps, int stash_cols, int col0,
                            cudaStream_t st);
// Copy rows between the x/s state and the speculative stash (dir 0: state ->
// stash, 1: stash -> state).
cudaError_t launch_stash_copy(int M, int d, float* state, float* stash, int rps, int stash_cols, int col0,
                              int dir, cudaStream_t st);

// Split q/k/v out of the QKV projection (sum of S partials).  q -> fp32 q_out
// [M, H*hd] (and, when qh is not NULL, bf16 q * log2(e)/sqrt(hd) into qh);
// k, v rounded to T -> scratch [M, KV*hd] (direct == false) or straight into
// the cache at pos % cap (direct == true).
template <typename T>
cudaError_t launch_qkv_post(int M, int H, int KV, int hd, const float* qkv, int S, size_t part_stride,
                            float* q_out, T* kscr, T* vscr, bool direct, KVView kv, RowMeta m,
                            int max_batch, bf16* qh, cudaStream_t st);

// GQA attention over the cache (+ chunk scratch), split over absolute key
// blocks of ATTN_BK positions, then merged in block order.  part holds the
// block partials of part_rows rows; longer chunks run in row slices.
constexpr int ATTN_BK = 256;
template <typename T>
cudaError_t launch_attention(int M, int H, int KV, int hd, const float* q, const T* kscr, const T* vscr,
                             bool inchunk_scratch, KVView kv, RowMeta m, int max_ctx, float* part,
                             int part_rows, T* out, cudaStream_t st);
// Copy chunk K/V from scratch into the cache (positions >= pend - cap).
template <typename T>
cudaError_t launch_kv_commit(int M, int KV, int hd, const T* kscr, const T* vscr, KVView kv, RowMeta m,
                             cudaStream_t st);

// act[m, i] = silu(sum_s g) * sum_s u, g = column i, u = column dff + i.
template <typename T>
cudaError_t launch_swiglu(int M, int dff, const float* gu, int S, size_t part_stride, T* act,
                          cudaStream_t st);

template <typename T>
cudaError_t launch_gather_rows(int R, int d, const int* rows, const T* src, T* dst, cudaStream_t st);

// Y[m, n] = sum_k X[m, k] W[n, k] with fp32 accumulation in increasing k
// (identical for every M).  X rows of ldx elements, Y rows of ldy floats.
template <typename T>
cudaError_t launch_gemm_simt(int M, int N, int K, const T* X, int ldx, const T* W, float* Y, int ldy,
                             cudaStream_t st);

// Greedy choice per row (largest logit, lowest id on ties).
cudaError_t launch_argmax(int R, int V, const float* logits, int* out, cudaStream_t st);
// Temperature / top-p sampling of R rows of V logits (see sample.cu): the
// draw of row i uses counter (seq[m], pos[m] + pos_add) with m = rows ? rows[i]
// : i; qbuf: [R, V] uint32 scratch (may alias the logits).  out: token ids.
cudaError_t launch_sample(int R, int V, const float* logits, uint32_t* qbuf, const int* rows, const int* seq,
                          const int* pos, int pos_add, float temperature, float top_p, unsigned long long seed,
                          int* out, cudaStream_t st);

// Caller buffers of a speculative decoding call (device copy, so a recorded
// step reads each call's buffers).
struct SpecIo {
  int* out;      // [B, max_new] accepted tokens
  int* out_len;  // [B]
  int max_new;
  int pad;
};

// Speculative acceptance for B sequences.  drafts[i * dstride + b] = d_{i+1},
// vtok [B, gamma+1] verifier choices.  Appends accepted tokens to io->out
// [B, max_new] at io->out_len, sets seq_len = p0 + n + 1 and pending = a_n
// for unfinished sequences; adds n to *accepted (device int64).  flags[0] <-
// every sequence finished; flags[1] counts steps; flags[2] <- 1 once more
// steps ran than max_new (which always suffice).  With use_cond the kernel
// sets graph conditional `cond` to 1 while another step is needed (no
// sequence finished everything, no step bound hit, error word err clear).
cudaError_t launch_spec_accept(int B, int gamma, int dstride, const int* seq_ids, int* seq_len,
                               const int* drafts, const int* vtok, int* pending, const SpecIo* io,
                               unsigned long long* accepted, int* flags, const int* err, unsigned long long cond,
                               bool use_cond, cudaStream_t st);

cudaError_t launch_fill_i32(int n, int* p, int v, cudaStream_t st);

// out[m, n] = sum_{s<S} part[s * ps + m * N + n] in order s = 0..S-1 (out may alias part).
cudaError_t launch_split_reduce(int M, int N, const float* part, int S, size_t ps, float* out, cudaStream_t st);

}  // namespace dory

/*
 * dory.h -- C ABI of the looped normalized-GPT inference library (libdory.so).
 *
 * The library runs the per-token forward of a looped nGPT language model on
 * one NVIDIA B200 (sm_100a): an input block run once, a shared recurrent block
 * run k times with the input re-injected every loop, an output block and an
 * LM head, over a KV cache in last-loop or per-loop mode.
 *
 * Sources (web pages about Dory1.0-4B; section names translated):
 *   [digest]  onedev.kr/papers/1692 "Dory1.0-4B는 반복 횟수로 추론 연산과
 *             정확도를 조절한다": "How it works" (block split, recurrence
 *             s0=x, u_t=N(s_{t-1}+x), s_t=N(F(u_t)), 72/112/192 layer
 *             applications, 36 MLP / 27 sliding-window / 9 full attention
 *             layers), "Premises & limits" (last-loop KV caching and its
 *             final-loop mismatch; self-speculative decoding with draft k=1,
 *             verify k=4, gamma=4, KV and activation reuse).
 *   [news]    lucasainews.com "NVIDIA, 루프 구조 4B 모델 Dory1.0-4B 4가지
 *             정밀도로 공개": "Looped structure" (input re-injected every loop),
 *             "How to run" (loop count 1..4 chosen at inference; the
 *             recurrent KV cache mode switch last_loop / per-loop).
 *   [trawling] trawling.dev/post/2766 "NVIDIA, 반복 연산형 4B 언어 모델 Dory
 *             공개": "KV 캐시와 실행 환경" (KV cache and runtime: the
 *             released weight formats BF16, MXFP8, NVFP4, Q5_K_M; MXFP8
 *             decodes 1.69x to 1.84x faster than BF16 at batch 1).
 *   [review]  blog.secrett2633.cloud "[논문리뷰] Dory1.0-4B: A Looped
 *             Normalized-GPT", "1. Key Terms" (nGPT: L2-normalised states;
 *             last-loop KV caching keeps the footprint of one loop).
 *
 * Conventions for every entry point:
 *   - Return DORY_OK or an error status; dory_last_error(h) gives the message.
 *   - Arguments are validated before any work is queued: an error leaves the
 *     handle and its caches unchanged.
 *   - Pointers marked "device" are CUDA device pointers, "host" are host
 *     pointers.  The caller owns every buffer it passes; the library keeps no
 *     pointer past the call except the weights and workspace given to
 *     dory_create, which must outlive the handle.
 *   - Work is queued on the caller's stream (a cudaStream_t passed as
 *     dory_stream; NULL is the legacy default stream) and returns before it
 *     finishes, except where a function says it synchronises.
 *   - The library never allocates device memory: all device state lives in
 *     the caller-provided workspace.
 *   - A handle is not thread-safe; use one host thread per handle.
 *   - Every entry point caches, per process, the kernel attributes,
 *     occupancy figures and tensor maps of the launches it has made.  This
 *     includes the functions without a handle (dory_gemm_bf16,
 *     dory_gemm_bf16_noalloc, dory_pack_weight_bf16, dory_quantize_mxfp8,
 *     dory_gemv_mxfp8, dory_sample).  Call the library from one host thread
 *     at a time.
 */
#ifndef DORY_H
#define DORY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dory_handle dory_handle;
typedef void* dory_stream; /* cudaStream_t */

typedef enum {
  DORY_OK = 0,
  DORY_ERR_INVALID_ARG = 1, /* bad pointer, size, k, gamma, seq id, ... */
  DORY_ERR_CAPACITY = 2,    /* request exceeds max_seq / max_chunk / max_batch */
  DORY_ERR_STATE = 3,       /* call not allowed in the sequence's current state */
  DORY_ERR_WORKSPACE = 4,   /* workspace too small or misaligned */
  DORY_ERR_CUDA = 5,        /* a CUDA runtime call failed */
  DORY_ERR_TIMEOUT = 6,     /* a device-side bounded wait gave up */
  DORY_ERR_UNSUPPORTED = 7  /* valid but not supported by this build */
} dory_status;

/* Recurrent-block KV cache mode ([digest] "Premises & limits"; [news] "How to run").
 * LAST_LOOP: one slot per attention layer; every loop overwrites it, so a
 *            token's cached K/V are those of its final loop and the cache size
 *            does not depend on k.  Queries in loop t < k of a later token see
 *            the final-loop K/V of earlier tokens.
 * PER_LOOP:  each recurrent attention layer keeps one slot per loop; loop t
 *            reads and writes slot t.  Cache size grows with k. */
typedef enum { DORY_LAST_LOOP = 0, DORY_PER_LOOP = 1 } dory_cache_mode;

typedef enum { DORY_F32 = 0, DORY_BF16 = 1 } dory_dtype;

/* Model shape and capacity.  Layer counts are physical layers: physical layers
 * alternate attention and MLP, attention first; attention layer j (counted
 * over the whole stack) is full causal when j % full_every == full_phase and
 * sliding-window (keys p-W < j <= p) otherwise ([digest] "How it works":
 * attention interleaved 3:1).  Weights and the KV cache are stored in dtype;
 * hidden states are fp32; GEMMs accumulate in fp32. */
typedef struct {
  int32_t d_model, vocab, n_heads, head_dim, n_kv_heads, d_ff;
  int32_t n_in, n_rec, n_out;     /* physical layers of the input, recurrent, output blocks */
  int32_t swa_window;             /* W */
  int32_t full_every, full_phase; /* 4, 3 for the 3:1 interleave */
  int32_t dtype;                  /* dory_dtype */
  int32_t max_batch;              /* number of sequence slots (seq ids 0..max_batch-1) */
  int32_t max_seq;                /* positions per sequence */
  int32_t k_max;                  /* largest loop count a call may use (1..4) */
  int32_t gamma_max;              /* largest speculative draft length (0 disables) */
  int32_t max_chunk;              /* most new tokens in one forward, summed over the batch */
  /* Paged cache of the full-attention layers (the sliding-window layers keep
   * a ring of swa_window + slack positions per sequence).  kv_page = 0: each
   * sequence slot reserves max_seq positions in every full-attention layer.
   * kv_page > 0 (a power of two in 16..4096): positions come in pages of
   * kv_page, drawn on demand from a pool of kv_pages pages per layer and
   * cache slot (0: enough for every slot to reach max_seq) and returned by
   * dory_reset, so a few long sequences and many short ones share one pool
   * (256K-token contexts without max_batch x 256K reservations).  A call
   * that needs more pages than are free fails with DORY_ERR_CAPACITY before
   * any work is queued. */
  int32_t kv_page;
  int32_t kv_pages;
} dory_config;

/* Device weight pointers, BORROWED (must outlive the handle).  All matrices
 * are row-major [out, in] in dtype.  The per-layer arrays are HOST arrays of
 * n_in+n_rec+n_out device pointers (copied at dory_create); entries for the
 * other layer kind are ignored.
 *   embed   [vocab, d]         token embedding (rows are used as given)
 *   lm_head [vocab, d]         untied LM head: logits = s . lm_head^T
 *   w_qkv   [q + 2 kv, d]      rows 0..q-1 = W_q, then W_k, then W_v
 *                              (q = n_heads*head_dim, kv = n_kv_heads*head_dim)
 *   w_o     [d, q]
 *   w_gu    [2 d_ff, d]        rows 0..d_ff-1 = W_gate, then W_up
 *   w_down  [d, d_ff]
 * The MLP is W_down (silu(W_gate h) * (W_up h)); attention head h reads KV
 * head h / (n_heads / n_kv_heads); the softmax scale is 1/sqrt(head_dim). */
typedef struct {
  const void* embed;
  const void* lm_head;
  const void* const* w_qkv;
  const void* const* w_o;
  const void* const* w_gu;
  const void* const* w_down;
} dory_weights;

typedef struct {
  int64_t steps;    /* verify passes */
  int64_t drafted;  /* draft tokens proposed */
  int64_t accepted; /* draft tokens accepted */
} dory_spec_stats;

/* Bytes of device workspace dory_create needs for this configuration.
 * alloc_mode PER_LOOP reserves k_max slots for every recurrent attention
 * layer (and still serves LAST_LOOP calls); LAST_LOOP reserves one. */
dory_status dory_workspace_size(const dory_config* cfg, dory_cache_mode alloc_mode, size_t* bytes);

/* Create a handle over caller-owned device memory.  workspace: device
 * pointer, 256-byte aligned, ws_bytes >= dory_workspace_size().  The
 * workspace is not cleared here; call dory_reset(h, -1, stream) before the
 * first prefill.  Host-only: queues no device work. */
dory_status dory_create(const dory_config* cfg, const dory_weights* w, dory_cache_mode alloc_mode,
                        void* workspace, size_t ws_bytes, dory_handle** out);

dory_status dory_destroy(dory_handle* h);

/* Empty sequence `seq` (or all sequences when seq == -1): its length becomes 0
 * and its cache mode and loop count are forgotten. */
dory_status dory_reset(dory_handle* h, int32_t seq, dory_stream stream);

/* Prefill: append lens[i] tokens to sequence seq_ids[i] for i < batch, as one
 * forward chunk per sequence at loop count k (the input block once, the
 * recurrent block k times on u_t = N(s_{t-1} + x), the output block and the
 * LM head: [digest] "How it works"), and choose the next token of each
 * sequence (greedy, lowest id on ties).
 *   seq_ids      host int32[batch], distinct, in [0, max_batch)
 *   tokens       device int32[sum(lens)], the sequences' tokens concatenated
 *   lens         host int32[batch], each >= 1; sum(lens) <= max_chunk
 *   k            1..k_max
 *   mode         fixed per sequence from its first prefill; per_loop
 *                sequences must keep the same k in every later call
 *   last_logits  device float[batch, vocab] or NULL: logits of each
 *                sequence's last new position
 *   next_tokens  device int32[batch]
 * Within a chunk, loop t of every position writes its loop-t K/V and attends
 * to the chunk's loop-t K/V plus the cached K/V of earlier calls. */
dory_status dory_prefill(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* tokens,
                         const int32_t* lens, int32_t k, dory_cache_mode mode, float* last_logits,
                         int32_t* next_tokens, dory_stream stream);

/* One decode step: append tokens_in[i] to sequence seq_ids[i] and choose its
 * next token (the same forward as dory_prefill on a one-token chunk; under
 * LAST_LOOP the recurrent layers overwrite their one cache slot in every
 * loop, [digest] "Premises & limits").  seq_ids host int32[batch]; tokens_in device int32[batch];
 * logits device float[batch, vocab] or NULL; next_tokens device int32[batch]. */
dory_status dory_decode_step(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* tokens_in,
                             int32_t k, dory_cache_mode mode, float* logits, int32_t* next_tokens,
                             dory_stream stream);

/* One decode step with a loop count per sequence: sequence seq_ids[i] runs
 * ks[i] loops of the recurrent block.  ks host int32[batch], each in
 * 1..k_max, non-increasing along the batch (sequences grouped by k): loop t
 * runs on the sequences with ks[i] >= t only, so the ones that finish early
 * skip the later loops.  Other arguments and errors as dory_decode_step; a
 * per_loop sequence must keep the k of its first call.  The loop count is
 * chosen per request at inference ([news] "How to run"); this call batches
 * requests with different k.  Each sequence's result equals a decode step of
 * that sequence at its own k, up to rounding. */
dory_status dory_decode_step_mixed(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* tokens_in,
                                   const int32_t* ks, dory_cache_mode mode, float* logits, int32_t* next_tokens,
                                   dory_stream stream);

/* Self-speculative greedy decoding ([digest] "Premises & limits"): each step
 * drafts gamma tokens one at a time at k_draft, verifies the chunk
 * [pending, d_1..d_gamma] at k_verify reusing the drafts' input-block output,
 * loop-1 state and K/V, accepts the longest prefix the verifier agrees with
 * plus the verifier's own next token, and rolls the cache back to the
 * accepted length.  Steps repeat until every sequence has max_new tokens.
 *   last_tokens  device int32[batch]: each sequence's pending token (the
 *                token chosen by its prefill or last decode, not yet in the cache)
 *   out_tokens   device int32[batch, max_new]; out_len device int32[batch]
 *   stats        host, may be NULL
 * k_draft must be 1 (loop-1 reuse); gamma in 1..gamma_max; k_verify in 1..k_max.
 * Needs len + max_new + 2*gamma + 1 <= max_seq for every sequence (a sequence
 * that finishes first keeps drafting from its frozen length while the others
 * continue).  Synchronises the stream after every verify step to test for
 * completion.
 * In PER_LOOP mode the output equals plain k_verify greedy decoding. */
dory_status dory_spec_decode(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* last_tokens,
                             int32_t k_draft, int32_t k_verify, int32_t gamma, dory_cache_mode mode,
                             int32_t max_new, int32_t* out_tokens, int32_t* out_len, dory_spec_stats* stats,
                             dory_stream stream);

/* KV bytes one sequence of ctx tokens holds at loop count k in `mode` (the
 * positions a future query can still read: the last W for a sliding-window
 * layer, all for a full layer).  Host only. */
dory_status dory_kv_bytes(const dory_handle* h, int32_t k, dory_cache_mode mode, int64_t ctx, int64_t* bytes);

/* Committed length of a sequence as known to the host (exact after every
 * call returns; dory_spec_decode synchronises before returning). */
dory_status dory_seq_len(const dory_handle* h, int32_t seq, int32_t* len);

/* Copy fp32 rows of the last forward pass's states into device dst[rows, d]:
 * which = 0: x (input-block output), 1: s_k (final loop state),
 * 2: output-block result.  rows = the last call's chunk rows. */
dory_status dory_read_state(dory_handle* h, int32_t which, float* dst, int32_t rows, dory_stream stream);

/* Copy a sequence's cached K and V of physical attention layer `layer`, slot
 * `slot` (0 unless PER_LOOP recurrent: loop t -> slot t-1), positions
 * [pos0, pos0+n) into device k_dst/v_dst [n, n_kv_heads, head_dim] (dtype).
 * Positions must still be retained (ring slots of sliding-window layers). */
dory_status dory_read_kv(dory_handle* h, int32_t layer, int32_t slot, int32_t seq, int32_t pos0, int32_t n,
                         void* k_dst, void* v_dst, dory_stream stream);

/* Projection GEMM on its own (the kernel every projection of the forward
 * uses): Y_s = X . W^T partial products for X [M, K], W [N, K] bf16 (device,
 * row-major, 16-byte aligned) with fp32 accumulation.  Y (device) must hold
 * 8 * M * N floats: the result is *splits slices Y[s][M][N] whose in-order
 * sum s = 0..*splits-1 is the product.  batch_hint selects the split the
 * decode path uses for that many sequences; invariant != 0 makes each row's
 * arithmetic independent of M.  impl: 0 auto, 1 SIMT kernel, 2 tcgen05 only
 * (DORY_ERR_CUDA if the shape is unsupported), 3 tcgen05 with one 64-column
 * sub-tile per pipeline stage (comparison variant), 4 tcgen05 with W in the
 * packed tile layout of dory_pack_weight_bf16.  err_word (device int, may be
 * NULL) receives DORY_ERR_TIMEOUT-class codes from bounded waits.  Queues work
 * on `stream`; no handle needed. */
dory_status dory_gemm_bf16(int32_t M, int32_t N, int32_t K, const void* X, const void* W, float* Y,
                           int32_t batch_hint, int32_t invariant, int32_t impl, int32_t* splits, int32_t* err_word,
                           dory_stream stream);

/* Projection GEMM for callers that cannot allocate device memory (no
 * counterpart on the pages: this is a library convenience).  Some callers
 * cannot hand dory_gemm_bf16 its 8 * M * N-float partial buffer: code running
 * while a CUDA graph is recorded (cudaMalloc is not allowed there), servers
 * whose device memory is one arena owned by someone else, real-time paths
 * that forbid allocation.  This variant keeps the split-K partial sums in an
 * 8 MiB array built into the library (held on every GPU that loads it, until
 * exit) and writes the finished product Y = X . W^T [M, N] fp32 (device).
 * X [M, K], W [N, K] bf16 device pointers, 16-byte aligned, N % 128 == 0,
 * K % 64 == 0; 8 * M * N <= 2097152 or DORY_ERR_CAPACITY (checked before any
 * work).  It calls no allocator.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  All calls share the array:
 * calls whose kernels overlap on the GPU (other streams or threads) corrupt
 * each other's results, so serialise them.  Queues work on `stream`. */
dory_status dory_gemm_bf16_noalloc(int32_t M, int32_t N, int32_t K, const void* X, const void* W, float* Y,
                                   int32_t batch_hint, dory_stream stream);

/* Timeout report of dory_gemm_bf16_noalloc (no counterpart on the pages).
 * Its GEMM's bounded waits give up after about a second; they then record
 * the fact in a second word built into the library next to the scratch
 * array, and every later call writes NaN into its Y until this function
 * clears the word.  Synchronises `stream`, reads and clears the word, and
 * returns DORY_ERR_TIMEOUT if a wait gave up since the last check
 * (DORY_OK otherwise).  Allocates nothing. */
dory_status dory_gemm_bf16_noalloc_status(dory_stream stream);

/* Repack a row-major [N, K] bf16 weight (device src, 16-byte aligned,
 * N % 128 == 0, K % 64 == 0) into device dst (N*K*2 bytes, distinct from src)
 * in the packed tile layout: 128-row x 64-column tiles, each stored as its
 * 16 KB shared-memory image with 128-byte swizzle (row r's 16-byte chunk c at
 * byte r*128 + (c XOR (r mod 8))*16), tile (n, k) at ((n*K/64) + k) * 16 KB.
 * The tensor-core GEMM streams packed weights with one bulk copy per pipeline
 * stage.  Queues work on `stream`. */
dory_status dory_pack_weight_bf16(const void* src, void* dst, int32_t N, int32_t K, dory_stream stream);

/* ---------------------------------------------------------------- MXFP8
 * 8-bit weights for decoding.  The pages list MXFP8 among the released weight
 * formats and measure it against BF16 at batch 1 ([trawling] "KV cache and
 * runtime"; [news] "Training and variants": 1.69x to 1.84x on a DGX Spark).  The format is the OCP
 * Microscaling Formats (MX) v1.0 MXFP8: FP8 E4M3 codes (bias 7, largest
 * finite 448, subnormals m/8 * 2^-6) and one E8M0 scale byte
 * (2^(byte - 127)) per 32 consecutive weights of a row.  Codes are
 * row-major [N, K] bytes; scales are row-major [N, K/32] bytes.  The scale of
 * weight (n, k) is scales[n*K/32 + k/32].
 *
 * Quantise a row-major bf16 weight w [N, K] (device, 16-byte aligned,
 * K % 32 == 0).  For each block, shared = floor(log2(max |w|)) - 8, clamped
 * to [-127, 127] (-127 for a block of zeros), and scale byte = shared + 127.
 * Each code is E4M3(w * 2^-shared), rounded to nearest-even, with
 * magnitudes above 448 clamped to 448; a value that rounds to zero keeps its
 * sign.  q: device [N, K] bytes (16-byte aligned); scales: device [N, K/32]
 * bytes.  w_deq (device, nullable, 16-byte aligned) receives the
 * dequantised weights 2^shared * E4M3(code) rounded to bf16 [N, K], which
 * is exact unless a block's scale is below 2^-120.  A non-finite weight sets
 * *err_word (device int32, nullable); dory_synchronize then reports
 * DORY_ERR_INVALID_ARG.  Queues work on `stream`. */
dory_status dory_quantize_mxfp8(const void* w, int32_t N, int32_t K, void* q, void* scales, void* w_deq,
                                int32_t* err_word, dory_stream stream);

/* y[i, n] = sum_k x[i, k] * 2^(scales[n, k/32] - 127) * E4M3(q[n, k]) for
 * i < M, n < N, with fp32 sums.  x is bf16 [M, ldx] (device) and y is fp32
 * [M, ldy] (device).  Each y[i, n] is summed in an order fixed by K alone,
 * so its bits do not depend on M.  Requires K % 32 == 0, ldx >= K,
 * ldy >= N and q 16-byte aligned.
 *   impl 2: tensor cores.  mma.sync with f16 operands and fp32 accumulators;
 *     one block's 32 products per accumulation, then the block scale.
 *     K <= 10240.  Any finite x; |x| below 2^-124 adds nothing.
 *   impl 1: CUDA cores.  K <= 40960; supported range |x| < 2^64 and scale
 *     bytes <= 198 (what the quantiser writes for |w| < 2^80).
 *   impl 3: tcgen05 GEMM fed by TMA.  Converter warps expand the codes to
 *     f16 in shared memory; each 32-weight block accumulates in its own TMEM
 *     columns and takes its scale in the epilogue.  Requires N % 128 == 0,
 *     K % 128 == 0, x 16-byte aligned, ldx % 8 == 0 (else
 *     DORY_ERR_UNSUPPORTED); |x| < 4.
 *   impl 4: impl 1's arithmetic (the same bits) with the weight rows
 *     streamed into shared memory by bulk copies; shapes it does not take
 *     (N % 8, more than 24 KB of weights per 8 rows, too many rows M for
 *     the staged activations) run as 1.
 *   impl 0: 4 where it takes the shape, else 1 (the same bits; measured
 *     faster than 1 and 2 in a 4B decode step).
 * An activation outside the range (non-finite for 2) sets *err_word (device,
 * nullable).  Queues work on `stream`. */
dory_status dory_gemv_mxfp8(int32_t M, int32_t N, int32_t K, const void* x, int32_t ldx, const void* q,
                            const void* scales, float* y, int32_t ldy, int32_t impl, int32_t* err_word,
                            dory_stream stream);

/* MXFP8 copies of a handle's projection weights and LM head (device
 * pointers, BORROWED: they must outlive the attachment).  The per-layer
 * arrays are indexed by physical layer.  qkv_* and o_* entries are read for
 * attention layers, gu_* and down_* entries for MLP layers.  An entry whose
 * code and scale pointers are both NULL (or a NULL array) leaves that matrix
 * in bf16. */
typedef struct {
  const void* lm_head_q;
  const void* lm_head_s;
  const void* const* qkv_q;
  const void* const* qkv_s;
  const void* const* o_q;
  const void* const* o_s;
  const void* const* gu_q;
  const void* const* gu_s;
  const void* const* down_q;
  const void* const* down_s;
} dory_mx_weights;

/* Attach MXFP8 copies (mx != NULL) or detach them (mx == NULL).  While they
 * are attached, the GEMMs of decode steps (plain, mixed-k and speculative)
 * run dory_gemv_mxfp8 on the copies.  Prefill keeps the bf16 weights given
 * to dory_create.  For a forward that is the dequantised model throughout,
 * create the handle with the w_deq output of dory_quantize_mxfp8.  Attaching
 * drops captured decode graphs and turns the L2 look-ahead off.  The handle
 * must hold bf16 weights, and d_model, n_heads * head_dim and d_ff must be
 * multiples of 32 (else DORY_ERR_UNSUPPORTED).  A copy with codes but no
 * scales, or codes that are not 16-byte aligned, gives DORY_ERR_INVALID_ARG
 * and leaves the previous attachment in place. */
dory_status dory_attach_mxfp8(dory_handle* h, const dory_mx_weights* mx);

/* ---------------------------------------------------------------- NVFP4
 * 4-bit weights for decoding ([trawling] "KV cache and runtime"; [news]
 * "Training and variants": 2.17x to 2.44x over BF16 at batch 1 on a DGX
 * Spark).  The format is NVIDIA's NVFP4:
 *   - FP4 E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte,
 *     the even k in the low nibble: q is [N, K/2] bytes;
 *   - one FP8 E4M3 scale per 16 consecutive weights of a row: scales is
 *     [N, K/16] bytes;
 *   - one per-tensor float scale g.
 *   w = E2M1(code) * E4M3(scale) * g.
 *
 * Quantise a row-major bf16 weight w [N, K] (device, 16-byte aligned,
 * K % 16 == 0):
 *   - g = the smallest power of two with 6 * 448 * g >= max |w|, written to
 *     the device float *g;
 *   - block scale = E4M3(amax_b / (6 g));
 *   - code = E2M1(w / (scale * g)), both rounded to nearest-even and
 *     saturating; codes are 0 for a block whose scale is 0, and a value that
 *     rounds to zero keeps its sign.
 * q is 8-byte aligned.  w_deq (nullable, 16-byte aligned) receives the exact
 * bf16 dequantisation.  A non-finite weight sets *err_word.  Queues three
 * launches on `stream`. */
dory_status dory_quantize_nvfp4(const void* w, int32_t N, int32_t K, void* q, void* scales, float* g, void* w_deq,
                                int32_t* err_word, dory_stream stream);

/* y[i, n] = sum_k x[i, k] * E2M1(q[n, k]) * E4M3(scales[n, k/16]) * g, with
 * fp32 sums, for x bf16 [M, ldx] (device) and y fp32 [M, ldy] (device).
 * tcgen05 GEMM fed by TMA: converter warps expand the codes to f16; each
 * 16-weight block accumulates in its own TMEM columns and takes its scale
 * in the epilogue.  Each y[i, n] is summed in an order fixed by K alone.
 * Requires N % 128 == 0, K % 256 == 0, x, q and scales 16-byte aligned,
 * ldx % 8 == 0 (else DORY_ERR_UNSUPPORTED); |x| < 4 (else *err_word).
 * Queues work on `stream`. */
dory_status dory_gemm_nvfp4(int32_t M, int32_t N, int32_t K, const void* x, int32_t ldx, const void* q,
                            const void* scales, const float* g, float* y, int32_t ldy, int32_t* err_word,
                            dory_stream stream);

/* NVFP4 copies of a handle's projection weights and LM head (device
 * pointers, BORROWED), indexed like dory_mx_weights, with each matrix's
 * tensor scale as a device float. */
typedef struct {
  const void* lm_head_q;
  const void* lm_head_s;
  const float* lm_head_g;
  const void* const* qkv_q;
  const void* const* qkv_s;
  const float* const* qkv_g;
  const void* const* o_q;
  const void* const* o_s;
  const float* const* o_g;
  const void* const* gu_q;
  const void* const* gu_s;
  const float* const* gu_g;
  const void* const* down_q;
  const void* const* down_s;
  const float* const* down_g;
} dory_nvfp4_weights;

/* Attach NVFP4 copies (nv != NULL) or detach them (nv == NULL).  While
 * attached, decode GEMMs (plain, mixed-k, speculative) run dory_gemm_nvfp4's
 * kernel with split-K slices.  A handle holds one low-bit format at a time:
 * attaching NVFP4 replaces attached MXFP8 copies and vice versa.  Needs bf16
 * weights, and d_model, n_heads * head_dim and d_ff multiples of 256 (else
 * DORY_ERR_UNSUPPORTED).  For a forward that is the dequantised model
 * throughout, create the handle with the w_deq output of
 * dory_quantize_nvfp4.  Drops captured decode graphs and turns the L2
 * look-ahead off. */
dory_status dory_attach_nvfp4(dory_handle* h, const dory_nvfp4_weights* nv);

/* Synchronise `stream` and report device-side errors (DORY_ERR_TIMEOUT when
 * a bounded wait in a kernel gave up; the handle stays usable). */
dory_status dory_synchronize(dory_handle* h, dory_stream stream);

/* Options. */
enum {
  DORY_OPT_CUDA_GRAPHS = 1, /* 1 (default): replay captured decode steps */
  DORY_OPT_PROFILE = 2,     /* 1: time every launch with CUDA events (slow) */
  DORY_OPT_GEMM_IMPL = 3,   /* bf16 GEMM: 0 auto, 1 SIMT reference kernel, 2 tcgen05 */
  DORY_OPT_PDL = 4,         /* 1 (default): programmatic dependent launches (process-wide) */
  DORY_OPT_PREFILL_TC = 5,  /* bf16 long-chunk attention, head_dim 128 (other widths as 1): 3 (default)
                               warp-specialised tcgen05, two 128-row query slots per CTA sharing a
                               TMA-fed key/value stream, P kept in TMEM; 2 tcgen05, one slot per CTA;
                               1 warp-level mma.sync; 0 CUDA cores */
  DORY_OPT_ATTN_CLUSTER = 6, /* 1 (default): decode attention as clusters of 16, 8 or 4 blocks per row and
                                KV head, chosen from the number of sequences; 4, 8, 16: that cluster size;
                                0: no clusters (process-wide) */
  /* bf16 decode steps: bytes of upcoming weights each GEMM prefetches into L2
   * past its own once its loads have landed (default 8 MiB; 0 turns the
   * look-ahead off).  Changes only when HBM reads happen, never what is
   * computed. */
  DORY_OPT_L2_LOOKAHEAD = 7,
  /* GEMM on attached MXFP8 copies (see dory_gemv_mxfp8's impl): 0 (default: 4 where it fits, else 1), 1 CUDA cores,
     2 mma.sync, 3 TMA-fed tcgen05 with split-K slices (matrices whose N or K it does not take use 1),
     4 CUDA cores fed by bulk copies (the same bits as 1; shapes it does not take use 1) */
  DORY_OPT_MX_GEMV = 8,
  /* bf16 decode and speculative steps of at most this many rows (default 0:
   * off; at most 16): the add + L2 norm after a layer and the SwiGLU of a
   * split gate-up product run inside the next projection GEMM, whose
   * epilogue warps build its operand in shared memory, instead of as kernels
   * of their own.  Same arithmetic, so the same bits, either way.  Measured
   * slower than the separate kernels at batch 1 on the 4B shape, hence off. */
  DORY_OPT_FUSED_OPERANDS = 9,
  /* bf16 decode steps: bytes of upcoming weights (past its own) that the O
   * projection after each decode attention prefetches into L2 as soon as it
   * is launched, before it waits for the attention, instead of the
   * DORY_OPT_L2_LOOKAHEAD range after its loads (default 0: that range).
   * Changes only when HBM reads happen, never what is computed. */
  DORY_OPT_ATTN_LOOKAHEAD = 10,
  /* bf16 decode GEMMs: before waiting for the previous kernel, each CTA asks
   * L2 for up to this many of its own weight tiles past those its
   * shared-memory ring takes (TMA prefetch; 0 turns it off).  Changes only
   * when HBM reads happen, never what is computed. */
  DORY_OPT_L2_OWN = 11
};
dory_status dory_set_option(dory_handle* h, int32_t opt, int64_t value);

/* Token choice of prefill and decode steps.  temperature 0 (default):
 * greedy, lowest id on ties.  temperature > 0: top-p sampling ([news] "How
 * to run" names temperature 1.0, top-p 0.95 for the released model): one
 * Philox4x32-10 draw per new token (key = seed, counter = (sequence id,
 * position of the new token, 0, 0)), integer nucleus masses
 * q_i = floor(exp2((l_i - max) log2(e) / T) * 2^31), nucleus = tokens with
 * q_i >= tau for the largest tau whose tail mass reaches ceil(top_p * sum q),
 * token = first id at which the running nucleus mass exceeds
 * floor(u * nucleus mass).  top_p in (0, 1].  Speculative decoding stays
 * greedy (DORY_ERR_UNSUPPORTED while temperature > 0). */
dory_status dory_set_sampling(dory_handle* h, float temperature, float top_p, uint64_t seed);

/* The sampler alone: rows of device logits [rows, vocab] (fp32), draw of row
 * i keyed by device seq[i], pos[i]; scratch device uint32[rows * vocab] (may
 * alias logits, which are then overwritten); out device int32[rows].
 * temperature > 0.  Queues work on `stream`. */
dory_status dory_sample(const float* logits, int32_t rows, int32_t vocab, const int32_t* seq, const int32_t* pos,
                        float temperature, float top_p, uint64_t seed, uint32_t* scratch, int32_t* out,
                        dory_stream stream);

/* Per-kernel launch statistics gathered while DORY_OPT_PROFILE is on:
 * fills up to n entries of names (host char[n][48]), launches, total_ms and
 * algorithmic bytes; returns the number of kernels in *count. */
dory_status dory_profile_read(dory_handle* h, int32_t n, char (*names)[48], int64_t* launches,
                              double* total_ms, double* bytes, int32_t* count);
dory_status dory_profile_reset(dory_handle* h);

/* Message of the last failed call on this host thread ("" if none), valid
 * until the next call on the thread.  h (nullable) is not read: the message
 * is kept per thread, whichever handle the failing call used. */
const char* dory_last_error(const dory_handle* h);

#ifdef __cplusplus
}
#endif
#endif /* DORY_H */

// Host runner and C ABI of the looped nGPT library.
//
// The forward of one chunk of new tokens follows the recurrence of the
// Dory1.0-4B digest (onedev.kr/papers/1692, "How it works"): the input block
// runs once, the shared recurrent block runs k times on u_t = N(s_{t-1} + x)
// with s_0 = x and s_t = N(F(u_t)), then the output block and the LM head
// run on s_k.  Every physical layer updates h <- N(h + sublayer(h)).  The KV
// cache follows the same digest's "Premises & limits": in last-loop mode a
// recurrent attention layer has one slot that every loop overwrites; in
// per-loop mode loop t has its own slot.
//
// All device state lives in the caller's workspace; nothing here allocates
// device memory.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <unordered_map>
#include <vector>

#include "dory.h"
#include "attn_decode.cuh"
#include "attn_prefill.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "mxfp8.cuh"

namespace dory {
bool g_pdl = true;
}

using namespace dory;

namespace {

thread_local std::string g_last_error;

dory_status fail(dory_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
dory_status fail(dory_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

}  // namespace

namespace dory {
// Lets other translation units of the library report through dory_last_error().
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace dory

namespace {

#define CK(expr)                                                                                  \
  do {                                                                                            \
    cudaError_t e_ = (expr);                                                                      \
    if (e_ != cudaSuccess) return fail(DORY_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

// Bump allocator over the workspace (or a size counter when base == nullptr).
struct Carve {
  char* base;
  size_t off = 0;
  template <typename P>
  P* take(size_t bytes) {
    off = (off + 255) & ~(size_t)255;
    P* p = base ? (P*)(base + off) : nullptr;
    off += bytes;
    return p;
  }
};

struct AttnLayer {
  int layer;      // physical layer index
  bool full;      // full causal (else sliding window)
  bool rec;       // in the recurrent block
  int cap;        // positions held: ring size (window) or max_seq (full)
  int nslots;     // 1, or k_max for per-loop recurrent layers
  char* K[8];
  char* V[8];
};

struct ProfRec {
  int name;
  double bytes;
  cudaEvent_t a, b;
};

}  // namespace

struct dory_handle {
  dory_config c{};
  int alloc_mode = 0;
  bool bf16 = false;
  int esz = 4;
  int L = 0, q_dim = 0, kv_dim = 0, qkv_dim = 0, slack = 0, M_max = 0, head_max = 0, nb_max = 0;
  const void* embed = nullptr;
  const void* head = nullptr;
  std::vector<const void*> w_qkv, w_o, w_gu, w_down;
  // MXFP8 copies read by the decode / speculative GEMMs, keyed by the bf16
  // weight they stand for (empty: none attached)
  struct MxMat {
    const uint8_t* q;
    const uint8_t* s;
    const float* g = nullptr;  // NVFP4 tensor scale (device)
    int fmt = 0;               // 0 MXFP8, 1 NVFP4
  };
  std::unordered_map<const void*, MxMat> mx;
  int mx_impl = 0;  // GEMV on the copies: 0 default (4 where it fits, else 1), 1 CUDA cores, 2 tensor cores,
                    // 3 tcgen05 GEMM, 4 CUDA cores fed by bulk copies
  std::vector<int> attn_of;
  std::vector<AttnLayer> attn;

  // device buffers (inside the workspace)
  char* ws = nullptr;
  size_t ws_bytes = 0;
  int *seq_len = nullptr, *err = nullptr, *seq_ids = nullptr, *tokens = nullptr, *next = nullptr;
  int *cu = nullptr, *head_rows = nullptr;
  int2* tiles = nullptr;  // prefill attention tiles (64 or 128 rows of one sequence)
  int tiles_cap = 0;
  int4* pf_items = nullptr;  // warp-specialised prefill attention: CTA work items
  int items_cap = 0;
  void* qh = nullptr;     // bf16 pre-scaled queries of long chunks
  RowMeta meta{};
  // the state h lives in one of two buffers: a GEMM that applies the
  // previous layer's update in its operand stage reads one and writes the other
  float* hb[2] = {nullptr, nullptr};
  int hc = 0;
  float *x = nullptr, *s = nullptr, *q = nullptr, *part_qkv = nullptr, *part_y = nullptr, *part_gu = nullptr,
        *attn_part = nullptr, *logits = nullptr;
  void *hop = nullptr, *ao = nullptr, *act = nullptr, *kscr = nullptr, *vscr = nullptr, *hop_head = nullptr;
  size_t part_rows = 0;      // rows of an unsplit GEMM output (prefill)
  size_t part_rows_dec = 0;  // rows per split slice on the decode / speculative path
  float *stash_x = nullptr, *stash_s = nullptr;
  int *drafts = nullptr, *pending = nullptr, *vtok = nullptr;
  unsigned long long* accepted = nullptr;
  SpecIo* spec_io = nullptr;
  int* spec_flags = nullptr;  // [0] all finished, [1] steps, [2] step bound hit
  unsigned* attn_counters = nullptr;  // [M_max * n_kv], zero between launches
  int nb_cap = 0;                     // key blocks per row the partial buffer holds
  int attn_rows = 0;                  // rows the partial buffer holds
  // weight stream of a decode step at each loop count k (L2 look-ahead)
  PfSeg* pf_segs = nullptr;           // [k_max][pf_nseg_max]
  int pf_nseg_max = 0;

  // host state
  std::vector<int> len, mode, kfix;  // per sequence; mode -1 = empty
  // paged full-attention cache: device page table [max_batch][pt_stride],
  // its host copy, the pages each sequence holds and the free pool
  int* page_table = nullptr;
  int pt_stride = 0, page_shift = 0, pool_pages = 0;
  std::vector<int> pt_host, free_pages;
  std::vector<int4> items_host;
  std::vector<std::vector<int>> seq_pages;
  std::vector<int> ids_on_device;     // seq ids last uploaded to seq_ids
  int last_rows = 0;
  bool graphs = true, profile = false;
  int prefill_tc = 3;  // long-chunk attention: 3 warp-specialised tcgen05, 2 one-slot tcgen05 (head_dim 128),
                       // 1 mma.sync, 0 CUDA cores
  int gemm_impl = 0;
  unsigned long long pf_lead = 8ull << 20;   // 0: no L2 look-ahead
  unsigned long long pf_attn = 0;            // early look-ahead of the GEMM after a decode attention (0: none)
  int pf_own = 0;                            // own weight tiles a decode GEMM CTA prefetches before its wait
  float temperature = 0.f, top_p = 1.f;      // temperature 0: greedy
  unsigned long long seed = 0;
  std::vector<std::vector<PfSeg>> pf_host;   // [k] -> stream of a k-loop decode step
  std::vector<char> pf_uploaded;             // [k]
  int pf_pos = -1;                           // next segment of the pass being issued; -1 off
  unsigned long long pf_done = 0;            // stream bytes already handed out for prefetch
  std::vector<std::string> prof_names;
  std::vector<ProfRec> prof_recs;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  struct Graph {
    long long key;
    int seen;
    cudaGraphExec_t exec;
    int hc_end;  // state buffer holding h when the recorded step ends
  };
  std::vector<Graph> graphs_cache;
  cudaStream_t cap_stream = nullptr;  // private stream used only to record graphs

  int fuse_rows = 0;  // operand stages for decode / speculative passes of at most this many rows (0 off)

  template <typename T>
  T* hop_t() const { return (T*)hop; }
  float* hcur() const { return hb[hc]; }
};

namespace {

// ------------------------------------------------------------------ layout
bool layer_is_attn(int l) { return l % 2 == 0; }

dory_status check_config(const dory_config* c) {
  if (!c) return fail(DORY_ERR_INVALID_ARG, "config is NULL");
  if (c->d_model <= 0 || c->vocab <= 0 || c->n_heads <= 0 || c->head_dim <= 0 || c->n_kv_heads <= 0 ||
      c->d_ff <= 0)
    return fail(DORY_ERR_INVALID_ARG, "non-positive model dimension");
  if (c->n_in < 0 || c->n_rec <= 0 || c->n_out < 0) return fail(DORY_ERR_INVALID_ARG, "bad block sizes");
  if (c->n_heads % c->n_kv_heads) return fail(DORY_ERR_INVALID_ARG, "n_heads %% n_kv_heads != 0");
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128)
    return fail(DORY_ERR_UNSUPPORTED, "head_dim must be 32, 64 or 128");
  int G = c->n_heads / c->n_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 5 || (G == 8 && c->head_dim <= 64)))
    return fail(DORY_ERR_UNSUPPORTED, "query heads per KV head must be 1, 2, 4, 5 or 8");
  if (c->d_model > 4096) return fail(DORY_ERR_UNSUPPORTED, "d_model > 4096");
  if (c->d_model % 8 || c->d_ff % 8) return fail(DORY_ERR_UNSUPPORTED, "d_model and d_ff must be multiples of 8");
  if (c->swa_window <= 0) return fail(DORY_ERR_INVALID_ARG, "swa_window must be >= 1");
  if (c->full_every <= 0 || c->full_phase < 0) return fail(DORY_ERR_INVALID_ARG, "bad full-attention pattern");
  if (c->dtype != DORY_F32 && c->dtype != DORY_BF16) return fail(DORY_ERR_INVALID_ARG, "bad dtype");
  if (c->max_batch <= 0 || c->max_seq <= 0 || c->max_chunk <= 0) return fail(DORY_ERR_INVALID_ARG, "bad capacity");
  if (c->k_max < 1 || c->k_max > 8) return fail(DORY_ERR_INVALID_ARG, "k_max must be in 1..8");
  if (c->gamma_max < 0 || c->gamma_max > 16) return fail(DORY_ERR_INVALID_ARG, "gamma_max must be in 0..16");
  if (c->kv_page != 0 && (c->kv_page < 16 || c->kv_page > 4096 || (c->kv_page & (c->kv_page - 1))))
    return fail(DORY_ERR_INVALID_ARG, "kv_page must be 0 or a power of two in 16..4096");
  if (c->kv_pages < 0) return fail(DORY_ERR_INVALID_ARG, "kv_pages must be >= 0");
  return DORY_OK;
}

// Fill the handle's layout; with h->ws == nullptr only sizes are computed.
size_t layout(dory_handle* h) {
  const dory_config& c = h->c;
  Carve cv{h->ws};
  h->bf16 = c.dtype == DORY_BF16;
  h->esz = h->bf16 ? 2 : 4;
  h->L = c.n_in + c.n_rec + c.n_out;
  h->q_dim = c.n_heads * c.head_dim;
  h->kv_dim = c.n_kv_heads * c.head_dim;
  h->qkv_dim = h->q_dim + 2 * h->kv_dim;
  // sliding-window rings keep W + slack positions so that speculative writes
  // past the accepted length never evict a key a later query still needs
  h->slack = ((c.gamma_max + 1 + 15) / 16) * 16;
  h->M_max = std::max(c.max_chunk, c.max_batch * (c.gamma_max + 1));
  h->head_max = std::max(c.max_batch * (c.gamma_max + 1), c.max_batch);
  h->nb_max = (c.max_seq + ATTN_BK - 1) / ATTN_BK + 1;
  h->nb_cap = std::max(h->nb_max, (c.max_seq + DEC_BK - 1) / DEC_BK + 1);
  const int M = h->M_max;
  const size_t e = h->esz;

  h->attn.clear();
  h->attn_of.assign(h->L, -1);
  if (c.kv_page > 0) {
    h->pt_stride = (c.max_seq + c.kv_page - 1) / c.kv_page;
    h->page_shift = 0;
    while ((1 << h->page_shift) < c.kv_page) ++h->page_shift;
    h->pool_pages = c.kv_pages > 0 ? c.kv_pages : c.max_batch * h->pt_stride;
  }
  int j = 0;
  for (int l = 0; l < h->L; ++l) {
    if (!layer_is_attn(l)) continue;
    AttnLayer a{};
    a.layer = l;
    a.full = (j % c.full_every) == c.full_phase;
    a.rec = l >= c.n_in && l < c.n_in + c.n_rec;
    a.cap = a.full ? c.max_seq : std::min(c.max_seq, c.swa_window + h->slack);
    a.nslots = (h->alloc_mode == DORY_PER_LOOP && a.rec) ? c.k_max : 1;
    size_t bytes = (size_t)c.max_batch * c.n_kv_heads * a.cap * c.head_dim * e;
    if (a.full && c.kv_page > 0) bytes = (size_t)h->pool_pages * c.n_kv_heads * c.kv_page * c.head_dim * e;
    for (int s = 0; s < a.nslots; ++s) {
      a.K[s] = cv.take<char>(bytes);
      a.V[s] = cv.take<char>(bytes);
    }
    h->attn_of[l] = (int)h->attn.size();
    h->attn.push_back(a);
    ++j;
  }
  const int d = c.d_model;
  if (c.kv_page > 0) h->page_table = cv.take<int>(sizeof(int) * (size_t)c.max_batch * h->pt_stride);
  h->seq_len = cv.take<int>(sizeof(int) * c.max_batch);
  h->err = cv.take<int>(sizeof(int) * 4);
  h->seq_ids = cv.take<int>(sizeof(int) * M);
  h->tokens = cv.take<int>(sizeof(int) * M);
  h->next = cv.take<int>(sizeof(int) * M);
  h->cu = cv.take<int>(sizeof(int) * (c.max_batch + 1));
  h->head_rows = cv.take<int>(sizeof(int) * h->head_max);
  h->tiles_cap = M / 64 + c.max_batch + 1;
  h->tiles = cv.take<int2>(sizeof(int2) * h->tiles_cap);
  h->items_cap = h->tiles_cap * c.n_heads;
  h->pf_items = cv.take<int4>(sizeof(int4) * h->items_cap);
  h->qh = cv.take<char>(2 * (size_t)M * h->q_dim);
  h->meta.seq = cv.take<int>(sizeof(int) * M);
  h->meta.pos = cv.take<int>(sizeof(int) * M);
  h->meta.p0 = cv.take<int>(sizeof(int) * M);
  h->meta.base = cv.take<int>(sizeof(int) * M);
  h->meta.pend = cv.take<int>(sizeof(int) * M);
  h->hb[0] = cv.take<float>(sizeof(float) * M * d);
  h->hb[1] = cv.take<float>(sizeof(float) * M * d);
  h->x = cv.take<float>(sizeof(float) * M * d);
  h->s = cv.take<float>(sizeof(float) * M * d);
  h->q = cv.take<float>(sizeof(float) * M * h->q_dim);
  h->hop = cv.take<char>(e * M * std::max(d, 1));
  h->ao = cv.take<char>(e * M * h->q_dim);
  h->act = cv.take<char>(e * M * c.d_ff);
  h->kscr = cv.take<char>(e * M * h->kv_dim);
  h->vscr = cv.take<char>(e * M * h->kv_dim);
  h->hop_head = cv.take<char>(e * h->head_max * d);
  // Split-K slices are used only by decode / speculative rows (at most
  // max_batch * (gamma_max + 1)); long prefill chunks never split K.
  h->part_rows_dec = (size_t)std::max(c.max_batch, c.max_batch * (c.gamma_max + 1));
  h->part_rows = (size_t)M;
  const size_t prow = std::max((size_t)kMaxSplitK * h->part_rows_dec, (size_t)M);
  h->part_qkv = cv.take<float>(sizeof(float) * prow * h->qkv_dim);
  h->part_y = cv.take<float>(sizeof(float) * prow * d);
  h->part_gu = cv.take<float>(sizeof(float) * prow * 2 * c.d_ff);
  // split-KV partials: decode / verify rows at full context, or a slice of
  // up to 256 chunk rows (the CUDA-core chunk attention runs in row slices)
  h->attn_rows = std::min(M, std::max(c.max_batch * (c.gamma_max + 1), 256));
  h->attn_part =
      cv.take<float>(sizeof(float) * (size_t)h->attn_rows * c.n_heads * h->nb_cap * (c.head_dim + 4));
  h->attn_counters = cv.take<unsigned>(sizeof(unsigned) * (size_t)M * c.n_kv_heads);
  h->logits = cv.take<float>(sizeof(float) * (size_t)h->head_max * c.vocab * kMaxSplitK);
  const int gc = c.gamma_max + 1;
  h->stash_x = cv.take<float>(sizeof(float) * (size_t)c.max_batch * gc * d);
  h->stash_s = cv.take<float>(sizeof(float) * (size_t)c.max_batch * gc * d);
  h->drafts = cv.take<int>(sizeof(int) * c.max_batch * gc);
  h->pending = cv.take<int>(sizeof(int) * c.max_batch);
  h->vtok = cv.take<int>(sizeof(int) * c.max_batch * gc);
  h->accepted = cv.take<unsigned long long>(sizeof(unsigned long long) * 2);
  h->spec_io = cv.take<SpecIo>(sizeof(SpecIo));
  h->spec_flags = cv.take<int>(sizeof(int) * 4);
  // two GEMMs per physical layer per application, plus the LM head
  h->pf_nseg_max = 2 * (c.n_in + c.n_out + c.k_max * c.n_rec) + 1;
  h->pf_segs = cv.take<PfSeg>(sizeof(PfSeg) * (size_t)c.k_max * h->pf_nseg_max);
  return cv.off + 256;
}

// ------------------------------------------------------------------ profiling
struct Scope {
  dory_handle* H;
  cudaStream_t st;
  ProfRec rec{};
  bool on;
  Scope(dory_handle* h, cudaStream_t s, const char* name, double bytes) : H(h), st(s), on(h->profile) {
    if (!on) return;
    int id = -1;
    for (size_t i = 0; i < H->prof_names.size(); ++i)
      if (H->prof_names[i] == name) id = (int)i;
    if (id < 0) {
      id = (int)H->prof_names.size();
      H->prof_names.push_back(name);
    }
    rec.name = id;
    rec.bytes = bytes;
    rec.a = event();
    rec.b = event();
    cudaEventRecord(rec.a, st);
  }
  cudaEvent_t event() {
    if (H->ev_used == H->ev_pool.size()) {
      cudaEvent_t e;
      cudaEventCreate(&e);
      H->ev_pool.push_back(e);
    }
    return H->ev_pool[H->ev_used++];
  }
  ~Scope() {
    if (!on) return;
    cudaEventRecord(rec.b, st);
    H->prof_recs.push_back(rec);
  }
};

// ------------------------------------------------------------------ forward pieces
template <typename T>
struct Fwd {
  dory_handle* H;
  cudaStream_t st;
  int M;        // chunk rows
  int max_ctx;  // bound on (position + 1) of every row
  bool direct;  // K/V of the chunk go straight into the cache
  int mode;     // dory_cache_mode
  int k;        // loop count of this pass (last loop = k)
  int batch;    // sequences in the call (selects the GEMM split)
  bool invariant;  // decode / speculative rows: GEMM arithmetic independent of M
  int n_tiles = 0;  // > 0: long-chunk attention on the tensor cores over H->tiles
  int tc5 = 0;      // ... by a tcgen05 kernel (128-row tiles): 2 one slot per CTA, 3 warp-specialised
  int n_items = 0;  // work items of the warp-specialised kernel (H->pf_items)
  int pf_k = 0;     // > 0: GEMMs follow the weight stream of a pf_k-loop decode step
  bool stage = true;  // layer updates may run in the next GEMM's operand stage
};

KVView kv_view(dory_handle* H, int l, int loop, int mode) {
  AttnLayer& a = H->attn[H->attn_of[l]];
  int slot = (mode == DORY_PER_LOOP && a.rec && loop >= 1) ? loop - 1 : 0;
  KVView v;
  v.K = a.K[slot];
  v.V = a.V[slot];
  v.cap = a.cap;
  v.window = a.full ? 0 : H->c.swa_window;
  v.limit = H->c.max_seq;
  v.err = H->err;
  if (a.full && H->page_table) {
    v.pt = H->page_table;
    v.pt_stride = H->pt_stride;
    v.page_shift = H->page_shift;
  }
  return v;
}

// Rows of head_dim elements in one K (or V) buffer of layer l's cache.
size_t kv_rows(dory_handle* H, int l) {
  const AttnLayer& a = H->attn[H->attn_of[l]];
  if (a.full && H->page_table) return (size_t)H->pool_pages * H->c.n_kv_heads * (1 << H->page_shift);
  return (size_t)H->c.max_batch * H->c.n_kv_heads * a.cap;
}

// Paged cache: give every listed sequence the pages that hold positions
// 0 .. upto[i] - 1, and upload the new page-table entries.  Checks the free
// pool first, so a refused call changes nothing.
dory_status ensure_pages(dory_handle* H, int n, const int32_t* seq_ids, const int64_t* upto, cudaStream_t st) {
  if (!H->page_table) return DORY_OK;
  const int P = H->c.kv_page;
  int64_t need = 0;
  for (int i = 0; i < n; ++i)
    need += std::max<int64_t>(0, (upto[i] + P - 1) / P - (int64_t)H->seq_pages[seq_ids[i]].size());
  if (need > (int64_t)H->free_pages.size())
    return fail(DORY_ERR_CAPACITY, "the paged cache needs %lld more pages, %zu are free", (long long)need,
                H->free_pages.size());
  for (int i = 0; i < n; ++i) {
    const int sq = seq_ids[i];
    std::vector<int>& mine = H->seq_pages[sq];
    const int first = (int)mine.size(), want = (int)((upto[i] + P - 1) / P);
    if (want <= first) continue;
    for (int q = first; q < want; ++q) {
      mine.push_back(H->free_pages.back());
      H->free_pages.pop_back();
      H->pt_host[(size_t)sq * H->pt_stride + q] = mine.back();
    }
    const size_t at = (size_t)sq * H->pt_stride + first;
    CK(cudaMemcpyAsync(H->page_table + at, H->pt_host.data() + at, sizeof(int) * (want - first),
                       cudaMemcpyHostToDevice, st));
  }
  return DORY_OK;
}

void release_pages(dory_handle* H, int seq) {
  if (!H->page_table) return;
  for (int p : H->seq_pages[seq]) H->free_pages.push_back(p);
  H->seq_pages[seq].clear();
}

// Rows per split slice of a GEMM output buffer for this pass.
template <typename T>
size_t prows(const Fwd<T>& f) {
  return f.invariant ? f.H->part_rows_dec : f.H->part_rows;
}

// Y (and, when the tensor-core kernel splits K, the slices after it) must
// hold kMaxSplitK slices of part_rows rows of ldy floats.
// prep: an operand stage the caller has checked with stage_ok (bf16
// tensor-core decode GEMMs only); X is then unused.
// after_attn: the GEMM follows a decode attention launch; its look-ahead
// then covers pf_attn bytes and is issued before it waits (see PfCtl).
template <typename T>
dory_status gemm(const Fwd<T>& f, int M, int N, int K, const T* X, int ldx, const void* W, float* Y, int ldy,
                 size_t part_rows, int* S_out, size_t* ps_out, const char* name, const Prep* prep = nullptr,
                 bool after_attn = false) {
  dory_handle* H = f.H;
  *S_out = 1;
  *ps_out = 0;
  if constexpr (sizeof(T) == 2) {
    // decode and speculative rows read the MXFP8 copy when one is attached
    if (f.invariant && !H->mx.empty()) {
      auto it = H->mx.find(W);
      if (it != H->mx.end() && it->second.fmt == 1) {
        // NVFP4: the TMA-fed tensor-core GEMM with split-K slices
        Scope sc(H, f.st, name, (double)N * K * (0.5 + 1.0 / 16) + (double)M * K * 2 + (double)M * N * 4);
        const int S = nv_gemm_splits(N, K);
        const size_t ps = part_rows * (size_t)ldy;
        cudaError_t e = launch_nv_gemm_tc(M, N, K, (const bf16*)X, ldx, it->second.q, it->second.s, it->second.g, Y,
                                          ldy, ps, S, H->err, f.st);
        if (e == cudaErrorNotSupported) return fail(DORY_ERR_UNSUPPORTED, "%s: shape not supported by NVFP4", name);
        if (e != cudaSuccess) return fail(DORY_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e));
        *S_out = S;
        *ps_out = ps;
        return DORY_OK;
      }
      if (it != H->mx.end()) {
        Scope sc(H, f.st, name, (double)N * K * (1.0 + 1.0 / kMxBlock) + (double)M * K * 2 + (double)M * N * 4);
        if (H->mx_impl == 3) {
          // TMA-fed tensor-core GEMM with split-K slices; shapes it does not take use the CUDA-core GEMV
          // (whose rows differ in their last bits, so a handle mixing the two loses row-count invariance)
          const int S = mx_gemm_splits(N, K);
          const size_t ps = part_rows * (size_t)ldy;
          cudaError_t e = launch_mx_gemm_tc(M, N, K, (const bf16*)X, ldx, it->second.q, it->second.s, Y, ldy, ps, S,
                                            H->err, f.st);
          if (e == cudaSuccess) {
            *S_out = S;
            *ps_out = ps;
            return DORY_OK;
          }
          if (e != cudaErrorNotSupported) return fail(DORY_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e));
        }
        const int impl = H->mx_impl == 3 ? 1 : H->mx_impl;
        const int S = impl == 2 ? 1 : mx_gemv_splits(N, K);
        const size_t ps = part_rows * (size_t)ldy;
        CK(launch_mx_gemv(M, N, K, (const bf16*)X, ldx, it->second.q, it->second.s, Y, ldy, H->err, f.st, impl, S,
                          ps));
        *S_out = S;
        *ps_out = ps;
        return DORY_OK;
      }
    }
  }
  double bytes = (double)N * K * sizeof(T) + (double)M * K * sizeof(T) + (double)M * N * 4;
  Scope sc(H, f.st, name, bytes);
  if constexpr (sizeof(T) == 2) {
    if (H->gemm_impl != 1) {
      int S = 1;
      size_t ps = 0;
      // L2 look-ahead while this GEMM is the next one of the weight stream
      PfCtl pfc;
      const PfCtl* pp = nullptr;
      if (f.invariant && H->pf_own > 0) {
        pfc.own = H->pf_own;
        pp = &pfc;
      }
      if (f.pf_k > 0 && H->pf_pos >= 0) {
        const std::vector<PfSeg>& v = H->pf_host[f.pf_k];
        if (H->pf_pos < (int)v.size() && v[H->pf_pos].p == (const char*)W) {
          const unsigned long long end = v[H->pf_pos].off + v[H->pf_pos].bytes;
          const unsigned long long total = v.back().off + v.back().bytes;
          pfc.segs = H->pf_segs + (size_t)(f.pf_k - 1) * H->pf_nseg_max;
          pfc.nseg = (int)v.size();
          pfc.first = H->pf_pos + 1;
          const bool early = after_attn && H->pf_attn > 0;
          pfc.early = early ? 1 : 0;
          pfc.lo = std::max(H->pf_done, end);
          pfc.hi = std::min(end + (early ? H->pf_attn : H->pf_lead), total);
          if (pfc.lo < pfc.hi) {
            // start the segment walk at the segment holding lo
            while (pfc.first + 1 < pfc.nseg && v[pfc.first + 1].off <= pfc.lo) ++pfc.first;
            H->pf_done = pfc.hi;
            pp = &pfc;
          }
          ++H->pf_pos;
        } else {
          H->pf_pos = -1;  // the pass left the stream: no further look-ahead
        }
      }
      // the projection after a decode attention leaves the attention's SMs free
      int cap = 0;
      if (after_attn && f.invariant) {
        const int busy = attn_decode_ctas(f.batch, H->c.n_kv_heads, H->c.head_dim, H->c.n_heads / H->c.n_kv_heads);
        cap = busy > 0 && busy < 148 ? 148 - busy : 0;
      }
      cudaError_t e = launch_gemm_tc(M, N, K, (const bf16*)X, ldx, (const bf16*)W, Y, ldy, part_rows,
                                     H->err, f.batch, f.invariant, &S, &ps, f.st, 0, false, pp, prep, cap);
      if (e == cudaSuccess) {
        *S_out = S;
        *ps_out = ps;
        return DORY_OK;
      }
      if (prep) return fail(DORY_ERR_CUDA, "%s: operand stage: %s", name, cudaGetErrorString(e));
      if (e != cudaErrorNotSupported) return fail(DORY_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e));
      if (H->gemm_impl == 2) return fail(DORY_ERR_UNSUPPORTED, "%s: shape not supported by tcgen05 GEMM", name);
    }
  }
  CK(launch_gemm_simt<T>(M, N, K, X, ldx, (const T*)W, Y, ldy, f.st));
  return DORY_OK;
}

#define RET(x)                          \
  do {                                  \
    dory_status r_ = (x);               \
    if (r_ != DORY_OK) return r_;       \
  } while (0)

// Whether the GEMM of weight W ([N, K]) on this pass can take operand stage p.
template <typename T>
bool stage_ok(const Fwd<T>& f, int N, int K, const void* W, const Prep& p) {
  const dory_handle* H = f.H;
  if (sizeof(T) != 2 || !f.stage || !f.invariant || f.M > H->fuse_rows || H->gemm_impl == 1) return false;
  if (!H->mx.empty() && H->mx.count(W)) return false;
  return gemm_tc_prep_ok(f.M, N, K, f.batch, p);
}

// Apply physical layers l0..l1-1.  copy_last (if not NULL) also receives the
// result of the last layer.
//
// Each layer ends with h <- N(h + y).  On decode and speculative passes of
// few rows that update is carried to the next layer's first GEMM, which
// applies it in its operand stage (reading h from one state buffer and
// writing the other), and the SwiGLU of the gate-up product is applied by
// the down projection's operand stage.  The last layer's update runs as its
// own kernel, and so does any update the next GEMM cannot take.
template <typename T>
dory_status run_layers(const Fwd<T>& f, int l0, int l1, int loop, float* copy_last = nullptr) {
  dory_handle* H = f.H;
  const dory_config& c = H->c;
  const int M = f.M, d = c.d_model;
  bool pend = false;  // h <- N(h + part_y) of the previous layer not yet applied
  int S_pend = 1;
  size_t ps_pend = 0;
  auto flush = [&](float* copy) -> dory_status {
    Scope sc(H, f.st, "addnorm", 0);
    CK(launch_addnorm<T>(M, d, H->hcur(), H->hcur(), H->part_y, S_pend, ps_pend, d, H->hop_t<T>(), copy, f.st,
                         !f.invariant));
    pend = false;
    return DORY_OK;
  };
  // operand stage applying the pending update, or NULL after flushing it
  auto take_pending = [&](int N, const void* W, Prep* p) -> const Prep* {
    if (!pend) return nullptr;
    p->mode = kPrepAddNorm;
    p->h_in = H->hcur();
    p->h_out = H->hb[H->hc ^ 1];
    p->y = H->part_y;
    p->S = S_pend;
    p->ps = ps_pend;
    p->ldy = d;
    return stage_ok(f, N, d, W, *p) ? p : nullptr;
  };
  for (int l = l0; l < l1; ++l) {
    int S;
    size_t ps;
    if (layer_is_attn(l)) {
      KVView kv = kv_view(H, l, loop, f.mode);
      Prep pq;
      const Prep* pre = take_pending(H->qkv_dim, H->w_qkv[l], &pq);
      if (pend && !pre) RET(flush(nullptr));
      RET(gemm<T>(f, M, H->qkv_dim, d, H->hop_t<T>(), d, H->w_qkv[l], H->part_qkv, H->qkv_dim, prows(f), &S, &ps,
                  pre ? "gemm_qkv_norm" : "gemm_qkv", pre));
      if (pre) {
        H->hc ^= 1;
        pend = false;
      }
      if (f.direct) {
        // fused: q from the partials, own K/V into the cache, split-KV attention
        Scope sc(H, f.st, "attn_decode", 0);
        CK(launch_attn_decode<T>(M, c.n_heads, c.n_kv_heads, c.head_dim, H->part_qkv, S, ps, kv, H->meta, f.max_ctx,
                                 H->attn_part, H->nb_cap, H->attn_rows, H->attn_counters, (T*)H->ao, f.batch,
                                 f.st));
      } else {
        // long chunks: K/V into scratch, attention, then the cache commit
        const bool tc = f.n_tiles > 0;
        {
          Scope sc(H, f.st, "qkv_post", 0);
          CK(launch_qkv_post<T>(M, c.n_heads, c.n_kv_heads, c.head_dim, H->part_qkv, S, ps, H->q, (T*)H->kscr,
                                (T*)H->vscr, false, kv, H->meta, c.max_batch, tc ? (bf16*)H->qh : nullptr, f.st));
        }
        if (tc) {
          Scope sc(H, f.st, "attn_prefill", 0);
          if (f.tc5 == 3)
            CK(launch_attn_prefill_ws(f.n_items, H->pf_items, H->tiles, M, c.n_heads, c.n_kv_heads, c.head_dim,
                                      (const bf16*)H->qh, (const bf16*)H->kscr, (const bf16*)H->vscr, kv,
                                      kv_rows(H, l), H->meta, (bf16*)H->ao, f.st));
          else if (f.tc5 == 2)
            CK(launch_attn_prefill_tc(f.n_tiles, H->tiles, c.n_heads, c.n_kv_heads, c.head_dim, (const bf16*)H->qh,
                                      (const bf16*)H->kscr, (const bf16*)H->vscr, kv, H->meta, (bf16*)H->ao, f.st));
          else
            CK(launch_attn_prefill(f.n_tiles, H->tiles, c.n_heads, c.n_kv_heads, c.head_dim, (const bf16*)H->qh,
                                   (const bf16*)H->kscr, (const bf16*)H->vscr, kv, H->meta, (bf16*)H->ao, f.st));
        } else {
          Scope sc(H, f.st, "attention", 0);
          CK(launch_attention<T>(M, c.n_heads, c.n_kv_heads, c.head_dim, H->q, (const T*)H->kscr,
                                 (const T*)H->vscr, true, kv, H->meta, f.max_ctx, H->attn_part, H->attn_rows,
                                 (T*)H->ao, f.st));
        }
        // A last-loop recurrent layer shares one slot across loops, so the
        // chunk's keys are committed only after the final loop: committing
        // loop t earlier would overwrite ring entries of earlier positions
        // that loop t+1 of this chunk still reads.
        const bool rec = H->attn[H->attn_of[l]].rec;
        if (!rec || f.mode == DORY_PER_LOOP || loop == f.k) {
          Scope sc(H, f.st, "kv_commit", 0);
          CK(launch_kv_commit<T>(M, c.n_kv_heads, c.head_dim, (const T*)H->kscr, (const T*)H->vscr, kv, H->meta,
                                 f.st));
        }
      }
      RET(gemm<T>(f, M, d, H->q_dim, (const T*)H->ao, H->q_dim, H->w_o[l], H->part_y, d, prows(f), &S, &ps, "gemm_o",
                  nullptr, f.direct));
    } else {
      bool fused = false;
      if constexpr (sizeof(T) == 2) {
        // long chunks: gate-up GEMM with SwiGLU in its epilogue
        if (!f.invariant && H->gemm_impl != 1) {
          if (pend) RET(flush(nullptr));
          Scope sc(H, f.st, "gemm_gate_up_glu", 4.0 * c.d_ff * d + 2.0 * M * d + 2.0 * M * c.d_ff);
          cudaError_t e = launch_gemm_glu(M, c.d_ff, d, (const bf16*)H->hop, d, (const bf16*)H->w_gu[l],
                                          (bf16*)H->act, H->err, f.st);
          if (e == cudaSuccess)
            fused = true;
          else if (e != cudaErrorNotSupported)
            return fail(DORY_ERR_CUDA, "gemm_gate_up_glu: %s", cudaGetErrorString(e));
        }
      }
      if (fused) {
        RET(gemm<T>(f, M, d, c.d_ff, (const T*)H->act, c.d_ff, H->w_down[l], H->part_y, d, prows(f), &S, &ps,
                    "gemm_down"));
      } else {
        Prep pg;
        const Prep* pre = take_pending(2 * c.d_ff, H->w_gu[l], &pg);
        if (pend && !pre) RET(flush(nullptr));
        RET(gemm<T>(f, M, 2 * c.d_ff, d, H->hop_t<T>(), d, H->w_gu[l], H->part_gu, 2 * c.d_ff, prows(f), &S, &ps,
                    pre ? "gemm_gate_up_norm" : "gemm_gate_up", pre));
        if (pre) {
          H->hc ^= 1;
          pend = false;
        }
        // the down projection applies the SwiGLU in its operand stage when it can
        Prep pd;
        pd.mode = kPrepSwiglu;
        pd.y = H->part_gu;
        pd.S = S;
        pd.ps = ps;
        pd.ldy = 2 * c.d_ff;
        const bool st_ok = stage_ok(f, d, c.d_ff, H->w_down[l], pd);
        if (!st_ok) {
          Scope sc(H, f.st, "swiglu", 0);
          CK(launch_swiglu<T>(M, c.d_ff, H->part_gu, S, ps, (T*)H->act, f.st));
        }
        RET(gemm<T>(f, M, d, c.d_ff, (const T*)H->act, c.d_ff, H->w_down[l], H->part_y, d, prows(f), &S, &ps,
                    st_ok ? "gemm_down_swiglu" : "gemm_down", st_ok ? &pd : nullptr));
      }
    }
    pend = true;
    S_pend = S;
    ps_pend = ps;
  }
  if (pend) RET(flush(copy_last));
  return DORY_OK;
}

// Embed + input block; x <- h.
template <typename T>
dory_status input_block(const Fwd<T>& f, const int* tokens) {
  dory_handle* H = f.H;
  const dory_config& c = H->c;
  {
    Scope sc(H, f.st, "embed", 0);
    H->hc = 0;  // every pass starts its state in the first buffer
    CK(launch_embed<T>(f.M, c.d_model, c.vocab, tokens, (const T*)H->embed, H->hcur(), H->hop_t<T>(),
                       c.n_in == 0 ? H->x : nullptr, H->err, f.st));
  }
  RET(run_layers<T>(f, 0, c.n_in, 0, H->x));
  return DORY_OK;
}

// Loops t0..k of the recurrent block; on entry h holds x (t0 == 1) or s
// holds s_{t0-1} (t0 > 1).  Leaves s_k in h and s.  If stash_col >= 0, s_1
// is written to the stash (rows_per_seq rps).
template <typename T>
dory_status loops(const Fwd<T>& f, int t0, int k, int stash_col, int rps) {
  dory_handle* H = f.H;
  const dory_config& c = H->c;
  const int d = c.d_model, gc = c.gamma_max + 1;
  for (int t = t0; t <= k; ++t) {
    // entry: u_t = N(s_{t-1} + x); s_0 = x; s_{t-1} = N(h) after loop t-1
    int src = (t == 1) ? 0 : (t == t0 ? 2 : 1);
    float* save = (t > 1 && t - 1 == 1 && stash_col >= 0) ? H->stash_s : nullptr;
    {
      Scope sc(H, f.st, "reinject", 0);
      CK(launch_reinject<T>(f.M, d, H->hcur(), H->x, src, H->s, true, H->hop_t<T>(), save, rps, gc,
                            stash_col < 0 ? 0 : stash_col, f.st));
    }
    RET(run_layers<T>(f, c.n_in, c.n_in + c.n_rec, t));
  }
  // exit: s_k = N(h) (or s_k = s when no loop ran here); s_k is kept in s,
  // or in the speculative stash when a stash column is given
  Scope sc(H, f.st, "reinject", 0);
  if (t0 > k) {
    CK(launch_reinject<T>(f.M, d, H->hcur(), H->x, 2, H->s, false, H->hop_t<T>(), nullptr, 1, 1, 0, f.st));
  } else if (stash_col >= 0 && k == 1) {
    CK(launch_reinject<T>(f.M, d, H->hcur(), H->x, 1, nullptr, false, H->hop_t<T>(), H->stash_s, rps, gc, stash_col,
                          f.st));
  } else {
    CK(launch_reinject<T>(f.M, d, H->hcur(), H->x, 1, nullptr, false, H->hop_t<T>(), H->s, 1, 1, 0, f.st));
  }
  return DORY_OK;
}

// Output block on h, then LM head + argmax on `nrows` rows (all rows when
// rows == nullptr, else the listed rows).  Choices go to `choice`.
template <typename T>
dory_status output_and_head(const Fwd<T>& f, int nrows, const int* rows, float* logits_out, int* choice) {
  dory_handle* H = f.H;
  const dory_config& c = H->c;
  const int d = c.d_model;
  RET(run_layers<T>(f, c.n_in + c.n_rec, H->L, 0));
  const T* X = H->hop_t<T>();
  if (rows) {
    Scope sc(H, f.st, "gather", 0);
    CK(launch_gather_rows<T>(nrows, d, rows, H->hop_t<T>(), (T*)H->hop_head, f.st));
    X = (const T*)H->hop_head;
  }
  // partial slices live in the internal logits buffer (kMaxSplitK slices
  // of head_max rows); a split result is reduced into the output in order
  int S;
  size_t ps;
  RET(gemm<T>(f, nrows, c.vocab, d, X, d, H->head, H->logits, c.vocab, H->head_max, &S, &ps, "gemm_lm_head"));
  float* lg = logits_out ? logits_out : H->logits;
  if (S != 1 || lg != H->logits) {
    Scope sc(H, f.st, "split_reduce", 0);
    CK(launch_split_reduce(nrows, c.vocab, H->logits, S, ps, lg, f.st));
  }
  if (H->temperature > 0.f) {
    // the draw of head row i is keyed by the sequence and the new token's position
    Scope sc(H, f.st, "sample", 0);
    CK(launch_sample(nrows, c.vocab, lg, (uint32_t*)H->logits, rows, H->meta.seq, H->meta.pos, 1, H->temperature,
                     H->top_p, H->seed, choice, f.st));
    return DORY_OK;
  }
  Scope sc(H, f.st, "argmax", 0);
  CK(launch_argmax(nrows, c.vocab, lg, choice, f.st));
  return DORY_OK;
}

dory_status upload_ids(dory_handle* H, const int32_t* ids, int n, cudaStream_t st) {
  if ((int)H->ids_on_device.size() == n && std::equal(ids, ids + n, H->ids_on_device.begin())) return DORY_OK;
  CK(cudaMemcpyAsync(H->seq_ids, ids, sizeof(int) * n, cudaMemcpyHostToDevice, st));
  H->ids_on_device.assign(ids, ids + n);
  return DORY_OK;
}

dory_status check_seqs(dory_handle* H, int batch, const int32_t* seq_ids, int k, int mode) {
  const dory_config& c = H->c;
  if (batch <= 0 || batch > c.max_batch) return fail(DORY_ERR_INVALID_ARG, "batch %d outside 1..%d", batch, c.max_batch);
  if (!seq_ids) return fail(DORY_ERR_INVALID_ARG, "seq_ids is NULL");
  if (k < 1 || k > c.k_max) return fail(DORY_ERR_INVALID_ARG, "k=%d outside 1..%d", k, c.k_max);
  if (mode != DORY_LAST_LOOP && mode != DORY_PER_LOOP) return fail(DORY_ERR_INVALID_ARG, "bad cache mode");
  if (mode == DORY_PER_LOOP && H->alloc_mode != DORY_PER_LOOP)
    return fail(DORY_ERR_STATE, "per_loop call on a handle allocated for last_loop");
  for (int i = 0; i < batch; ++i) {
    int sq = seq_ids[i];
    if (sq < 0 || sq >= c.max_batch) return fail(DORY_ERR_INVALID_ARG, "seq id %d outside 0..%d", sq, c.max_batch - 1);
    for (int j = 0; j < i; ++j)
      if (seq_ids[j] == sq) return fail(DORY_ERR_INVALID_ARG, "seq id %d repeated", sq);
    if (H->mode[sq] >= 0 && H->mode[sq] != mode)
      return fail(DORY_ERR_STATE, "sequence %d was started in the other cache mode", sq);
    if (mode == DORY_PER_LOOP && H->mode[sq] >= 0 && H->kfix[sq] != k)
      return fail(DORY_ERR_STATE, "per_loop sequence %d was started at k=%d, not %d", sq, H->kfix[sq], k);
  }
  return DORY_OK;
}

void mark_started(dory_handle* H, int batch, const int32_t* seq_ids, int k, int mode) {
  for (int i = 0; i < batch; ++i) {
    int sq = seq_ids[i];
    if (H->mode[sq] < 0) {
      H->mode[sq] = mode;
      H->kfix[sq] = k;
    }
  }
}

template <typename T>
dory_status prefill_t(dory_handle* H, int batch, const int32_t* seq_ids, const int32_t* tokens, const int32_t* lens,
                      int k, int mode, float* last_logits, int32_t* next_tokens, cudaStream_t st) {
  const dory_config& c = H->c;
  std::vector<int> cu(batch + 1, 0), rows(batch);
  int max_ctx = 0;
  for (int i = 0; i < batch; ++i) {
    cu[i + 1] = cu[i] + lens[i];
    rows[i] = cu[i + 1] - 1;
    max_ctx = std::max(max_ctx, H->len[seq_ids[i]] + lens[i]);
  }
  const int M = cu[batch];
  RET(upload_ids(H, seq_ids, batch, st));
  CK(cudaMemcpyAsync(H->cu, cu.data(), sizeof(int) * (batch + 1), cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(H->head_rows, rows.data(), sizeof(int) * batch, cudaMemcpyHostToDevice, st));
  CK(launch_plan_ragged(batch, M, H->cu, H->seq_ids, H->seq_len, H->meta, st));
  int max_len = *std::max_element(lens, lens + batch);
  // short chunks write K/V straight into the cache (the decode attention,
  // whose split-KV partials hold attn_rows rows)
  Fwd<T> f{H, st, M, max_ctx, max_len <= H->slack + 1 && M <= H->attn_rows, mode, k, batch, false};
  if (!f.direct && H->bf16 && attn_prefill_supported(c.head_dim) && H->prefill_tc) {
    f.tc5 = H->prefill_tc >= 2 && attn_prefill_tc_supported(c.head_dim) ? H->prefill_tc : 0;
    std::vector<int2> tl(H->tiles_cap);
    const int n = prefill_tiles(batch, cu.data(), tl.data(), H->tiles_cap, f.tc5 ? 128 : 64);
    if (n < 0) return fail(DORY_ERR_CAPACITY, "too many prefill attention tiles");
    CK(cudaMemcpyAsync(H->tiles, tl.data(), sizeof(int2) * n, cudaMemcpyHostToDevice, st));
    f.n_tiles = n;
    if (f.tc5 == 3) {
      // each tile's sequence and last position, for pairing and ordering
      std::vector<int> last(n), sq(n);
      for (int t = 0, b = 0; t < n; ++t) {
        while (tl[t].x >= cu[b + 1]) ++b;
        sq[t] = b;
        last[t] = H->len[seq_ids[b]] + (tl[t].y - 1 - cu[b]);
      }
      H->items_host.resize(H->items_cap);
      const int ni = prefill_ws_items(n, last.data(), sq.data(), c.n_heads, c.n_kv_heads, H->items_host.data(),
                                      H->items_cap);
      if (ni < 0) return fail(DORY_ERR_CAPACITY, "too many prefill attention items");
      CK(cudaMemcpyAsync(H->pf_items, H->items_host.data(), sizeof(int4) * ni, cudaMemcpyHostToDevice, st));
      f.n_items = ni;
    }
  }
  RET(input_block<T>(f, tokens));
  RET(loops<T>(f, 1, k, -1, 1));
  RET(output_and_head<T>(f, batch, H->head_rows, last_logits, next_tokens));
  CK(launch_advance_ragged(batch, H->seq_ids, H->cu, H->seq_len, st));
  for (int i = 0; i < batch; ++i) H->len[seq_ids[i]] += lens[i];
  H->last_rows = M;
  return DORY_OK;
}

// The weights a k-loop decode step reads, in the order its GEMMs read them:
// per physical layer QKV then O (attention) or gate-up then down (MLP); the
// input block, k passes over the recurrent block, the output block, the LM
// head.  Uploaded once per k (outside any graph capture).
dory_status ensure_stream(dory_handle* H, int k, cudaStream_t st) {
  if (H->pf_lead == 0 || !H->bf16 || H->gemm_impl == 1 || !H->mx.empty()) return DORY_OK;
  if ((int)H->pf_host.size() <= k) {
    H->pf_host.resize(k + 1);
    H->pf_uploaded.resize(k + 1, 0);
  }
  if (H->pf_uploaded[k]) return DORY_OK;
  const dory_config& c = H->c;
  const unsigned long long d = c.d_model, e = 2;
  std::vector<PfSeg>& v = H->pf_host[k];
  v.clear();
  unsigned long long off = 0;
  auto add = [&](const void* p, unsigned long long bytes) {
    v.push_back({(const char*)p, off, bytes});
    off += bytes;
  };
  auto layer = [&](int l) {
    if (layer_is_attn(l)) {
      add(H->w_qkv[l], (unsigned long long)H->qkv_dim * d * e);
      add(H->w_o[l], d * H->q_dim * e);
    } else {
      add(H->w_gu[l], 2ull * c.d_ff * d * e);
      add(H->w_down[l], d * c.d_ff * e);
    }
  };
  for (int l = 0; l < c.n_in; ++l) layer(l);
  for (int t = 1; t <= k; ++t)
    for (int l = c.n_in; l < c.n_in + c.n_rec; ++l) layer(l);
  for (int l = c.n_in + c.n_rec; l < H->L; ++l) layer(l);
  add(H->head, (unsigned long long)c.vocab * d * e);
  if ((int)v.size() > H->pf_nseg_max) return fail(DORY_ERR_STATE, "weight stream larger than its buffer");
  CK(cudaMemcpyAsync(H->pf_segs + (size_t)(k - 1) * H->pf_nseg_max, v.data(), sizeof(PfSeg) * v.size(),
                     cudaMemcpyHostToDevice, st));
  H->pf_uploaded[k] = 1;
  return DORY_OK;
}

// Let the GEMMs of a pass follow the weight stream of a k-loop decode step
// from its segment `pos` on (L2 look-ahead), when that stream is uploaded.
template <typename T>
void follow_stream(dory_handle* H, Fwd<T>& f, int k, int pos) {
  const bool on = H->pf_lead > 0 && H->mx.empty() && (int)H->pf_uploaded.size() > k && H->pf_uploaded[k];
  f.pf_k = on ? k : 0;
  H->pf_pos = on ? pos : -1;
  H->pf_done = 0;
}

template <typename T>
dory_status decode_body(dory_handle* H, int batch, const int32_t* tokens_in, int k, int mode, int max_ctx,
                        float* logits, int32_t* next_tokens, cudaStream_t st) {
  const bool pf = H->pf_lead > 0 && H->mx.empty() && (int)H->pf_uploaded.size() > k && H->pf_uploaded[k];
  H->pf_pos = pf ? 0 : -1;
  H->pf_done = 0;
  CK(launch_plan_uniform(batch, 1, 0, H->seq_ids, H->seq_len, H->meta, st));
  Fwd<T> f{H, st, batch, max_ctx, true, mode, k, batch, true};
  f.pf_k = pf ? k : 0;
  RET(input_block<T>(f, tokens_in));
  RET(loops<T>(f, 1, k, -1, 1));
  RET(output_and_head<T>(f, batch, nullptr, logits, next_tokens));
  CK(launch_advance(batch, H->seq_ids, H->seq_len, 1, st));
  return DORY_OK;
}

// Decode steps without logits replay a CUDA graph of the whole step (captured
// on the second call with the same batch, k and mode; the first call also
// initialises the kernels' attributes outside any capture).  Inputs are copied
// into the handle's buffers first, outputs copied out after, so the graph only
// touches workspace memory; attention grids are sized for max_seq.
template <typename T>
dory_status decode_t(dory_handle* H, int batch, const int32_t* seq_ids, const int32_t* tokens_in, int k, int mode,
                     float* logits, int32_t* next_tokens, cudaStream_t st) {
  int max_ctx = 0;
  for (int i = 0; i < batch; ++i) max_ctx = std::max(max_ctx, H->len[seq_ids[i]] + 1);
  RET(upload_ids(H, seq_ids, batch, st));
  RET(ensure_stream(H, k, st));
  const bool use_graph = H->graphs && !H->profile && logits == nullptr;
  if (!use_graph) {
    RET(decode_body<T>(H, batch, tokens_in, k, mode, max_ctx, logits, next_tokens, st));
  } else {
    const long long key = ((long long)batch << 16) | (k << 4) | mode;
    dory_handle::Graph* g = nullptr;
    for (auto& e : H->graphs_cache)
      if (e.key == key) g = &e;
    if (!g) {
      H->graphs_cache.push_back({key, 0, nullptr, 0});
      g = &H->graphs_cache.back();
    }
    CK(cudaMemcpyAsync(H->tokens, tokens_in, sizeof(int) * batch, cudaMemcpyDeviceToDevice, st));
    if (!g->exec && g->seen == 0) {
      g->seen = 1;
      RET(decode_body<T>(H, batch, H->tokens, k, mode, H->c.max_seq, nullptr, H->next, st));
    } else {
      if (!g->exec) {
        // record on a private stream (the caller's may be the legacy default
        // stream, which cannot be captured); nothing runs while recording
        if (!H->cap_stream) CK(cudaStreamCreateWithFlags(&H->cap_stream, cudaStreamNonBlocking));
        cudaStream_t cs = H->cap_stream;
        cudaGraph_t graph = nullptr;
        CK(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal));
        dory_status r = decode_body<T>(H, batch, H->tokens, k, mode, H->c.max_seq, nullptr, H->next, cs);
        cudaError_t e = cudaStreamEndCapture(cs, &graph);
        if (r != DORY_OK) {
          if (graph) cudaGraphDestroy(graph);
          return r;
        }
        if (e != cudaSuccess) return fail(DORY_ERR_CUDA, "graph capture: %s", cudaGetErrorString(e));
        e = cudaGraphInstantiate(&g->exec, graph, 0);
        cudaGraphDestroy(graph);
        if (e != cudaSuccess) {
          g->exec = nullptr;
          return fail(DORY_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(e));
        }
        g->hc_end = H->hc;
      }
      CK(cudaGraphLaunch(g->exec, st));
      H->hc = g->hc_end;
    }
    CK(cudaMemcpyAsync(next_tokens, H->next, sizeof(int) * batch, cudaMemcpyDeviceToDevice, st));
  }
  for (int i = 0; i < batch; ++i) H->len[seq_ids[i]] += 1;
  H->last_rows = batch;
  return DORY_OK;
}

// A decode step with a loop count per sequence; rows are ordered by
// non-increasing k, so loop t runs on the prefix of rows whose k >= t.  Rows
// that have finished keep their last output (and, in last-loop mode, their
// own final-loop K/V); the exit normalisation s_k = N(h) covers every row.
// The decode GEMMs are row-count invariant, so each row's arithmetic does
// not depend on how many rows share a loop.
template <typename T>
dory_status decode_mixed_t(dory_handle* H, int batch, const int32_t* seq_ids, const int32_t* tokens_in,
                           const int32_t* ks, int mode, float* logits, int32_t* next_tokens, cudaStream_t st) {
  const dory_config& c = H->c;
  int max_ctx = 0;
  for (int i = 0; i < batch; ++i) max_ctx = std::max(max_ctx, H->len[seq_ids[i]] + 1);
  const int kmax = ks[0], d = c.d_model;
  RET(upload_ids(H, seq_ids, batch, st));
  RET(ensure_stream(H, kmax, st));
  CK(launch_plan_uniform(batch, 1, 0, H->seq_ids, H->seq_len, H->meta, st));
  Fwd<T> f{H, st, batch, max_ctx, true, mode, kmax, batch, true};
  follow_stream(H, f, kmax, 0);  // the same weights as a kmax-loop step
  RET(input_block<T>(f, tokens_in));
  for (int t = 1; t <= kmax; ++t) {
    int rows = 0;
    while (rows < batch && ks[rows] >= t) ++rows;
    Fwd<T> g = f;
    g.M = rows;
    // an operand stage writes the updated state of its rows to the other
    // state buffer; rows that finished their loops would be left behind in
    // this one, so a pass over part of the batch updates in place
    g.stage = rows == batch;
    {
      // u_t = N(s_{t-1} + x), s_0 = x, s_{t-1} = N(h)
      Scope sc(H, st, "reinject", 0);
      CK(launch_reinject<T>(rows, d, H->hcur(), H->x, t == 1 ? 0 : 1, H->s, true, H->hop_t<T>(), nullptr, 1, 1, 0, st));
    }
    RET(run_layers<T>(g, c.n_in, c.n_in + c.n_rec, t));
  }
  {
    Scope sc(H, st, "reinject", 0);
    CK(launch_reinject<T>(batch, d, H->hcur(), H->x, 1, nullptr, false, H->hop_t<T>(), H->s, 1, 1, 0, st));
  }
  RET(output_and_head<T>(f, batch, nullptr, logits, next_tokens));
  CK(launch_advance(batch, H->seq_ids, H->seq_len, 1, st));
  for (int i = 0; i < batch; ++i) H->len[seq_ids[i]] += 1;
  H->last_rows = batch;
  return DORY_OK;
}

// One step of self-speculative decoding for B sequences: gamma draft passes
// at k = 1, the input block and loop 1 of d_gamma, the verify pass from loop
// 2 at k_verify, then acceptance on the device.  cond: the graph conditional
// the acceptance sets while another step is needed (0: none).
template <typename T>
dory_status spec_step(dory_handle* H, int B, int kv_, int gamma, int mode, int max_ctx, cudaStream_t st,
                      unsigned long long cond) {
  const dory_config& c = H->c;
  const int gc = c.gamma_max + 1;
  // drafts: y0, d1..d_{gamma-1} at k = 1, one token per sequence each
  for (int i = 0; i < gamma; ++i) {
    CK(launch_plan_uniform(B, 1, i, H->seq_ids, H->seq_len, H->meta, st));
    Fwd<T> f{H, st, B, max_ctx, true, mode, 1, B, true};
    follow_stream(H, f, 1, 0);  // a draft is a k = 1 step
    const int* tok = i == 0 ? H->pending : H->drafts + (i - 1) * B;
    RET(input_block<T>(f, tok));
    CK(launch_stash_copy(B, c.d_model, H->x, H->stash_x, 1, gc, i, 0, st));
    RET(loops<T>(f, 1, 1, i, 1));
    RET(output_and_head<T>(f, B, nullptr, nullptr, H->drafts + i * B));
  }
  // d_gamma: input block and loop 1 only
  {
    CK(launch_plan_uniform(B, 1, gamma, H->seq_ids, H->seq_len, H->meta, st));
    Fwd<T> f{H, st, B, max_ctx, true, mode, 1, B, true};
    follow_stream(H, f, 1, 0);  // the first two blocks of a k = 1 step
    RET(input_block<T>(f, H->drafts + (gamma - 1) * B));
    CK(launch_stash_copy(B, c.d_model, H->x, H->stash_x, 1, gc, gamma, 0, st));
    Scope sc(H, st, "reinject", 0);
    CK(launch_reinject<T>(B, c.d_model, H->hcur(), H->x, 0, nullptr, true, H->hop_t<T>(), nullptr, 1, 1, 0, st));
    RET(run_layers<T>(f, c.n_in, c.n_in + c.n_rec, 1));
    CK(launch_reinject<T>(B, c.d_model, H->hcur(), H->x, 1, nullptr, false, H->hop_t<T>(), H->stash_s, 1, gc,
                          gamma, st));
  }
  // verify [y0, d1..d_gamma] at k_verify from the stashed x and s_1
  const int rps = gamma + 1, M = B * rps;
  CK(launch_plan_uniform(B, rps, 0, H->seq_ids, H->seq_len, H->meta, st));
  Fwd<T> f{H, st, M, max_ctx, true, mode, kv_, B, true};
  follow_stream(H, f, kv_, 2 * (c.n_in + c.n_rec));  // a k_verify step from its loop 2 on
  CK(launch_stash_copy(M, c.d_model, H->x, H->stash_x, rps, gc, 0, 1, st));
  CK(launch_stash_copy(M, c.d_model, H->s, H->stash_s, rps, gc, 0, 1, st));
  RET(loops<T>(f, 2, kv_, -1, rps));
  RET(output_and_head<T>(f, M, nullptr, nullptr, H->vtok));
  CK(launch_spec_accept(B, gamma, B, H->seq_ids, H->seq_len, H->drafts, H->vtok, H->pending, H->spec_io,
                        H->accepted, H->spec_flags, H->err, cond, cond != 0, st));
  H->last_rows = M;
  return DORY_OK;
}

// The whole speculative loop as one CUDA graph: a conditional while node
// whose body is one recorded step; the acceptance kernel decides on the
// device whether the body runs again, so the host waits once, at the end.
template <typename T>
dory_status spec_graph(dory_handle* H, int B, int kv_, int gamma, int mode, cudaStream_t st, bool* built) {
  *built = false;
  const long long key = (1ll << 40) | ((long long)B << 16) | (gamma << 8) | (kv_ << 4) | mode;
  dory_handle::Graph* g = nullptr;
  for (auto& e : H->graphs_cache)
    if (e.key == key) g = &e;
  if (!g) {
    if (!H->cap_stream) CK(cudaStreamCreateWithFlags(&H->cap_stream, cudaStreamNonBlocking));
    cudaGraph_t graph = nullptr;
    CK(cudaGraphCreate(&graph, 0));
    cudaGraphConditionalHandle cond = 0;
    cudaError_t e = cudaGraphConditionalHandleCreate(&cond, graph, 1, cudaGraphCondAssignDefault);
    cudaGraphNodeParams np = {};
    np.type = cudaGraphNodeTypeConditional;
    np.conditional.handle = cond;
    np.conditional.type = cudaGraphCondTypeWhile;
    np.conditional.size = 1;
    cudaGraphNode_t node = nullptr;
    if (e == cudaSuccess) e = cudaGraphAddNode(&node, graph, nullptr, 0, &np);
    if (e != cudaSuccess) {
      cudaGraphDestroy(graph);
      return DORY_OK;  // no conditional nodes here: the caller runs the host loop
    }
    cudaGraph_t body = np.conditional.phGraph_out[0];
    const int hc0 = H->hc;
    dory_status r = DORY_OK;
    e = cudaStreamBeginCaptureToGraph(H->cap_stream, body, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal);
    if (e == cudaSuccess) {
      r = spec_step<T>(H, B, kv_, gamma, mode, H->c.max_seq, H->cap_stream, (unsigned long long)cond);
      cudaGraph_t out = nullptr;
      e = cudaStreamEndCapture(H->cap_stream, &out);
    }
    cudaGraphExec_t exec = nullptr;
    if (r == DORY_OK && e == cudaSuccess) e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    cudaGetLastError();  // a refused capture or instantiation leaves no sticky error
    if (r != DORY_OK) return r;
    if (e != cudaSuccess) {
      H->hc = hc0;
      return DORY_OK;  // the caller runs the host loop
    }
    H->graphs_cache.push_back({key, 1, exec, H->hc});
    g = &H->graphs_cache.back();
  }
  CK(cudaGraphLaunch(g->exec, st));
  H->hc = g->hc_end;
  *built = true;
  return DORY_OK;
}

template <typename T>
dory_status spec_t(dory_handle* H, int B, const int32_t* seq_ids, const int32_t* last_tokens, int kv_, int gamma,
                   int mode, int max_new, int32_t* out_tokens, int32_t* out_len, dory_spec_stats* stats,
                   cudaStream_t st) {
  const dory_config& c = H->c;
  int max_ctx = 0;
  for (int i = 0; i < B; ++i) max_ctx = std::max(max_ctx, H->len[seq_ids[i]] + max_new + 2 * gamma + 1);
  RET(upload_ids(H, seq_ids, B, st));
  RET(ensure_stream(H, 1, st));
  RET(ensure_stream(H, kv_, st));
  SpecIo io{out_tokens, out_len, max_new, 0};
  CK(cudaMemcpyAsync(H->spec_io, &io, sizeof io, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(H->pending, last_tokens, sizeof(int) * B, cudaMemcpyDeviceToDevice, st));
  CK(cudaMemsetAsync(out_len, 0, sizeof(int) * B, st));
  CK(cudaMemsetAsync(H->accepted, 0, sizeof(unsigned long long), st));
  CK(cudaMemsetAsync(H->spec_flags, 0, sizeof(int) * 4, st));
  bool on_device = false;
  if (H->graphs && !H->profile) RET(spec_graph<T>(H, B, kv_, gamma, mode, st, &on_device));
  if (!on_device) {
    // host loop: one step, then the host reads whether another is needed
    for (int64_t steps = 0;; ++steps) {
      RET(spec_step<T>(H, B, kv_, gamma, mode, max_ctx, st, 0));
      int flags[4] = {0, 0, 0, 0};
      CK(cudaMemcpyAsync(flags, H->spec_flags, sizeof flags, cudaMemcpyDeviceToHost, st));
      CK(cudaStreamSynchronize(st));
      if (flags[0] || flags[2]) break;
    }
  }
  // the one wait of the call: lengths, acceptance counts and step flags
  std::vector<int> lens(c.max_batch);
  int flags[4] = {0, 0, 0, 0}, err[4] = {0, 0, 0, 0};
  unsigned long long acc = 0;
  CK(cudaMemcpyAsync(lens.data(), H->seq_len, sizeof(int) * c.max_batch, cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(&acc, H->accepted, sizeof(acc), cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(flags, H->spec_flags, sizeof flags, cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(err, H->err, sizeof err, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  for (int i = 0; i < B; ++i) H->len[seq_ids[i]] = lens[seq_ids[i]];
  H->last_rows = B * (gamma + 1);
  if (stats) {
    stats->steps = flags[1];
    stats->drafted = (int64_t)flags[1] * gamma * B;
    stats->accepted = (int64_t)acc;
  }
  if (err[0] == DEV_ERR_TIMEOUT) return fail(DORY_ERR_TIMEOUT, "a device-side wait timed out during speculative decoding");
  if (flags[2] || !flags[0]) return fail(DORY_ERR_STATE, "speculative loop did not finish");
  return DORY_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* dory_last_error(const dory_handle*) { return g_last_error.c_str(); }

dory_status dory_workspace_size(const dory_config* cfg, dory_cache_mode alloc_mode, size_t* bytes) {
  RET(check_config(cfg));
  if (!bytes) return fail(DORY_ERR_INVALID_ARG, "bytes is NULL");
  if (alloc_mode != DORY_LAST_LOOP && alloc_mode != DORY_PER_LOOP) return fail(DORY_ERR_INVALID_ARG, "bad alloc mode");
  dory_handle tmp;
  tmp.c = *cfg;
  tmp.alloc_mode = alloc_mode;
  *bytes = layout(&tmp);
  return DORY_OK;
}

dory_status dory_create(const dory_config* cfg, const dory_weights* w, dory_cache_mode alloc_mode, void* workspace,
                        size_t ws_bytes, dory_handle** out) {
  RET(check_config(cfg));
  if (!w || !out || !workspace) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if ((uintptr_t)workspace % 256) return fail(DORY_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  size_t need = 0;
  RET(dory_workspace_size(cfg, alloc_mode, &need));
  if (ws_bytes < need) return fail(DORY_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
  const int L = cfg->n_in + cfg->n_rec + cfg->n_out;
  if (!w->embed || !w->lm_head || !w->w_qkv || !w->w_o || !w->w_gu || !w->w_down)
    return fail(DORY_ERR_INVALID_ARG, "NULL weight pointer");
  for (int l = 0; l < L; ++l) {
    bool ok = layer_is_attn(l) ? (w->w_qkv[l] && w->w_o[l]) : (w->w_gu[l] && w->w_down[l]);
    if (!ok) return fail(DORY_ERR_INVALID_ARG, "layer %d: NULL weight", l);
  }
  dory_handle* H = new dory_handle();
  H->c = *cfg;
  H->alloc_mode = alloc_mode;
  H->ws = (char*)workspace;
  H->ws_bytes = ws_bytes;
  layout(H);
  H->embed = w->embed;
  H->head = w->lm_head;
  H->w_qkv.assign(w->w_qkv, w->w_qkv + L);
  H->w_o.assign(w->w_o, w->w_o + L);
  H->w_gu.assign(w->w_gu, w->w_gu + L);
  H->w_down.assign(w->w_down, w->w_down + L);
  H->len.assign(cfg->max_batch, 0);
  H->mode.assign(cfg->max_batch, -1);
  H->kfix.assign(cfg->max_batch, 0);
  if (H->page_table) {
    H->pt_host.assign((size_t)cfg->max_batch * H->pt_stride, 0);
    H->seq_pages.assign(cfg->max_batch, {});
    H->free_pages.clear();
    for (int p = H->pool_pages - 1; p >= 0; --p) H->free_pages.push_back(p);
  }
  *out = H;
  return DORY_OK;
}

dory_status dory_destroy(dory_handle* h) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  for (auto e : h->ev_pool) cudaEventDestroy(e);
  for (auto& g : h->graphs_cache)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  delete h;
  return DORY_OK;
}

dory_status dory_reset(dory_handle* h, int32_t seq, dory_stream stream) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  cudaStream_t st = (cudaStream_t)stream;
  if (seq == -1) {
    CK(cudaMemsetAsync(h->seq_len, 0, sizeof(int) * h->c.max_batch, st));
    CK(cudaMemsetAsync(h->err, 0, sizeof(int) * 4, st));
    CK(cudaMemsetAsync(h->attn_counters, 0, sizeof(unsigned) * (size_t)h->M_max * h->c.n_kv_heads, st));
    std::fill(h->len.begin(), h->len.end(), 0);
    std::fill(h->mode.begin(), h->mode.end(), -1);
    for (int q = 0; q < h->c.max_batch; ++q) release_pages(h, q);
    return DORY_OK;
  }
  if (seq < 0 || seq >= h->c.max_batch) return fail(DORY_ERR_INVALID_ARG, "seq %d out of range", seq);
  CK(cudaMemsetAsync(h->seq_len + seq, 0, sizeof(int), st));
  h->len[seq] = 0;
  h->mode[seq] = -1;
  release_pages(h, seq);
  return DORY_OK;
}

dory_status dory_prefill(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* tokens,
                         const int32_t* lens, int32_t k, dory_cache_mode mode, float* last_logits,
                         int32_t* next_tokens, dory_stream stream) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  RET(check_seqs(h, batch, seq_ids, k, mode));
  if (!tokens || !lens || !next_tokens) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  int64_t total = 0;
  for (int i = 0; i < batch; ++i) {
    if (lens[i] < 1) return fail(DORY_ERR_INVALID_ARG, "lens[%d] = %d < 1", i, lens[i]);
    total += lens[i];
    if ((int64_t)h->len[seq_ids[i]] + lens[i] > h->c.max_seq)
      return fail(DORY_ERR_CAPACITY, "sequence %d would exceed max_seq", seq_ids[i]);
  }
  if (total > h->c.max_chunk) return fail(DORY_ERR_CAPACITY, "%lld tokens > max_chunk %d", (long long)total, h->c.max_chunk);
  {
    std::vector<int64_t> upto(batch);
    for (int i = 0; i < batch; ++i) upto[i] = (int64_t)h->len[seq_ids[i]] + lens[i];
    RET(ensure_pages(h, batch, seq_ids, upto.data(), (cudaStream_t)stream));
  }
  dory_status r = h->bf16 ? prefill_t<bf16>(h, batch, seq_ids, tokens, lens, k, mode, last_logits, next_tokens,
                                             (cudaStream_t)stream)
                          : prefill_t<float>(h, batch, seq_ids, tokens, lens, k, mode, last_logits, next_tokens,
                                             (cudaStream_t)stream);
  if (r == DORY_OK) mark_started(h, batch, seq_ids, k, mode);
  return r;
}

dory_status dory_decode_step(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* tokens_in,
                             int32_t k, dory_cache_mode mode, float* logits, int32_t* next_tokens,
                             dory_stream stream) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  RET(check_seqs(h, batch, seq_ids, k, mode));
  if (!tokens_in || !next_tokens) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  for (int i = 0; i < batch; ++i)
    if (h->len[seq_ids[i]] + 1 > h->c.max_seq)
      return fail(DORY_ERR_CAPACITY, "sequence %d would exceed max_seq", seq_ids[i]);
  {
    std::vector<int64_t> upto(batch);
    for (int i = 0; i < batch; ++i) upto[i] = (int64_t)h->len[seq_ids[i]] + 1;
    RET(ensure_pages(h, batch, seq_ids, upto.data(), (cudaStream_t)stream));
  }
  dory_status r = h->bf16 ? decode_t<bf16>(h, batch, seq_ids, tokens_in, k, mode, logits, next_tokens,
                                            (cudaStream_t)stream)
                          : decode_t<float>(h, batch, seq_ids, tokens_in, k, mode, logits, next_tokens,
                                            (cudaStream_t)stream);
  if (r == DORY_OK) mark_started(h, batch, seq_ids, k, mode);
  return r;
}

dory_status dory_decode_step_mixed(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* tokens_in,
                                   const int32_t* ks, dory_cache_mode mode, float* logits, int32_t* next_tokens,
                                   dory_stream stream) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  if (!seq_ids || !ks || !tokens_in || !next_tokens) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (batch <= 0 || batch > h->c.max_batch)
    return fail(DORY_ERR_INVALID_ARG, "batch %d outside 1..%d", batch, h->c.max_batch);
  for (int i = 0; i < batch; ++i) {
    RET(check_seqs(h, 1, seq_ids + i, ks[i], mode));  // range, mode and per-loop k of each sequence
    if (i > 0 && ks[i] > ks[i - 1]) return fail(DORY_ERR_INVALID_ARG, "k must not increase along the batch");
    for (int j = 0; j < i; ++j)
      if (seq_ids[j] == seq_ids[i]) return fail(DORY_ERR_INVALID_ARG, "seq id %d repeated", seq_ids[i]);
    if (h->len[seq_ids[i]] + 1 > h->c.max_seq)
      return fail(DORY_ERR_CAPACITY, "sequence %d would exceed max_seq", seq_ids[i]);
  }
  const cudaStream_t st = (cudaStream_t)stream;
  {
    std::vector<int64_t> upto(batch);
    for (int i = 0; i < batch; ++i) upto[i] = (int64_t)h->len[seq_ids[i]] + 1;
    RET(ensure_pages(h, batch, seq_ids, upto.data(), st));
  }
  dory_status r = h->bf16 ? decode_mixed_t<bf16>(h, batch, seq_ids, tokens_in, ks, mode, logits, next_tokens, st)
                          : decode_mixed_t<float>(h, batch, seq_ids, tokens_in, ks, mode, logits, next_tokens, st);
  if (r == DORY_OK)
    for (int i = 0; i < batch; ++i) mark_started(h, 1, seq_ids + i, ks[i], mode);
  return r;
}

dory_status dory_spec_decode(dory_handle* h, int32_t batch, const int32_t* seq_ids, const int32_t* last_tokens,
                             int32_t k_draft, int32_t k_verify, int32_t gamma, dory_cache_mode mode, int32_t max_new,
                             int32_t* out_tokens, int32_t* out_len, dory_spec_stats* stats, dory_stream stream) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  RET(check_seqs(h, batch, seq_ids, k_verify, mode));
  if (k_draft != 1) return fail(DORY_ERR_UNSUPPORTED, "k_draft must be 1 (loop-1 reuse)");
  if (h->temperature > 0.f) return fail(DORY_ERR_UNSUPPORTED, "speculative decoding is greedy only");
  if (gamma < 1 || gamma > h->c.gamma_max) return fail(DORY_ERR_INVALID_ARG, "gamma %d outside 1..%d", gamma, h->c.gamma_max);
  if (max_new < 1) return fail(DORY_ERR_INVALID_ARG, "max_new must be >= 1");
  if (!last_tokens || !out_tokens || !out_len) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (batch * (gamma + 1) > h->M_max) return fail(DORY_ERR_CAPACITY, "batch*(gamma+1) exceeds chunk capacity");
  for (int i = 0; i < batch; ++i) {
    int sq = seq_ids[i];
    if (h->mode[sq] < 0) return fail(DORY_ERR_STATE, "sequence %d has no prefill", sq);
    // a sequence that finishes first stays frozen at <= len + max_new + gamma
    // committed positions while the others continue, and each later step
    // still writes gamma positions past its length
    if ((int64_t)h->len[sq] + max_new + 2 * gamma + 1 > h->c.max_seq)
      return fail(DORY_ERR_CAPACITY, "sequence %d: len + max_new + 2*gamma + 1 exceeds max_seq", sq);
  }
  {
    std::vector<int64_t> upto(batch);
    for (int i = 0; i < batch; ++i) upto[i] = (int64_t)h->len[seq_ids[i]] + max_new + 2 * gamma + 1;
    RET(ensure_pages(h, batch, seq_ids, upto.data(), (cudaStream_t)stream));
  }
  return h->bf16 ? spec_t<bf16>(h, batch, seq_ids, last_tokens, k_verify, gamma, mode, max_new, out_tokens, out_len,
                                stats, (cudaStream_t)stream)
                 : spec_t<float>(h, batch, seq_ids, last_tokens, k_verify, gamma, mode, max_new, out_tokens, out_len,
                                 stats, (cudaStream_t)stream);
}

dory_status dory_kv_bytes(const dory_handle* h, int32_t k, dory_cache_mode mode, int64_t ctx, int64_t* bytes) {
  if (!h || !bytes) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (k < 1 || ctx < 0) return fail(DORY_ERR_INVALID_ARG, "bad k or ctx");
  int64_t total = 0;
  for (const AttnLayer& a : h->attn) {
    int64_t keep = a.full ? ctx : std::min<int64_t>(ctx, h->c.swa_window);
    int slots = (mode == DORY_PER_LOOP && a.rec) ? k : 1;
    total += keep * 2 * h->kv_dim * h->esz * slots;
  }
  *bytes = total;
  return DORY_OK;
}

dory_status dory_seq_len(const dory_handle* h, int32_t seq, int32_t* len) {
  if (!h || !len) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (seq < 0 || seq >= h->c.max_batch) return fail(DORY_ERR_INVALID_ARG, "seq out of range");
  *len = h->len[seq];
  return DORY_OK;
}

dory_status dory_read_state(dory_handle* h, int32_t which, float* dst, int32_t rows, dory_stream stream) {
  if (!h || !dst) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (rows < 1 || rows > h->last_rows) return fail(DORY_ERR_INVALID_ARG, "rows %d outside 1..%d", rows, h->last_rows);
  const float* src = which == 0 ? h->x : which == 1 ? h->s : which == 2 ? h->hcur() : nullptr;
  if (!src) return fail(DORY_ERR_INVALID_ARG, "bad state selector");
  CK(cudaMemcpyAsync(dst, src, sizeof(float) * rows * h->c.d_model, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return DORY_OK;
}

dory_status dory_read_kv(dory_handle* h, int32_t layer, int32_t slot, int32_t seq, int32_t pos0, int32_t n,
                         void* k_dst, void* v_dst, dory_stream stream) {
  if (!h || !k_dst || !v_dst) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (layer < 0 || layer >= h->L || h->attn_of[layer] < 0) return fail(DORY_ERR_INVALID_ARG, "not an attention layer");
  const AttnLayer& a = h->attn[h->attn_of[layer]];
  if (slot < 0 || slot >= a.nslots) return fail(DORY_ERR_INVALID_ARG, "slot out of range");
  if (seq < 0 || seq >= h->c.max_batch || pos0 < 0 || n < 1 || pos0 + n > h->len[seq])
    return fail(DORY_ERR_INVALID_ARG, "positions outside the sequence");
  if (!a.full && pos0 < h->len[seq] - a.cap) return fail(DORY_ERR_INVALID_ARG, "positions no longer in the ring");
  const int hd = h->c.head_dim, KV = h->c.n_kv_heads;
  const size_t row = (size_t)hd * h->esz;
  cudaStream_t st = (cudaStream_t)stream;
  for (int i = 0; i < n; ++i) {
    int p = pos0 + i;
    for (int g = 0; g < KV; ++g) {
      size_t src = (((size_t)seq * KV + g) * a.cap + (p % a.cap)) * row;
      if (a.full && h->page_table) {
        const int P = h->c.kv_page;
        src = (((size_t)h->pt_host[(size_t)seq * h->pt_stride + p / P] * KV + g) * P + p % P) * row;
      }
      size_t dst = ((size_t)i * KV + g) * row;
      CK(cudaMemcpyAsync((char*)k_dst + dst, a.K[slot] + src, row, cudaMemcpyDeviceToDevice, st));
      CK(cudaMemcpyAsync((char*)v_dst + dst, a.V[slot] + src, row, cudaMemcpyDeviceToDevice, st));
    }
  }
  return DORY_OK;
}

dory_status dory_gemm_bf16(int32_t M, int32_t N, int32_t K, const void* X, const void* W, float* Y,
                           int32_t batch_hint, int32_t invariant, int32_t impl, int32_t* splits, int32_t* err_word,
                           dory_stream stream) {
  if (M < 1 || N < 1 || K < 1 || !X || !W || !Y || !splits) return fail(DORY_ERR_INVALID_ARG, "bad GEMM arguments");
  cudaStream_t st = (cudaStream_t)stream;
  *splits = 1;
  if (impl != 1) {
    int S = 1;
    size_t ps = 0;
    cudaError_t e = launch_gemm_tc(M, N, K, (const bf16*)X, K, (const bf16*)W, Y, N, (size_t)M, err_word,
                                   batch_hint < 1 ? 1 : batch_hint, invariant != 0, &S, &ps, st, impl == 3 ? 1 : 0,
                                   impl == 4);
    if (e == cudaSuccess) {
      *splits = S;
      return DORY_OK;
    }
    if (e != cudaErrorNotSupported || impl >= 2) return fail(DORY_ERR_CUDA, "tcgen05 GEMM: %s", cudaGetErrorString(e));
  }
  CK(launch_gemm_simt<bf16>(M, N, K, (const bf16*)X, K, (const bf16*)W, Y, N, st));
  return DORY_OK;
}

dory_status dory_pack_weight_bf16(const void* src, void* dst, int32_t N, int32_t K, dory_stream stream) {
  if (!src || !dst || N < 1 || K < 1) return fail(DORY_ERR_INVALID_ARG, "bad pack arguments");
  if (N % 128 || K % 64) return fail(DORY_ERR_UNSUPPORTED, "packing needs N %% 128 == 0 and K %% 64 == 0");
  if (((uintptr_t)src & 15) || ((uintptr_t)dst & 15)) return fail(DORY_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  CK(launch_pack_weight((const bf16*)src, dst, N, K, (cudaStream_t)stream));
  return DORY_OK;
}

dory_status dory_synchronize(dory_handle* h, dory_stream stream) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  int err[4] = {0, 0, 0, 0};
  CK(cudaMemcpyAsync(err, h->err, sizeof err, cudaMemcpyDeviceToHost, (cudaStream_t)stream));
  CK(cudaStreamSynchronize((cudaStream_t)stream));
  if (err[0] != DEV_ERR_NONE) {
    CK(cudaMemsetAsync(h->err, 0, sizeof(int) * 4, (cudaStream_t)stream));
    if (err[0] == DEV_ERR_TIMEOUT) return fail(DORY_ERR_TIMEOUT, "a device-side wait timed out");
    if (err[0] == DEV_ERR_BAD_TOKEN) return fail(DORY_ERR_INVALID_ARG, "a token id was outside [0, vocab)");
    if (err[0] == DEV_ERR_BAD_INDEX) return fail(DORY_ERR_CAPACITY, "a cache position was outside max_seq");
    if (err[0] == DEV_ERR_RANGE) return fail(DORY_ERR_INVALID_ARG, "a value was outside a kernel's supported range");
    return fail(DORY_ERR_CUDA, "device error code %d", err[0]);
  }
  return DORY_OK;
}

dory_status dory_set_option(dory_handle* h, int32_t opt, int64_t value) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  switch (opt) {
    case DORY_OPT_CUDA_GRAPHS: h->graphs = value != 0; return DORY_OK;
    case DORY_OPT_PROFILE: h->profile = value != 0; return DORY_OK;
    case DORY_OPT_PDL: dory::g_pdl = value != 0; return DORY_OK;
    case DORY_OPT_PREFILL_TC:
      if (value < 0 || value > 3) return fail(DORY_ERR_INVALID_ARG, "bad prefill attention kernel");
      h->prefill_tc = (int)value;
      return DORY_OK;
    case DORY_OPT_ATTN_CLUSTER:
      if (value != 0 && value != 1 && value != 4 && value != 8 && value != 16)
        return fail(DORY_ERR_INVALID_ARG, "attention cluster option must be 0, 1, 4, 8 or 16");
      if (value != dory::g_attn_cluster) {
        for (auto& g : h->graphs_cache)
          if (g.exec) cudaGraphExecDestroy(g.exec);
        h->graphs_cache.clear();
      }
      dory::g_attn_cluster = (int)value;
      return DORY_OK;
    case DORY_OPT_L2_LOOKAHEAD:
      if (value < 0 || value > (1ll << 40)) return fail(DORY_ERR_INVALID_ARG, "bad look-ahead");
      if ((unsigned long long)value != h->pf_lead) {
        // graphs captured with the old setting are dropped
        for (auto& g : h->graphs_cache)
          if (g.exec) cudaGraphExecDestroy(g.exec);
        h->graphs_cache.clear();
      }
      h->pf_lead = (unsigned long long)value & ~127ull;
      return DORY_OK;
    case DORY_OPT_MX_GEMV:
      if (value < 0 || value > 4) return fail(DORY_ERR_INVALID_ARG, "bad MXFP8 GEMV impl");
      if (value != h->mx_impl) {
        for (auto& g : h->graphs_cache)
          if (g.exec) cudaGraphExecDestroy(g.exec);
        h->graphs_cache.clear();
      }
      h->mx_impl = (int)value;
      return DORY_OK;
    case DORY_OPT_GEMM_IMPL:
      if (value < 0 || value > 2) return fail(DORY_ERR_INVALID_ARG, "bad GEMM impl");
      h->gemm_impl = (int)value;
      return DORY_OK;
    case DORY_OPT_L2_OWN:
      if (value < 0 || value > (1 << 20)) return fail(DORY_ERR_INVALID_ARG, "bad own-tile prefetch count");
      if (value != h->pf_own) {
        for (auto& g : h->graphs_cache)
          if (g.exec) cudaGraphExecDestroy(g.exec);
        h->graphs_cache.clear();
      }
      h->pf_own = (int)value;
      return DORY_OK;
    case DORY_OPT_ATTN_LOOKAHEAD:
      if (value < 0 || value > (1ll << 40)) return fail(DORY_ERR_INVALID_ARG, "bad look-ahead");
      if ((unsigned long long)value != h->pf_attn) {
        for (auto& g : h->graphs_cache)
          if (g.exec) cudaGraphExecDestroy(g.exec);
        h->graphs_cache.clear();
      }
      h->pf_attn = (unsigned long long)value & ~127ull;
      return DORY_OK;
    case DORY_OPT_FUSED_OPERANDS:
      if (value < 0 || value > 16) return fail(DORY_ERR_INVALID_ARG, "fused operand rows must be in 0..16");
      if (value != h->fuse_rows) {
        for (auto& g : h->graphs_cache)
          if (g.exec) cudaGraphExecDestroy(g.exec);
        h->graphs_cache.clear();
      }
      h->fuse_rows = (int)value;
      return DORY_OK;
  }
  return fail(DORY_ERR_INVALID_ARG, "unknown option %d", opt);
}

dory_status dory_quantize_mxfp8(const void* w, int32_t n, int32_t k, void* q, void* scales, void* w_deq,
                                int32_t* err_word, dory_stream stream) {
  if (!w || !q || !scales || n < 1 || k < 1) return fail(DORY_ERR_INVALID_ARG, "bad quantiser arguments");
  if (k % kMxBlock) return fail(DORY_ERR_UNSUPPORTED, "K must be a multiple of %d", kMxBlock);
  if (((uintptr_t)w & 15) || ((uintptr_t)q & 15) || ((uintptr_t)w_deq & 15))
    return fail(DORY_ERR_INVALID_ARG, "w, q and w_deq must be 16-byte aligned");
  CK(launch_mx_quantize((const bf16*)w, n, k, (uint8_t*)q, (uint8_t*)scales, (bf16*)w_deq, err_word,
                        (cudaStream_t)stream));
  return DORY_OK;
}

dory_status dory_gemv_mxfp8(int32_t m, int32_t n, int32_t k, const void* x, int32_t ldx, const void* q,
                            const void* scales, float* y, int32_t ldy, int32_t impl, int32_t* err_word,
                            dory_stream stream) {
  if (!x || !q || !scales || !y || m < 1 || n < 1 || k < 1 || ldx < k || ldy < n || impl < 0 || impl > 4)
    return fail(DORY_ERR_INVALID_ARG, "bad GEMV arguments");
  if (impl == 3 && (n % 128 || k % 128 || ((uintptr_t)x & 15) || ldx % 8))
    return fail(DORY_ERR_UNSUPPORTED, "impl 3 needs N %% 128 == 0, K %% 128 == 0, x 16-byte aligned, ldx %% 8 == 0");
  if (k % kMxBlock || k > (impl == 2 ? 10240 : 40960))
    return fail(DORY_ERR_UNSUPPORTED, "K must be a multiple of 32 and at most %d", impl == 2 ? 10240 : 40960);
  if ((uintptr_t)q & 15) return fail(DORY_ERR_INVALID_ARG, "q must be 16-byte aligned");
  CK(launch_mx_gemv(m, n, k, (const bf16*)x, ldx, (const uint8_t*)q, (const uint8_t*)scales, y, ldy, err_word,
                    (cudaStream_t)stream, impl));
  return DORY_OK;
}

dory_status dory_attach_mxfp8(dory_handle* h, const dory_mx_weights* mx) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  std::unordered_map<const void*, dory_handle::MxMat> map;
  if (mx) {
    const dory_config& c = h->c;
    if (!h->bf16) return fail(DORY_ERR_UNSUPPORTED, "MXFP8 copies stand for bf16 weights only");
    if (c.d_model % kMxBlock || h->q_dim % kMxBlock || c.d_ff % kMxBlock)
      return fail(DORY_ERR_UNSUPPORTED, "d_model, n_heads * head_dim and d_ff must be multiples of %d", kMxBlock);
    bool ok = true;
    auto add = [&](const void* w, const void* const* qs, const void* const* ss, int l) {
      const void* q = qs ? qs[l] : nullptr;
      const void* sc = ss ? ss[l] : nullptr;
      if (!q && !sc) return;  // this matrix stays bf16
      if (!q || !sc || ((uintptr_t)q & 15)) ok = false;
      map[w] = {(const uint8_t*)q, (const uint8_t*)sc};
    };
    for (int l = 0; l < h->L; ++l) {
      if (layer_is_attn(l)) {
        add(h->w_qkv[l], mx->qkv_q, mx->qkv_s, l);
        add(h->w_o[l], mx->o_q, mx->o_s, l);
      } else {
        add(h->w_gu[l], mx->gu_q, mx->gu_s, l);
        add(h->w_down[l], mx->down_q, mx->down_s, l);
      }
    }
    const void* hq[1] = {mx->lm_head_q};
    const void* hs[1] = {mx->lm_head_s};
    add(h->head, hq, hs, 0);
    if (!ok) return fail(DORY_ERR_INVALID_ARG, "each MXFP8 copy needs codes (16-byte aligned) and scales");
  }
  // graphs captured with the other weights are dropped
  for (auto& g : h->graphs_cache)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  h->graphs_cache.clear();
  h->mx.swap(map);
  return DORY_OK;
}

dory_status dory_quantize_nvfp4(const void* w, int32_t n, int32_t k, void* q, void* scales, float* g, void* w_deq,
                                int32_t* err_word, dory_stream stream) {
  if (!w || !q || !scales || !g || n < 1 || k < 1) return fail(DORY_ERR_INVALID_ARG, "bad quantiser arguments");
  if (k % 16) return fail(DORY_ERR_UNSUPPORTED, "K must be a multiple of 16");
  if (((uintptr_t)w & 15) || ((uintptr_t)q & 7) || ((uintptr_t)w_deq & 15) || ((uintptr_t)g & 3))
    return fail(DORY_ERR_INVALID_ARG, "w and w_deq must be 16-byte, q 8-byte and g 4-byte aligned");
  CK(launch_nv_quantize((const bf16*)w, n, k, (uint8_t*)q, (uint8_t*)scales, g, (bf16*)w_deq, err_word,
                        (cudaStream_t)stream));
  return DORY_OK;
}

dory_status dory_gemm_nvfp4(int32_t m, int32_t n, int32_t k, const void* x, int32_t ldx, const void* q,
                            const void* scales, const float* g, float* y, int32_t ldy, int32_t* err_word,
                            dory_stream stream) {
  if (!x || !q || !scales || !g || !y || m < 1 || n < 1 || k < 1 || ldx < k || ldy < n)
    return fail(DORY_ERR_INVALID_ARG, "bad GEMM arguments");
  if (n % 128 || k % 256 || ((uintptr_t)x & 15) || ldx % 8 || ((uintptr_t)q & 15) || ((uintptr_t)scales & 15))
    return fail(DORY_ERR_UNSUPPORTED, "NVFP4 GEMM needs N %% 128 == 0, K %% 256 == 0, x, q and scales 16-byte "
                                      "aligned, ldx %% 8 == 0");
  CK(launch_nv_gemm_tc(m, n, k, (const bf16*)x, ldx, (const uint8_t*)q, (const uint8_t*)scales, g, y, ldy, 0, 1,
                       err_word, (cudaStream_t)stream));
  return DORY_OK;
}

dory_status dory_attach_nvfp4(dory_handle* h, const dory_nvfp4_weights* nv) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  std::unordered_map<const void*, dory_handle::MxMat> map;
  if (nv) {
    const dory_config& c = h->c;
    if (!h->bf16) return fail(DORY_ERR_UNSUPPORTED, "NVFP4 copies stand for bf16 weights only");
    if (c.d_model % 256 || h->q_dim % 256 || c.d_ff % 256)
      return fail(DORY_ERR_UNSUPPORTED, "d_model, n_heads * head_dim and d_ff must be multiples of 256");
    bool ok = true;
    auto add = [&](const void* w, const void* const* qs, const void* const* ss, const float* const* gs, int l) {
      const void* q = qs ? qs[l] : nullptr;
      const void* sc = ss ? ss[l] : nullptr;
      const float* g = gs ? gs[l] : nullptr;
      if (!q && !sc && !g) return;  // this matrix stays bf16
      if (!q || !sc || !g || ((uintptr_t)q & 15) || ((uintptr_t)sc & 15)) ok = false;
      dory_handle::MxMat m;
      m.q = (const uint8_t*)q;
      m.s = (const uint8_t*)sc;
      m.g = g;
      m.fmt = 1;
      map[w] = m;
    };
    for (int l = 0; l < h->L; ++l) {
      if (layer_is_attn(l)) {
        add(h->w_qkv[l], nv->qkv_q, nv->qkv_s, nv->qkv_g, l);
        add(h->w_o[l], nv->o_q, nv->o_s, nv->o_g, l);
      } else {
        add(h->w_gu[l], nv->gu_q, nv->gu_s, nv->gu_g, l);
        add(h->w_down[l], nv->down_q, nv->down_s, nv->down_g, l);
      }
    }
    const void* hq[1] = {nv->lm_head_q};
    const void* hs[1] = {nv->lm_head_s};
    const float* hg[1] = {nv->lm_head_g};
    add(h->head, hq, hs, hg, 0);
    if (!ok) return fail(DORY_ERR_INVALID_ARG, "each NVFP4 copy needs codes and scales (16-byte aligned) and g");
  }
  for (auto& g : h->graphs_cache)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  h->graphs_cache.clear();
  h->mx.swap(map);
  return DORY_OK;
}

dory_status dory_set_sampling(dory_handle* h, float temperature, float top_p, uint64_t seed) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  if (!(temperature >= 0.f) || !(top_p > 0.f) || top_p > 1.f)
    return fail(DORY_ERR_INVALID_ARG, "temperature must be >= 0 and top_p in (0, 1]");
  if (temperature != h->temperature || top_p != h->top_p || seed != h->seed) {
    // graphs captured with the old choice rule are dropped
    for (auto& g : h->graphs_cache)
      if (g.exec) cudaGraphExecDestroy(g.exec);
    h->graphs_cache.clear();
  }
  h->temperature = temperature;
  h->top_p = top_p;
  h->seed = seed;
  return DORY_OK;
}

dory_status dory_sample(const float* logits, int32_t rows, int32_t vocab, const int32_t* seq, const int32_t* pos,
                        float temperature, float top_p, uint64_t seed, uint32_t* scratch, int32_t* out,
                        dory_stream stream) {
  if (!logits || !seq || !pos || !scratch || !out) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  if (rows <= 0 || vocab <= 0) return fail(DORY_ERR_INVALID_ARG, "rows and vocab must be positive");
  if (!(temperature > 0.f) || !(top_p > 0.f) || top_p > 1.f)
    return fail(DORY_ERR_INVALID_ARG, "temperature must be > 0 and top_p in (0, 1]");
  CK(launch_sample(rows, vocab, logits, scratch, nullptr, seq, pos, 0, temperature, top_p, seed, out,
                   (cudaStream_t)stream));
  return DORY_OK;
}

dory_status dory_profile_reset(dory_handle* h) {
  if (!h) return fail(DORY_ERR_INVALID_ARG, "NULL handle");
  h->prof_recs.clear();
  h->ev_used = 0;
  return DORY_OK;
}

dory_status dory_profile_read(dory_handle* h, int32_t n, char (*names)[48], int64_t* launches, double* total_ms,
                              double* bytes, int32_t* count) {
  if (!h || !count) return fail(DORY_ERR_INVALID_ARG, "NULL argument");
  CK(cudaDeviceSynchronize());
  const size_t K = h->prof_names.size();
  std::vector<int64_t> cnt(K, 0);
  std::vector<double> ms(K, 0.0), by(K, 0.0);
  for (auto& r : h->prof_recs) {
    float t = 0.f;
    CK(cudaEventElapsedTime(&t, r.a, r.b));
    cnt[r.name] += 1;
    ms[r.name] += t;
    by[r.name] += r.bytes;
  }
  *count = (int32_t)K;
  for (int i = 0; i < (int)K && i < n; ++i) {
    if (names) {
      strncpy(names[i], h->prof_names[i].c_str(), 47);
      names[i][47] = 0;
    }
    if (launches) launches[i] = cnt[i];
    if (total_ms) total_ms[i] = ms[i];
    if (bytes) bytes[i] = by[i];
  }
  return DORY_OK;
}

}  // extern "C"

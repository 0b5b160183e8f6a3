// Prefill attention on the tensor cores (bf16).
#pragma once

#include "kernels.cuh"

namespace dory {

// Host: split each sequence's chunk rows [cu[b], cu[b+1]) into tiles of
// `rows` rows (int2 {first, end}); returns the count, or -1 past `cap`.
int prefill_tiles(int n_seq, const int* cu, int2* tiles, int cap, int rows = 64);
bool attn_prefill_supported(int head_dim);
// The tcgen05 kernel (S and O accumulators in TMEM): head_dim 128, tiles of
// 128 rows.
bool attn_prefill_tc_supported(int head_dim);

// qh: [M, H*hd] bf16 queries pre-scaled by log2(e)/sqrt(hd); kscr/vscr: the
// chunk's K/V [M, KV*hd]; keys before each sequence's chunk come from kv.
// out: [M, H*hd] bf16.
// launch_attn_prefill: warp-level mma.sync, 64-row tiles; launch_attn_prefill_tc:
// tcgen05 with TMEM accumulators, 128-row tiles.
cudaError_t launch_attn_prefill(int n_tiles, const int2* tiles, int H, int KV, int hd, const bf16* qh,
                                const bf16* kscr, const bf16* vscr, KVView kv, RowMeta m, bf16* out,
                                cudaStream_t st);
cudaError_t launch_attn_prefill_tc(int n_tiles, const int2* tiles, int H, int KV, int hd, const bf16* qh,
                                   const bf16* kscr, const bf16* vscr, KVView kv, RowMeta m, bf16* out,
                                   cudaStream_t st);

// The warp-specialised tcgen05 kernel (head_dim 128, 128-row tiles): each
// CTA runs one work item, two query slots that share a key/value stream over
// a range of key tiles.  a = {tile, head, tile, head} (second tile -1: one
// slot); b = {first key tile, end key tile, merge unit, pieces | piece << 8}:
// an item cut into `pieces` key ranges has one CTA per range; they merge
// through the partial buffer, units unit .. unit + pieces - 1 (unit -1: not
// cut, range [0, INT_MAX)).
struct PfItem {
  int4 a, b;
};
// Partial rows of a cut item: fp32 O (128) then the running max and sum.
constexpr int kPfPartStride = 132;
constexpr int kPfMaxPieces = 4;
// Host: work items for one layer kind (window 0: full causal).  Heads of a
// KV group pair on the same tile (an odd head left over pairs consecutive
// tiles of one sequence); items longer than the per-SM share of all key
// tiles are cut into up to kPfMaxPieces key ranges while merge units
// (one per piece) last; items come largest first.  tile_first_pos,
// tile_last_pos, tile_seq: each tile's first and last position and sequence.
// Returns the count (and the merge units used in *units), or -1 past `cap`.
int prefill_ws_items(int n_tiles, const int* tile_first_pos, const int* tile_last_pos, const int* tile_seq, int H,
                     int KV, int window, int n_sm, int max_units, PfItem* items, int cap, int* units);
// kv_rows: rows of head_dim elements in each of kv.K, kv.V.  counters
// (2 x max_units ints, zero) and part (max_units x 2 x 128 x kPfPartStride
// floats) serve the cut items; a launch that completes leaves counters at zero.
cudaError_t launch_attn_prefill_ws(int n_items, const PfItem* items, const int2* tiles, int M, int H, int KV, int hd,
                                   const bf16* qh, const bf16* kscr, const bf16* vscr, KVView kv, size_t kv_rows,
                                   RowMeta m, int* counters, int max_units, float* part, bf16* out,
                                   cudaStream_t st);

}  // namespace dory

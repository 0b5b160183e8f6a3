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
// CTA runs one work item of two query slots that share a key/value stream.
// prefill_ws_items (host) pairs the heads of each KV group on the same tile
// (an odd head left over pairs consecutive tiles of one sequence) and orders
// the items by their number of key tiles, largest first; tile_last_pos[t] and
// tile_seq[t] are tile t's last position and sequence.  Returns the count, or
// -1 past `cap`.  kv_rows: rows of head_dim elements in each of kv.K, kv.V.
int prefill_ws_items(int n_tiles, const int* tile_last_pos, const int* tile_seq, int H, int KV, int4* items,
                     int cap);
cudaError_t launch_attn_prefill_ws(int n_items, const int4* items, const int2* tiles, int M, int H, int KV, int hd,
                                   const bf16* qh, const bf16* kscr, const bf16* vscr, KVView kv, size_t kv_rows,
                                   RowMeta m, bf16* out, cudaStream_t st);

}  // namespace dory

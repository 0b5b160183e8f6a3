// Prefill attention on the tensor cores (bf16).
#pragma once

#include "kernels.cuh"

namespace dory {

// Host: split each sequence's chunk rows [cu[b], cu[b+1]) into tiles of 64
// rows (int2 {first, end}); returns the count, or -1 past `cap`.
int prefill_tiles(int n_seq, const int* cu, int2* tiles, int cap);
bool attn_prefill_supported(int head_dim);

// qh: [M, H*hd] bf16 queries pre-scaled by log2(e)/sqrt(hd); kscr/vscr: the
// chunk's K/V [M, KV*hd]; keys before each sequence's chunk come from kv.
// out: [M, H*hd] bf16.
cudaError_t launch_attn_prefill(int n_tiles, const int2* tiles, int H, int KV, int hd, const bf16* qh,
                                const bf16* kscr, const bf16* vscr, KVView kv, RowMeta m, bf16* out,
                                cudaStream_t st);

}  // namespace dory

// Fused GQA attention for decode and speculative chunks.
#pragma once

#include "kernels.cuh"

namespace dory {

constexpr int DEC_BK = 128;  // keys per block (absolute-position aligned)

// Use the cluster kernels (blocks per row and KV head merged through
// distributed shared memory) when the device can schedule them: 0 never,
// 1 with the cluster size chosen from the number of sequences, 4 / 8 / 16
// with that cluster size.
extern int g_attn_cluster;

// Attention of M rows whose K/V go straight into the cache.  qkv: the QKV
// projection's S split-K partial slices (slice stride ps floats, rows of
// q_dim + 2 kv_dim).  part: [part_rows, H, nb_cap, hd + 4] scratch, used
// only when the cluster kernels cannot run (then M <= part_rows is
// required); counters: [M * KV] zeros (left zero on return).  out: [M, H * hd]
// in the storage type.  batch: sequences in the call (rows may be several
// per sequence); selects how many blocks share one row's keys.
// Blocks the bf16 tensor-core decode attention runs for one row per
// sequence of `batch` sequences (0 when it would not run).
int attn_decode_ctas(int batch, int KV, int hd, int G);

template <typename T>
cudaError_t launch_attn_decode(int M, int H, int KV, int hd, const float* qkv, int S, size_t ps, KVView kv,
                               RowMeta m, int max_ctx, float* part, int nb_cap, int part_rows, unsigned* counters,
                               T* out, int batch, cudaStream_t st);

}  // namespace dory

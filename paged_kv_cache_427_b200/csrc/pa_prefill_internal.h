// pa_prefill_internal.h - host-side interface between the C ABI (pa_api.cu) and the prefill
// kernel files: the validated arguments, the tensor maps and the kernel table entry.
#pragma once

#include "pa_internal.h"

namespace pa {

// Causal attention of a step's new tokens (prefill): query row r = query_start[s] + j is
// token j of sequence s's q_len new tokens, at position context_len - q_len + j.
struct PrefillArgs {
  void *out;
  int out_dtype;
  int64_t out_t, out_h;  // elements
  const void *query;
  int64_t q_t, q_h;      // elements
  const int32_t *block_tables;
  int64_t bt_s;
  const int32_t *context_lens;
  const int32_t *query_start;
  int num_seqs;
  int num_kv_heads;
  int max_blocks;
  int64_t num_blocks;
  int64_t num_tokens;   // query rows
  float scale_log2;
  unsigned int *err;
  long long wait_cycles;
  int grouped_maps;  // 1: the maps are the grouped view (one box per block and kv head)
  // Shared-prefix pass (pa_decode_shared_prefix) when pre_o is not null: the query rows are the
  // decode queries of consecutive sequences (query_start unused), group g's members are
  // sequences group_start[g] .. group_start[g+1]-1, and every member's rows attend, with no
  // causal limit, to positions 0 .. P-1 of the group's shared prefix, P = prefix_lens of the
  // first member, read through the first member's block table.  The work is cut into items
  // of pre_kv kv tiles; item sigma of (member, head) stores O / l and (m, l), m in base 2.
  const int32_t *group_start;  // [num_groups + 1]
  const int32_t *prefix_lens;  // [num_seqs]
  int num_groups;
  int pre_kv;                  // kv tiles (128 positions) per item
  int pre_splits;              // item slots per (sequence, query head)
  float *pre_o;                // [num_seqs][num_heads][pre_splits][head_dim]
  float *pre_ml;               // [num_seqs][num_heads][pre_splits][2]
};

// The prefill's tensor maps: the caches (grouped view, or 8-row boxes) and the query rows.
struct PrefillMaps {
  CUtensorMap k;
  CUtensorMap v;
  CUtensorMap q;
};

struct PrefillKernel {
  cudaError_t (*launch)(const PrefillArgs &, const PrefillMaps *, int num_ctas, cudaStream_t);
  const void *kernel;
  int threads_per_cta;
  int smem_bytes;
  int tokens_per_tile;  // query tokens of one tile (128 rows / query heads per kv head)
  int tma_rows;
};

bool prefill_kernel_bf16(int head_dim, int block_size, int group, PrefillKernel *k);
bool prefill_kernel_f16(int head_dim, int block_size, int group, PrefillKernel *k);

}  // namespace pa

// pa_internal.h - host-side interface between the C ABI (pa_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

struct CacheWriteArgs {
  const char *key;
  const char *value;
  int64_t k_tok, k_head, v_tok, v_head;  // bytes
  char *key_cache;
  char *value_cache;
  int64_t c_blk, c_head;  // bytes
  int row_bytes;
  const int64_t *slots;
  int64_t num_tokens;
  int num_kv_heads;
  int block_size;
  int64_t num_slots;
  unsigned int *err;
};

// Everything a decode launch needs, already validated.  Strides are in elements.
struct DecodeArgs {
  void *out;
  int out_dtype;
  int64_t out_s, out_h;
  const void *query;
  int64_t q_s, q_h;
  int q_heads_contiguous;  // query heads of one group form one contiguous run
  const void *key_cache;
  const void *value_cache;
  int64_t kv_blk, kv_head;
  const int32_t *block_tables;
  int64_t bt_s;
  const int32_t *context_lens;
  int num_seqs;
  int num_kv_heads;
  int max_blocks;
  int64_t num_blocks;
  float scale_log2;  // scale * log2(e): logits are kept in base-2 units
  int num_workers;   // warps sharing the work
  int piece_cost;    // the split's cost of a (sequence, kv head) start, in chunks (see the split)
  // workspace (see pa_api.cu for the layout)
  unsigned int *counters;
  int2 *pair_meta;
  float *part_ml;
  float *part_o;
  unsigned int *err;
  const float *k_scale;   // FP8 caches: per kv head, the key/value of a code is code * scale
  const float *v_scale;
  int separate_reduce;
  long long wait_cycles;  // limit of every wait on a copy (about one second by default)
  int test_stall;         // test hook: 1 every worker's first stage expects 16 bytes nobody
                          // sends, 2 only the odd-numbered workers'
  // Measurement aid (pa_set_decode_timeline): kTimelineWords 64-bit records per worker warp
  // (those with index < timeline_warps), or null.
  unsigned long long *timeline;
  long long timeline_warps;
  // Shared prefixes (pa_decode_shared_prefix), or null: sequence s decodes only positions
  // prefix_lens[s] .. L-1 when 0 < prefix_lens[s] < L and prefix_lens[s] is a multiple of the
  // block size (otherwise its whole context), and merges the pre_splits partial results
  // (pre_o, pre_ml, laid out as in the prefill's shared-prefix pass) that the prefix pass left
  // for its first ceil(ceil(prefix / pre_kv_tokens)) items.
  const int32_t *prefix_lens;
  const float *pre_o;
  const float *pre_ml;
  int pre_splits;
  int pre_kv_tokens;  // positions per prefix item
  // The grid before this one is the prefix pass, launched in stream order after every writer of
  // this grid's inputs: the decode streams at once and waits for that grid only before a merge
  // that reads its partial results (and before its producer exits, so that this grid cannot
  // complete first).
  int prefix_overlap;
  // Fused decode step (pa_decode_step with one new token per sequence), when fused != 0: the
  // kernel also performs this cache write (its merge warps, after the previous grid), and reads
  // position L-1 of sequence s from the new token s (step.key / step.value) instead of the
  // cache, so that the decode never waits for the write.
  int fused;
  CacheWriteArgs step;
};

// Fields of one worker warp's timeline record.
enum TimelineField {
  kTlStart = 0,     // global ns when the warp begins (after the CTA's set-up)
  kTlFirst = 1,     // its first tile has landed
  kTlLast = 2,      // its last tile is consumed (before its last piece's epilogue)
  kTlDone = 3,      // the warp is finished (epilogue and merges included)
  kTlSm = 4,        // the SM it ran on
  kTlChunks = 5,    // chunks in its share
  kTlIssue = 6,     // the producer may read the caches (the previous grid has finished)
  kTlMerged = 7,    // the CTA's merge warp is finished (the pieces it published, merged)
  kTimelineWords = 8
};

// TMA descriptors of the two caches, viewed as 5-D tensors (64 elements, block_size rows,
// head_dim / 64 column halves, kv heads, blocks) read in 128-byte swizzled boxes of
// 64 x tma_rows x head_dim/64: one box holds a whole (rows x head_dim) tile as
// [half][row][128 bytes].
struct TmaMaps {
  CUtensorMap k;
  CUtensorMap v;
};

struct DecodeKernel {
  cudaError_t (*launch)(const DecodeArgs &, const TmaMaps *, int num_ctas, bool overlap_previous,
                        cudaStream_t);
  cudaError_t (*launch_reduce)(const DecodeArgs &, cudaStream_t);
  const void *kernel;  // for occupancy queries
  int warps_per_cta;    // worker warps per CTA (each takes one share of the chunk list)
  int threads_per_cta;  // all threads of a CTA (workers plus any helper warp)
  int smem_bytes;
  int chunk_tokens;
  int tma_rows;  // 0: the kernel reads the caches with 1-D bulk copies; else TMA box rows
};

// Kernel tables, one per element type.  `tensor_cores` selects the mma.sync kernel (16-bit
// types only).  Return false when the combination is not built.
bool decode_kernel_f32(int head_dim, int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_bf16(int head_dim, int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_f16(int head_dim, int block_size, int group, bool tensor_cores, DecodeKernel *k);


// Whole-block copies from one pair of caches to another (the same pair for copy-on-write,
// device and pinned host memory for swapping).
struct CopyBlocksArgs {
  const char *src_key, *src_value;
  char *dst_key, *dst_value;
  int64_t src_blk, src_head;  // bytes
  int64_t dst_blk, dst_head;  // bytes
  int tile_bytes;             // block_size * row bytes: one (block, kv head) tile
  const int64_t *pairs;
  int64_t num_pairs;
  int num_kv_heads;
  int64_t src_blocks, dst_blocks;
  unsigned int *err;
};

cudaError_t launch_reshape_and_cache(const CacheWriteArgs &a, int num_sms, cudaStream_t st);

// Quantising write into FP8 E4M3 caches: code(x / scale[h]) per element, x of element type
// src_dtype (fp32, bf16 or fp16).
struct CacheWriteFp8Args {
  const char *key;
  const char *value;
  int src_dtype;
  int64_t k_tok, k_head, v_tok, v_head;  // bytes
  unsigned char *key_cache;
  unsigned char *value_cache;
  int64_t c_blk, c_head;  // bytes
  int head_dim;
  const int64_t *slots;
  int64_t num_tokens;
  int num_kv_heads;
  int block_size;
  int64_t num_slots;
  const float *k_scale;
  const float *v_scale;
  unsigned int *err;
};

cudaError_t launch_reshape_and_cache_fp8(const CacheWriteFp8Args &a, int num_sms, cudaStream_t st);

// Tensor-core decode for FP8 E4M3 caches with a bf16 or fp16 query (head_dim 128 only).
bool decode_kernel_fp8(int q_dtype, int head_dim, int block_size, int group, DecodeKernel *k);

// For the allocation-free entry point: the scratch bytes a pa_decode call with these shapes
// needs (0 when the arguments are invalid), decode into a given scratch buffer, and set the
// message pa_last_error() returns.
size_t decode_scratch_need(const pa_tensor *query, const pa_tensor *key_cache, int32_t block_size,
                           int32_t num_kv_heads);
int decode_into(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                const pa_tensor *value_cache, const pa_tensor *block_tables,
                const pa_tensor *context_lens, float scale, int32_t block_size,
                int32_t num_kv_heads, void *workspace, size_t workspace_bytes, void *stream);
void set_last_error(const char *msg);
cudaError_t launch_copy_blocks(const CopyBlocksArgs &a, int num_sms, cudaStream_t st);

}  // namespace pa

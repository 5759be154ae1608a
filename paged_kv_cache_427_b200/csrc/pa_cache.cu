// pa_cache.cu - the write side of the paged KV cache on sm_100a: slot-mapped insertion of new
// tokens and whole-block copies.
//
// Sources: [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization
// support, distributed inference" 4.1 (each generated token appends one mapping to the block
// table; sequences may share physical blocks, e.g. in parallel sampling) and [P4] "vLLM core
// architecture: model loading, PagedAttention principle, KV cache management" 2.2.1 (logical
// and physical blocks of one fixed size; shared blocks for beam search).
//
// Both operations are pure byte moves, tiny next to attention (at most a few MB per step), and
// are written as grid-stride loops over 16-byte vectors: every thread moves one 16-byte piece
// of one (token or block, kv head) row, so a warp covers 512 contiguous bytes per access.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// One thread per 16-byte piece of one (token, kv head) row, keys and values together.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(CacheWriteArgs a) {
  // Launched as a programmatic dependent of the kernel before it: wait for that kernel (and its
  // memory) before touching anything.  Then a decode launched to overlap this grid may start;
  // it waits for this grid's writes before it reads the caches.
  wait_for_previous_grid();
  allow_next_grid();
  const int vec_per_row = a.row_bytes >> 4;
  const int64_t total = a.num_tokens * a.num_kv_heads * vec_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int v = (int)(idx % vec_per_row);
    const int64_t th = idx / vec_per_row;
    const int h = (int)(th % a.num_kv_heads);
    const int64_t t = th / a.num_kv_heads;
    const int64_t slot = __ldg(a.slots + t);
    if (slot < 0) continue;  // padding token
    if (slot >= a.num_slots) {
      if (h == 0 && v == 0) set_error(a.err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = slot / a.block_size;
    const int64_t off = slot % a.block_size;
    const int64_t dst = blk * a.c_blk + h * a.c_head + off * a.row_bytes + v * 16;
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(a.key + t * a.k_tok + h * a.k_head) + v);
    const uint4 vv =
        __ldg(reinterpret_cast<const uint4 *>(a.value + t * a.v_tok + h * a.v_head) + v);
    *reinterpret_cast<uint4 *>(a.key_cache + dst) = kv;
    *reinterpret_cast<uint4 *>(a.value_cache + dst) = vv;
  }
}

// One thread per 16-byte piece of one (pair, kv head) tile, keys and values together.  Source
// and destination caches may be the same tensors (copy-on-write) or live in different memory
// (swap between device memory and pinned host memory mapped into the device's address space).
__global__ void __launch_bounds__(256) copy_blocks_kernel(CopyBlocksArgs a) {
  wait_for_previous_grid();  // launched as a programmatic dependent, as the write kernel
  allow_next_grid();
  const int vec_per_tile = a.tile_bytes >> 4;
  const int64_t total = a.num_pairs * a.num_kv_heads * vec_per_tile;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int v = (int)(idx % vec_per_tile);
    const int64_t ph = idx / vec_per_tile;
    const int h = (int)(ph % a.num_kv_heads);
    const int64_t p = ph / a.num_kv_heads;
    const int64_t src = __ldg(a.pairs + 2 * p);
    const int64_t dst = __ldg(a.pairs + 2 * p + 1);
    if (src < 0 || src >= a.src_blocks || dst < 0 || dst >= a.dst_blocks) {
      if (h == 0 && v == 0) set_error(a.err, PA_DEVERR_COPY_PAIR);
      continue;
    }
    const int64_t so = src * a.src_blk + h * a.src_head + (int64_t)v * 16;
    const int64_t d = dst * a.dst_blk + h * a.dst_head + (int64_t)v * 16;
    const uint4 kv = *reinterpret_cast<const uint4 *>(a.src_key + so);
    const uint4 vv = *reinterpret_cast<const uint4 *>(a.src_value + so);
    *reinterpret_cast<uint4 *>(a.dst_key + d) = kv;
    *reinterpret_cast<uint4 *>(a.dst_value + d) = vv;
  }
}

// One thread per 16 codes (16 elements) of one (token, kv head) row, keys and values together.
// Each element is divided by its head's scale in fp32 (IEEE division) before the conversion.
template <typename S>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(CacheWriteFp8Args a) {
  wait_for_previous_grid();  // launched as a programmatic dependent, as the 16-bit write
  allow_next_grid();
  const int vec_per_row = a.head_dim >> 4;
  const int64_t total = a.num_tokens * a.num_kv_heads * vec_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int v = (int)(idx % vec_per_row);
    const int64_t th = idx / vec_per_row;
    const int h = (int)(th % a.num_kv_heads);
    const int64_t t = th / a.num_kv_heads;
    const int64_t slot = __ldg(a.slots + t);
    if (slot < 0) continue;  // padding token
    if (slot >= a.num_slots) {
      if (h == 0 && v == 0) set_error(a.err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t dst = (slot / a.block_size) * a.c_blk + h * a.c_head +
                        (slot % a.block_size) * a.head_dim + v * 16;
    const float ks = __ldg(a.k_scale + h), vs = __ldg(a.v_scale + h);
    *reinterpret_cast<uint4 *>(a.key_cache + dst) =
        fp8_codes16<S>(a.key + t * a.k_tok + h * a.k_head + (int64_t)v * 16 * sizeof(S), ks);
    *reinterpret_cast<uint4 *>(a.value_cache + dst) =
        fp8_codes16<S>(a.value + t * a.v_tok + h * a.v_head + (int64_t)v * 16 * sizeof(S), vs);
  }
}

static int grid_for(int64_t items, int num_sms) {
  const int64_t blocks = (items + 255) / 256;
  const int64_t cap = (int64_t)num_sms * 8;
  return (int)(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

// Launch as a programmatic dependent of the kernel before it on `st`: the grid may become
// resident while that kernel finishes (its launch latency hidden behind that kernel's last
// CTAs); every thread waits for that kernel and its memory before it reads or writes anything.
template <typename A>
cudaError_t launch_dependent(void (*kernel)(A), int grid, cudaStream_t st, const A &a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_reshape_and_cache(const CacheWriteArgs &a, int num_sms, cudaStream_t st) {
  const int64_t items = a.num_tokens * a.num_kv_heads * (a.row_bytes / 16);
  if (items == 0) return cudaSuccess;
  return launch_dependent(reshape_and_cache_kernel, grid_for(items, num_sms), st, a);
}

cudaError_t launch_copy_blocks(const CopyBlocksArgs &a, int num_sms, cudaStream_t st) {
  const int64_t items = a.num_pairs * a.num_kv_heads * (a.tile_bytes / 16);
  if (items == 0) return cudaSuccess;
  return launch_dependent(copy_blocks_kernel, grid_for(items, num_sms), st, a);
}

cudaError_t launch_reshape_and_cache_fp8(const CacheWriteFp8Args &a, int num_sms, cudaStream_t st) {
  const int64_t items = a.num_tokens * a.num_kv_heads * (a.head_dim / 16);
  if (items == 0) return cudaSuccess;
  const int grid = grid_for(items, num_sms);
  if (a.src_dtype == PA_F32) return launch_dependent(reshape_and_cache_fp8_kernel<float>, grid, st, a);
  if (a.src_dtype == PA_BF16)
    return launch_dependent(reshape_and_cache_fp8_kernel<__nv_bfloat16>, grid, st, a);
  return launch_dependent(reshape_and_cache_fp8_kernel<__half>, grid, st, a);
}

}  // namespace pa

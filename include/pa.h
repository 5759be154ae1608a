/*
 * pa.h - C ABI of a paged KV-cache decode-attention library for NVIDIA B200 (sm_100a).
 *
 * Sources (web tutorials on vLLM, cited by page and section):
 *   [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization support,
 *        distributed inference", section 4.1: the KV cache is cut into fixed-size blocks; a
 *        block table records the physical block behind each logical block; generating a token
 *        appends one mapping; several sequences may share physical blocks.
 *   [P3] "Core inference engine (part 1): vLLM architecture, PagedAttention principle,
 *        Continuous Batching mechanism", section 2.2: pages of a fixed number of tokens (e.g.
 *        16) scattered through memory and found through a page table; shared prompt pages;
 *        page size is a tuning parameter (8 vs 32).
 *   [P4] "vLLM core architecture: model loading, PagedAttention principle, KV cache
 *        management", section 2.2.1 (logical block, physical block of the same size, block
 *        table; block size 16 by default, 8 or 32 as alternatives) and section 2.2.2
 *        (attention assembles each sequence's complete KV sequence through its block table).
 *
 * Conventions shared by every call
 *   - Tensors are described by pa_tensor: a device pointer, an element type, a shape and
 *     strides counted in elements.  The caller owns every buffer; the library never frees or
 *     keeps a caller pointer beyond the call.  All buffers of one call live on the current CUDA
 *     device.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Every
 *     call only enqueues work on that stream and returns; none reads device data on the host
 *     or synchronises, except pa_get_device_error, which says so.  Launch sizes come from
 *     shapes only, never from the values in context_lens.
 *   - Host-side checks (shapes, element types, strides, 16-byte alignment, that every tensor
 *     lies inside one device allocation) reject bad arguments before anything is enqueued;
 *     the call then returns a negative pa_status and pa_last_error() describes the problem.
 *   - Values that only the device sees (block ids, slots, context lengths) are checked by the
 *     kernels: a bad value sets a bit in the per-device error word (pa_get_device_error) and
 *     the offending access is redirected or skipped, never performed out of bounds.  The
 *     result for the affected sequence is then unspecified.
 *
 * Layouts
 *   key_cache, value_cache  [num_blocks, num_kv_heads, block_size, head_dim]; the innermost
 *                           two dimensions contiguous (so one (block, kv head) tile is one
 *                           contiguous run of block_size * head_dim elements); the two caches
 *                           share shape, element type and strides.  Physical-block-major order
 *                           follows [P4] 2.2.2; head before token is this library's choice.
 *   query, out              [num_seqs, num_heads, head_dim], head_dim contiguous.
 *   key, value (new tokens) [num_tokens, num_kv_heads, head_dim], head_dim contiguous.
 *   block_tables            [num_seqs, max_blocks] int32, row-major with unit inner stride.
 *   context_lens            [num_seqs] int32, contiguous; counts every token of the sequence,
 *                           including the one written in this step.
 *   slot_mapping            [num_tokens] int64, contiguous; slot = block * block_size + offset,
 *                           negative = padding token (nothing stored).
 *   block_mapping           [num_pairs, 2] int64, contiguous (src, dst) block ids.
 * Query head h reads kv head h / (num_heads / num_kv_heads).
 *
 * Supported: element types fp32, bf16, fp16 (query and caches of one type; out either that
 * type or fp32); head_dim 64 or 128; block_size 8, 16 or 32; num_heads / num_kv_heads in
 * {1, 2, 4, 8}.  Other combinations return PA_ERR_UNSUPPORTED.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_VERSION 7

/* Symbols of this ABI are the only ones the shared library exports. */
#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

typedef enum pa_dtype {
  PA_F32 = 0,
  PA_BF16 = 1,
  PA_F16 = 2,
  PA_I32 = 3,
  PA_I64 = 4,
  PA_FP8_E4M3 = 5 /* KV caches only, with per-kv-head fp32 scales: see pa_decode_fp8 */
} pa_dtype;

#define PA_MAX_DIMS 5

typedef struct pa_tensor {
  void *data;                  /* device pointer of element [0, 0, ...] */
  int32_t dtype;               /* pa_dtype */
  int32_t ndim;                /* 1 .. PA_MAX_DIMS */
  int64_t shape[PA_MAX_DIMS];  /* sizes; entries past ndim are ignored */
  int64_t stride[PA_MAX_DIMS]; /* strides in elements; entries past ndim are ignored */
} pa_tensor;

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1, /* NULL pointer, negative size, unknown flag, ... */
  PA_ERR_SHAPE = -2,       /* shapes disagree with each other or with block_size/num_kv_heads */
  PA_ERR_DTYPE = -3,       /* element type not allowed for this argument */
  PA_ERR_UNSUPPORTED = -4, /* valid but not built: head_dim, block_size or group size */
  PA_ERR_CUDA = -5,        /* a CUDA runtime call or a launch failed; see pa_last_error() */
  PA_ERR_WORKSPACE = -6,   /* workspace missing, too small or misaligned */
  PA_ERR_LAYOUT = -7       /* stride or alignment requirement not met, or tensor not inside
                              one device allocation of the current device */
} pa_status;

/* Bits of the per-device error word set by kernels (see pa_get_device_error). */
#define PA_DEVERR_BLOCK_ID 0x1u    /* a block-table entry needed for a context lay outside
                                      [0, num_blocks); block 0 was read instead */
#define PA_DEVERR_CONTEXT_LEN 0x2u /* context_len < 0 (treated as 0) or > max_blocks *
                                      block_size (clamped) */
#define PA_DEVERR_SLOT 0x4u        /* slot >= num_blocks * block_size; the token was skipped */
#define PA_DEVERR_COPY_PAIR 0x8u   /* a copy pair held an id outside [0, num_blocks); skipped */
#define PA_DEVERR_TIMEOUT 0x10u    /* an asynchronous copy did not complete within about one
                                      second; the kernel abandoned its work and returned, and
                                      the results of that call are unspecified.  Recovery:
                                      reading the word with pa_get_device_error while this bit
                                      is set marks every decode workspace the library has seen
                                      (the library-owned ones, the callers' workspaces, and the
                                      static scratch of pa_decode_noalloc) so that the next
                                      decode call using it zeroes its merge counters first;
                                      no other step is needed */

#define PA_DEVERR_PREFIX 0x20u     /* pa_decode_shared_prefix: a group's members disagree on
                                      their shared prefix (length or physical blocks), or a
                                      prefix is not a whole number of blocks; such a sequence
                                      is decoded over its whole context instead where it can
                                      be, otherwise its result is unspecified */

/* Flags of pa_decode_ex. */
#define PA_DECODE_SEPARATE_REDUCE 0x1u /* merge split contexts in a second kernel instead of
                                          in the last warp to finish each (sequence, kv head) */
#define PA_DECODE_CUDA_CORES 0x2u      /* 16-bit caches: use the CUDA-core kernel instead of the
                                          tensor-core (mma.sync + TMA) one; fp32 caches always
                                          use the CUDA-core kernel */
#define PA_DECODE_OVERLAP_PREVIOUS 0x4u /* let the decode kernel start while the kernel launched
                                          just before it on `stream` is still running
                                          (programmatic dependent launch): it reads context_lens
                                          and block_tables, and may zero the out rows of empty
                                          contexts, before it waits for that kernel; it reads
                                          the caches and the query only after.  Use it only when
                                          that kernel writes none of context_lens, block_tables
                                          and out, e.g. right after pa_reshape_and_cache */

/*
 * pa_reshape_and_cache - store this step's new keys and values into their cache slots.
 * [P2] 4.1: each generated token appends one logical->physical mapping; the scheduler hands
 * the token a slot, and its K/V rows go to offset slot % block_size of physical block
 * slot / block_size, for every kv head:
 *   key_cache[slot / bs, h, slot % bs, :] = key[i, h, :]   (value alike), for slot >= 0.
 * key, value: [T, Hkv, D]; caches as above; slot_mapping: [T] int64.  Copies are bit-exact.
 * Slots must be distinct within a call (otherwise which token lands is unspecified).
 * A slot >= num_blocks * block_size sets PA_DEVERR_SLOT and that token is skipped.
 */
PA_API int pa_reshape_and_cache(const pa_tensor *key, const pa_tensor *value,
                         const pa_tensor *key_cache, const pa_tensor *value_cache,
                         const pa_tensor *slot_mapping, void *stream);

/*
 * pa_decode_step - one whole decode step: pa_reshape_and_cache(key, value, key_cache,
 * value_cache, slot_mapping) followed by pa_decode_ex(out, query, key_cache, value_cache,
 * block_tables, context_lens, ..., num_workers = 0, PA_DECODE_OVERLAP_PREVIOUS, workspace),
 * i.e. the write side of [P2] 4.1 and the attention of [P4] 2.2.2 for the same step.
 * One new token per sequence (key->shape[0] == number of sequences) in bf16 or f16 caches:
 * the step is ONE kernel.  Token s is sequence s's position context_lens[s] - 1; the kernel
 * stores it into slot slot_mapping[s] and, for that position, attends to the rows of key and
 * value themselves, so no part of the decode waits for the store.  A slot that is not that
 * position under block_tables (or a token of an empty context) is still stored as asked and
 * sets PA_DEVERR_SLOT; out rows of empty contexts are zeroed.  Any other shape (several
 * tokens per sequence, fp32 caches): two kernels, the write and then the decode, launched as
 * a programmatic dependent of the write: its prologue (context_lens, block_tables, the split
 * of the work) runs while the write finishes, and it reads the caches only after.  Both
 * halves are validated before either is launched, so a refused call launches nothing.
 * In both forms the decode waits for the kernel launched before it on `stream` before it
 * reads the caches or the query (programmatic dependent launch, as under
 * PA_DECODE_OVERLAP_PREVIOUS, with the same rule for what that kernel may write).
 * workspace: as for pa_decode_ex, or NULL for the library-owned one of pa_decode.
 * With a caller workspace initialised beforehand (pa_workspace_init) the call allocates
 * nothing and can be captured into a CUDA graph (one graph node per kernel, the programmatic
 * dependency kept as a graph edge); the graph is valid as long as the tensors it was captured
 * with stay where they are.  Errors as for the two calls; on PA_ERR_CUDA from the decode launch
 * of the two-kernel form the cache write may already have been launched.
 */
PA_API int pa_decode_step(const pa_tensor *key, const pa_tensor *value,
                          const pa_tensor *key_cache, const pa_tensor *value_cache,
                          const pa_tensor *slot_mapping, const pa_tensor *out,
                          const pa_tensor *query, const pa_tensor *block_tables,
                          const pa_tensor *context_lens, float scale, int32_t block_size,
                          int32_t num_kv_heads, void *workspace, size_t workspace_bytes,
                          void *stream);

/*
 * FP8 KV cache ([P2] 4.3 lists FP8 E4M3, 8-bit floating point, about half the memory of 16-bit,
 * among the supported storage formats; storing the KV cache in it with one fp32 scale per kv
 * head is this library's reading).  E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 fraction
 * bits, subnormals below 2^-6, no infinities, largest finite magnitude 448, NaN = S.1111.111.
 * The cache holds code(x / scale[h]); attention reads decode(code) * scale[h].
 *
 * pa_reshape_and_cache_fp8 - pa_reshape_and_cache into FP8 caches: for each element x of
 * key[i, h, :] (value alike) the code of x / k_scale[h] is stored, the division in fp32
 * (correctly rounded), the code the nearest E4M3 value (ties to the even code), magnitudes
 * beyond 448 saturated to 448, NaN kept.  key, value: [T, Hkv, D] fp32, bf16 or fp16;
 * caches: fp8_e4m3 [NB, Hkv, bs, D]; k_scale, v_scale: fp32 [Hkv] device memory.  Slots as for
 * pa_reshape_and_cache.  The codes equal the oracle's bit for bit.
 */
PA_API int pa_reshape_and_cache_fp8(const pa_tensor *key, const pa_tensor *value,
                                    const pa_tensor *key_cache, const pa_tensor *value_cache,
                                    const pa_tensor *slot_mapping, const pa_tensor *k_scale,
                                    const pa_tensor *v_scale, void *stream);

/*
 * pa_decode_fp8 - pa_decode_ex over FP8 caches: K_t = decode(code) * k_scale[g] and V_t =
 * decode(code) * v_scale[g] for kv head g, then the same attention.  query: bf16 or fp16;
 * out: fp32 or the query's type.  head_dim 128 (other sizes PA_ERR_UNSUPPORTED); block_size
 * 8/16/32; 1/2/4/8 query heads per kv head.  The tensor-core kernel widens each tile to fp16
 * (exact) and scales each query head by a power of two into the fp16 range (1/alpha folded
 * into its logit scale), so the accuracy is that of the 16-bit caches.  workspace NULL: the
 * library-owned workspace of pa_decode; otherwise as for pa_decode_ex.  Flags as for
 * pa_decode_ex except PA_DECODE_CUDA_CORES (PA_ERR_UNSUPPORTED).  pa_copy_blocks and
 * pa_swap_blocks move FP8 blocks as bytes.
 */
PA_API int pa_decode_fp8(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                         const pa_tensor *value_cache, const pa_tensor *block_tables,
                         const pa_tensor *context_lens, const pa_tensor *k_scale,
                         const pa_tensor *v_scale, float scale, int32_t block_size,
                         int32_t num_kv_heads, int32_t num_workers, uint32_t flags,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_decode_step_fp8 - one whole decode step over FP8 caches: pa_reshape_and_cache_fp8(key,
 * value, key_cache, value_cache, slot_mapping, k_scale, v_scale) followed by pa_decode_fp8(out,
 * query, ..., num_workers = 0, PA_DECODE_OVERLAP_PREVIOUS, workspace), as pa_decode_step is for
 * 16-bit caches.  One new token per sequence (key->shape[0] == number of sequences) whose
 * key/value have the query's 16-bit type: ONE kernel.  Token s is sequence s's position
 * context_lens[s] - 1; the kernel quantises it into slot slot_mapping[s] (codes identical to
 * pa_reshape_and_cache_fp8's) and attends to those same codes for that position, so no part of
 * the decode waits for the write; a slot that is not that position is stored as asked and sets
 * PA_DEVERR_SLOT.  Any other shape or an fp32 key/value: two kernels, the write and then the
 * decode launched to overlap it.  Both halves are validated before either is launched.
 * workspace as for pa_decode_fp8 (NULL: the library-owned one).  Errors as for the two calls.
 */
PA_API int pa_decode_step_fp8(const pa_tensor *key, const pa_tensor *value,
                              const pa_tensor *key_cache, const pa_tensor *value_cache,
                              const pa_tensor *slot_mapping, const pa_tensor *k_scale,
                              const pa_tensor *v_scale, const pa_tensor *out,
                              const pa_tensor *query, const pa_tensor *block_tables,
                              const pa_tensor *context_lens, float scale, int32_t block_size,
                              int32_t num_kv_heads, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * pa_prefill - causal attention of a step's new tokens (a prompt, or a chunk of one, of each
 * sequence joining or continuing in the batch: [P2] 4.2) over the paged cache.  Sequence s
 * brings q_len = query_start[s+1] - query_start[s] new tokens, already written into its blocks
 * (pa_reshape_and_cache); they are its last q_len positions, and new token j (query row
 * query_start[s] + j, position p = context_lens[s] - q_len + j) attends to positions 0 .. p:
 *   out[r, h, :] = softmax_{t <= p}(scale * q[r, h, :] . K_t) . V_t,
 * K_t, V_t assembled through the block table as in pa_decode ([P4] 2.2.2).
 *   query, out: [T, Hq, D] (T = query_start[S]); out fp32 or the caches' type.
 *   query_start: [S + 1] int32, non-decreasing from 0; block_tables [S, max_blocks];
 *   context_lens [S].  Caches bf16 or fp16 (fp32 / FP8: PA_ERR_UNSUPPORTED), head_dim 64 or
 *   128, block_size 8/16/32, 1/2/4/8 query heads per kv head.
 *   query and out need a contiguous head_dim and 16-byte aligned data and token/head strides
 *   (PA_ERR_LAYOUT otherwise).
 * A sequence with q_len > context_len, or whose rows fall outside [0, T), sets
 * PA_DEVERR_CONTEXT_LEN and its rows are not written.  Rows of tokens past query_start[S] are
 * not written.  Asynchronous on `stream`; every tensor is the caller's and stays so.
 * One kernel on the fifth-generation tensor cores: a persistent grid, one CTA per SM, each
 * taking tiles of 128 query rows (128/G tokens x G heads) of one (sequence, kv head) and
 * streaming that sequence's K/V tiles up to the tile's last position by TMA; tcgen05 MMAs
 * compute S = QK^T and O = PV into tensor memory, with P kept to ~16 bits (two bf16/fp16
 * terms).  Caches whose blocks are kv heads x rows x head_dim contiguous are read one
 * (block, kv head) tile per copy, other layouts in 8-row copies.
 */
PA_API int pa_prefill(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                      const pa_tensor *value_cache, const pa_tensor *block_tables,
                      const pa_tensor *context_lens, const pa_tensor *query_start, float scale,
                      int32_t block_size, int32_t num_kv_heads, void *stream);

/*
 * pa_copy_blocks - copy whole physical blocks (all kv heads, all slots, both caches):
 *   key_cache[dst] = key_cache[src], value_cache[dst] = value_cache[src]
 * for each (src, dst) row of block_mapping [N, 2] int64.  This is the copy-on-write a block
 * shared by several sequences ([P2] 4.1 parallel sampling, [P3] 2.2 shared prompt pages,
 * [P4] 2.2.1 beam search) needs before one sharer writes into it.  Bit-exact.
 * Preconditions: dst ids distinct, and no dst is also a src in the same call.  A pair with an
 * id outside [0, num_blocks) sets PA_DEVERR_COPY_PAIR and is skipped.
 */
PA_API int pa_copy_blocks(const pa_tensor *key_cache, const pa_tensor *value_cache,
                   const pa_tensor *block_mapping, void *stream);

/*
 * pa_swap_blocks - move whole physical blocks between two caches, typically the device cache
 * and a swap cache in pinned host memory ([P4] 2.3.2: blocks, not whole requests, are swapped
 * out to CPU memory and back):
 *   dst_key_cache[dst] = src_key_cache[src], dst_value_cache[dst] = src_value_cache[src]
 * for each (src, dst) row of block_mapping [N, 2] int64 (src indexes the source caches, dst the
 * destination caches).  Both cache pairs have the element type, kv heads, block_size and
 * head_dim of the other; their block counts may differ.  Each tensor (the mapping included) is
 * device memory of the current device or pinned host memory mapped into its address space
 * (cudaHostAlloc / cudaMallocHost; the extent of host memory is not checked); pageable host
 * memory returns PA_ERR_LAYOUT.  One kernel moves every block, 16 bytes per thread, so host
 * memory is read or written directly over the host link.  Bit-exact.  Preconditions: dst ids
 * distinct; the source and destination blocks do not overlap.  A pair with an id outside its
 * cache sets PA_DEVERR_COPY_PAIR and is skipped.
 */
PA_API int pa_swap_blocks(const pa_tensor *src_key_cache, const pa_tensor *src_value_cache,
                          const pa_tensor *dst_key_cache, const pa_tensor *dst_value_cache,
                          const pa_tensor *block_mapping, void *stream);

/*
 * pa_decode - one decode step of paged attention.  For every sequence s and query head h,
 * with g = h / (num_heads / num_kv_heads) and L = context_lens[s], the context is assembled
 * through the block table ([P4] 2.2.2):
 *   K_t = key_cache[block_tables[s, t / bs], g, t % bs, :]   (V alike),  0 <= t < L,
 * and   out[s, h, :] = softmax_t(scale * q[s, h, :] . K_t) . V_t,
 * accumulated in fp32.  L = 0 gives a zero row.  Block-table entries past ceil(L / bs) are
 * never read.  The per-block loop printed in [P4] 2.2.2 states only the principle; this is the
 * full-context softmax it stands for.
 *
 * Long contexts are split across warps; partial results are merged with the log-sum-exp rule.
 * pa_decode uses a library-owned workspace per device, allocated (cudaMalloc, then zeroed on
 * `stream`) the first time a call needs more than the current one holds: such a first call
 * must not happen during stream capture, and concurrent pa_decode calls on different streams
 * of one device must not overlap on the GPU (they share that workspace); use pa_decode_ex
 * with a workspace per stream for that.
 */
PA_API int pa_decode(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
              const pa_tensor *value_cache, const pa_tensor *block_tables,
              const pa_tensor *context_lens, float scale, int32_t block_size,
              int32_t num_kv_heads, void *stream);

/*
 * pa_decode_ex - pa_decode with caller-chosen parallel split and caller-owned workspace.
 *   num_workers   number of warps that split the step's work, each taking a contiguous share
 *                 of the (sequence, kv head, 16-row chunk) list of equal cost (a chunk costs
 *                 one, each (sequence, kv head) start a few more); 0 = one full wave of the
 *                 device.  1 computes every sequence in a single warp (no merging at all).
 *   flags         0 or PA_DECODE_SEPARATE_REDUCE.
 *   workspace     device memory of at least pa_decode_workspace_bytes(...) bytes, 256-byte
 *                 aligned, zero-filled before its first use (pa_workspace_init).  Every call
 *                 that completes leaves it ready for the next call.  Calls sharing one
 *                 workspace must not overlap on the GPU.
 */
PA_API int pa_decode_ex(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                 const pa_tensor *value_cache, const pa_tensor *block_tables,
                 const pa_tensor *context_lens, float scale, int32_t block_size,
                 int32_t num_kv_heads, int32_t num_workers, uint32_t flags, void *workspace,
                 size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace pa_decode_ex needs for num_seqs sequences of the given head counts and
 * head_dim with num_workers warps (0 = the largest default of the current device).  Returns
 * 0 on invalid arguments.
 */
PA_API size_t pa_decode_workspace_bytes(int64_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t num_workers);

/* The number of warps pa_decode uses for a configuration on the current device (0 on error). */
PA_API int32_t pa_decode_default_workers(int32_t dtype, int32_t head_dim, int32_t block_size,
                                  int32_t group_size);

/* Zero-fill a decode workspace on `stream` (before its first use; after a PA_DEVERR_TIMEOUT,
 * pa_get_device_error already arranges for the counters to be zeroed again). */
PA_API int pa_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Free the library-owned decode workspaces of every device (synchronises each device). */
PA_API int pa_release_workspaces(void);

/* Message for the last non-OK return of a pa_* call on this host thread ("" if none). */
PA_API const char *pa_last_error(void);

/*
 * Read the current device's error word into *flags (a mask of PA_DEVERR_* bits), after
 * waiting for `stream` to finish; clear it afterwards when `clear` is non-zero.  This call
 * synchronises `stream`.
 */
PA_API int pa_get_device_error(void *stream, uint32_t *flags, int32_t clear);

/*
 * pa_decode_noalloc - pa_decode for callers that cannot allocate device memory.
 *
 * The vLLM tutorials have no counterpart to this call; it exists for users of this library.
 * Some callers may not call cudaMalloc: code that runs while a stream is being captured into a
 * CUDA graph, engines that reserve all device memory up front for their own pool and forbid
 * later allocations, and latency-critical loops that cannot afford the implicit device
 * synchronisation an allocation or a free may cause.  pa_decode allocates its workspace on
 * first use and pa_decode_ex needs one from the caller; this call needs neither.
 *
 * Same arguments, semantics and tolerances as pa_decode.  Its scratch (merge counters and
 * partial results) is a fixed device array of PA_NOALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits.  A call whose shapes
 * need more scratch than that (roughly: more than about 3,000 (sequence, kv head) pairs at
 * head_dim 128 and 4 query heads per kv head) returns PA_ERR_WORKSPACE without launching.
 * Every call looks up the array's device address (cudaGetSymbolAddress, which allocates
 * nothing); the first call on a device, or the first after the module was reloaded, also
 * clears the array on `stream`: make that first call before any stream capture.  After a
 * PA_DEVERR_TIMEOUT, reading the error word (pa_get_device_error) is the whole recovery: the
 * next call zeroes the array's merge counters on its stream before the decode.  The call itself allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.  All calls share the one array, so
 * calls that overlap on the GPU (for instance on two streams) race and give wrong results;
 * issue them in one stream or one after another.
 */
#define PA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
PA_API int pa_decode_noalloc(const pa_tensor *out, const pa_tensor *query,
                             const pa_tensor *key_cache, const pa_tensor *value_cache,
                             const pa_tensor *block_tables, const pa_tensor *context_lens,
                             float scale, int32_t block_size, int32_t num_kv_heads, void *stream);

/*
 * pa_decode_shared_prefix - pa_decode for a batch whose sequences come in groups that share a
 * prompt prefix stored once: several sequences' block tables name the same physical blocks
 * ([P2] 4.1, parallel sampling and shared prompts; [P3] 2.2, shared prompt pages).  Same
 * result as pa_decode (within the same tolerances); the shared prefix is read once per kv head
 * for all members instead of once per member.
 *   group_start  [num_groups + 1] int32, non-decreasing from 0: group g is the consecutive
 *                sequences group_start[g] .. group_start[g+1] - 1 (a sequence in no group is a
 *                group of one).
 *   prefix_lens  [num_seqs] int32: the number of leading positions sequence s shares with the
 *                other members of its group; equal within a group, a multiple of block_size,
 *                and every member's block-table entries for those positions equal the first
 *                member's.  0 = nothing shared.
 * Two kernels on `stream`: the prefix pass computes, on the fifth-generation tensor cores,
 * every member's query rows (128 rows = 128 / G members x G heads per tile) against its group's
 * prefix, read once through the first member's block table, in items of 512 positions, and
 * stores partial results (O / l, running maximum, sum); the decode kernel then walks each
 * sequence's positions prefix_lens[s] .. L-1 and merges its pieces with the prefix partials by
 * the log-sum-exp rule.  A sequence with prefix_lens[s] >= L is decoded over its whole context.
 * Disagreements (a member's prefix length or blocks differ from the first member's, a prefix
 * not a multiple of block_size) set PA_DEVERR_PREFIX.  Caches bf16 or fp16 (otherwise
 * PA_ERR_UNSUPPORTED); head_dim, block_size and group sizes as for pa_prefill; out fp32 or the
 * caches' type.  workspace: device memory of at least pa_decode_shared_prefix_workspace_bytes
 * bytes, 256-byte aligned, zeroed before its first use (pa_workspace_init), or NULL for a
 * library-owned one (as for pa_decode).  The decode starts as a programmatic dependent of the
 * prefix pass; the prefix pass itself starts after the kernel before it on `stream`.
 */
PA_API int pa_decode_shared_prefix(const pa_tensor *out, const pa_tensor *query,
                                   const pa_tensor *key_cache, const pa_tensor *value_cache,
                                   const pa_tensor *block_tables, const pa_tensor *context_lens,
                                   const pa_tensor *group_start, const pa_tensor *prefix_lens,
                                   float scale, int32_t block_size, int32_t num_kv_heads,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace pa_decode_shared_prefix needs (0 on invalid arguments): the decode
 * workspace of pa_decode_ex plus the prefix pass's partial results for prefixes of up to
 * max_blocks_per_seq * block_size positions. */
PA_API size_t pa_decode_shared_prefix_workspace_bytes(int64_t num_seqs, int32_t num_heads,
                                                      int32_t num_kv_heads, int32_t head_dim,
                                                      int64_t max_blocks_per_seq,
                                                      int32_t block_size);

/*
 * Measurement aids (not part of the attention path).
 *
 * pa_set_decode_timeline - when buf is not NULL, every later launch of the tensor-core decode
 * kernel (pa_decode, pa_decode_ex, pa_decode_step, pa_decode_fp8, pa_decode_noalloc) writes, for
 * each worker warp w < bytes / 64, eight 64-bit words at buf + 64 w: the global nanosecond
 * timer when the warp starts, when its first tile has landed, when it has consumed its last
 * tile, when it is finished; the SM it ran on; the chunks in its share; the timer when its CTA
 * may read the caches (the previous grid, under PA_DECODE_OVERLAP_PREVIOUS, has finished); the
 * timer when its CTA's merge warp is finished.  buf: device memory, 8-byte aligned, kept by the
 * caller.  NULL stops the recording.  Launches that overlap on the GPU overwrite each other's
 * records.
 */
PA_API int pa_set_decode_timeline(void *buf, size_t bytes);

/*
 * pa_hbm_read_probe - read `bytes` of device memory once, as a read-only bandwidth probe (the
 * ceiling of a read stream such as decode, next to the copy bandwidth).  mode 0: 16-byte vector
 * loads from every SM; mode 1: 32 KB bulk asynchronous copies into shared memory (the copy
 * engine the decode kernels use; a tail shorter than 32 KB is not read).  buf: 128-byte aligned
 * device memory; sink: device memory of two 32-bit words, the first receives a fold of the
 * loaded words, the second gets bit 0 set if a copy did not complete within about a second.
 * Asynchronous on `stream`.
 */
PA_API int pa_hbm_read_probe(const void *buf, size_t bytes, int32_t mode, void *sink,
                             void *stream);

/* PA_VERSION of the library actually loaded. */
PA_API int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */

// pa_decode_mma.cuh - the tensor-core decode kernel for 16-bit caches (bf16 or fp16).
//
// Same work split, cursor and merge as the CUDA-core kernel (pa_decode_common.cuh); what
// changes is how a chunk of 16 key/value rows is consumed:
//   * Loads: each chunk's key and value tiles arrive by TMA tensor copies in the 128-byte
//     swizzled layout, one box per tile (the caches are described as 5-D tensors 64 elements x
//     block_size rows x head_dim/64 column halves x kv_heads x blocks, so a box holds 16 rows
//     (8 at block_size 8) of a whole head row); the block id of each box comes from the block
//     table, fetched a chunk ahead.  The swizzle makes every ldmatrix below free of
//     shared-memory bank conflicts.
//   * q.K: mma.sync m16n8k16 with the 16 tokens as M, the query heads of the GQA group as N
//     (padded to 8 with zeros) and head_dim as K; A comes from the key tile by ldmatrix, B (the
//     group's query rows) is loaded once per piece into registers.  Products of two 16-bit
//     values are exact in the fp32 accumulator; the scale is applied to the fp32 result, in the
//     same FFMA that subtracts the running maximum.
//   * softmax: base-2 logits, per-head chunk maxima over 8 lanes by shuffles, the running
//     maximum moved only when a chunk exceeds it by more than 2^8 (weights stay <= 256).
//   * P.V: mma.sync with head_dim as M (V tile read transposed by ldmatrix.trans), the tokens as
//     K and the heads as N.  P is split into two 16-bit terms (P = hi + lo, hi = round(P),
//     lo = round(P - hi)) so the weights keep about 16 significant bits: one 16-bit rounding of P
//     alone would cost ~2^-9 relative error per weight.  With at most 4 heads per kv head the lo
//     terms ride in the MMA's unused head columns (one MMA per V fragment for both terms).  P
//     reaches the B operand in registers: movmatrix.trans of each lane's packed C fragment.
// Warp specialization keeps the copies off the critical path: four worker warps per CTA
// consume chunks from their own rings, one producer warp issues all copies (see the kernel).
#pragma once

#include "pa_decode.cuh"

namespace pa {

template <typename T>
struct MmaType;
template <>
struct MmaType<__nv_bfloat16> {
  static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  // (x, y) -> packed hi and lo terms (hi = round(p), lo = round(p - hi): hi + lo keeps about 16
  // significant bits of p), x in the lower half of each
  static __device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
  }
  // (x, y) -> their packed hi terms (sel = 0) or lo terms (sel = 1), as split2 gives them
  static __device__ __forceinline__ uint32_t term2(float x, float y, float sel) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(-sel, hf.x, x), fmaf(-sel, hf.y, y));
    return *reinterpret_cast<const uint32_t *>(&r);
  }
  static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};
template <>
struct MmaType<__half> {
  static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(x, y);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
  }
  // (x, y) -> their packed hi terms (sel = 0) or lo terms (sel = 1), as split2 gives them
  static __device__ __forceinline__ uint32_t term2(float x, float y, float sel) {
    const __half2 h = __floats2half2_rn(x, y);
    const float2 hf = __half22float2(h);
    const __half2 r = __floats2half2_rn(fmaf(-sel, hf.x, x), fmaf(-sel, hf.y, y));
    return *reinterpret_cast<const uint32_t *>(&r);
  }
  static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};

// Four FP8 E4M3 values (bytes 0..3 of w) -> two f16x2: lo = (byte 0, byte 1), hi = (byte 2,
// byte 3), the lower byte in the lower half.  Exact: every E4M3 value is an f16.
__device__ __forceinline__ void fp8x4_to_f16x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Transpose of an 8x8 matrix of 16-bit values held by the warp (lane l: row l / 4, columns
// 2 (l % 4) and + 1, the lower column in the lower half) into the same layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// TMA tensor copy of one box of the 5-D cache view (row in block y, kv head z, block w) into
// shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap *map, int y, int z,
                                              int w, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(0), "r"(z), "r"(w),
      "r"(smem_u32(bar))
      : "memory");
}

// The same with an L2 cache policy (createpolicy): the decode streams every key and value tile
// once, so its copies are marked evict-first and leave L2 to what the launch reads again (the
// pieces' partial results, the block tables, the queries).
__device__ __forceinline__ void tma_load_tile_hint(uint32_t dst, const CUtensorMap *map, int y, int z,
                                                   int w, uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(0), "r"(z), "r"(w),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Prefetch one box of the 5-D cache view into L2 (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_tile(const CUtensorMap *map, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.prefetch.tensor.5d.L2.global.tile [%0, {%1, %2, %3, %4, %5}];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(0), "r"(y), "r"(0), "r"(z), "r"(w)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Non-blocking test of a barrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2  // stages per worker, 16-bit caches
#endif
#ifndef PA_EARLY_ISSUE
#define PA_EARLY_ISSUE 0  // issue the first stages before the previous grid has finished
#endif
#ifndef PA_FP8_MAX_STAGES
#define PA_FP8_MAX_STAGES 5  // most stages per worker, FP8 caches
#endif

// KVB: bytes per cache element (2: bf16/fp16, 1: FP8 E4M3).  The query is 16-bit either way.
template <int D, int BS, int G, int KVB = 2>
struct MmaTraits {
  static constexpr int kChunk = 16;                     // tokens per chunk (M of q.K)
  static constexpr int kHalves = D * KVB / 128;         // 128-byte column blocks of a row
  static constexpr int kBoxRows = BS < 16 ? BS : 16;    // rows per TMA box
  static constexpr int kCopies = 16 / kBoxRows;         // blocks touched per chunk
  static constexpr int kBoxBytes = kBoxRows * D * KVB;  // one box: [block][row][128 B]
  static constexpr int kTileBytes = 16 * D * KVB;       // key (or value) bytes of a chunk
  static constexpr int kQBytes = G * D * 2;
  // a fused decode step's new key and value rows of the chunk holding position L-1 (16-bit,
  // the query's type; quantised in shared memory for FP8 caches)
  static constexpr int kNewBytes = 2 * D * 2;
  static constexpr int kNewOff = 2 * kTileBytes + kQBytes;
  static constexpr int kStageBytes = 2 * kTileBytes + (kQBytes + kNewBytes + 1023) / 1024 * 1024;
  static constexpr int kWorkers = 4;                    // consumer warps
  static constexpr int kThreads = (kWorkers + 2) * 32;  // + one producer and one merge warp
  // Two stages per worker: one being computed, one in flight.  A third stage puts more bytes
  // in flight than HBM needs to run at full rate; the longer queues only raise the latency
  // every worker sees and widen the spread of finishing times (measured: the Llama-shaped
  // decode 60 -> 58 us, the long mixed batch 275 -> 259 us).
  // FP8 stages hold half the bytes, so a worker needs more of them for the same bytes in flight:
  // as many as keep two CTAs per SM (about 110 KB of shared memory each), at most kMaxFp8Stages.
  static constexpr int kMaxFp8Stages = PA_FP8_MAX_STAGES;
  static constexpr int kFp8Stages = (110 * 1024) / (kWorkers * kStageBytes) < kMaxFp8Stages
                                        ? (110 * 1024) / (kWorkers * kStageBytes)
                                        : kMaxFp8Stages;
  static constexpr int kStages = KVB == 2 ? PA_DECODE_STAGES : kFp8Stages;
  static constexpr int kRingBytes = kWorkers * kStages * kStageBytes;
  static constexpr int kMetaOff = 0;
  static constexpr int kFullOff = kStages * 32;
  static constexpr int kEmptyOff = kFullOff + kStages * 8;
  static constexpr int kSmallBytes = (kEmptyOff + kStages * 8 + 127) / 128 * 128;
  static constexpr int kShareOff = kRingBytes + kWorkers * kSmallBytes;
  static constexpr int kMboxEntries = 4;                // split pieces (at most 2) + done
  static constexpr int kMboxOff = kShareOff + kWorkers * 32 + 16;
  static constexpr int kMcountOff = kMboxOff + kWorkers * kMboxEntries * 32;
  static constexpr int kSmemBytes = kMcountOff + kWorkers * 4 + 1024;  // + 1 KB alignment
  static constexpr int kKSteps = D / 16;                // k-steps of q.K
  static constexpr int kMTiles = D / 16;                // m-tiles of P.V
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(D * KVB >= 128, "rows of at least one 128-byte swizzle span");
  static_assert(G <= 8, "at most 8 query heads per kv head");
};

// Shared-memory record of one worker's share, written by the worker for the producer.
struct ShareRecord {
  int s, rem, len, pad;
  long long g0, n;
};

// Mailbox entry from a worker to the merge warp: a split piece whose (o, m, l) are stored, or,
// with npieces == 0, the worker's last message.
struct MailEntry {
  PieceInfo p;
  int pad[3];
};
static_assert(sizeof(MailEntry) == 32, "mailbox entries are 32 bytes");

__device__ __forceinline__ void st_release_cta(unsigned int *p, unsigned int v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned int ld_acquire_cta(const unsigned int *p) {
  unsigned int v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Worker side: hand entry `idx` of this worker's mailbox to the merge warp.  The piece's global
// stores by all lanes are ordered before the release that publishes the entry.
__device__ __forceinline__ void mail_post(MailEntry *box, unsigned int *count, int idx,
                                          const PieceInfo &p, int lane) {
  __threadfence_block();
  __syncwarp();
  if (lane == 0) {
    box[idx].p = p;
    st_release_cta(count, (unsigned int)(idx + 1));
  }
  __syncwarp();
}

// Offset in a tile of row r (0..15), column half h: boxes of kBoxRows rows, each [half][row].
template <typename Tr>
__device__ __forceinline__ uint32_t tile_offset(int r, int h) {
  return (r / Tr::kBoxRows) * Tr::kBoxBytes + h * (Tr::kBoxRows * 128) + (r % Tr::kBoxRows) * 128;
}

// Warp specialization: warps 0..3 are workers (each consumes its own share of the chunk list
// from its own ring of stages), warp 4 is the producer: its lane k walks worker k's share and
// issues that worker's copies (one TMA box per key tile and per value tile, plus the query rows
// when a new (sequence, kv head) starts) as soon as the worker releases a stage.  The workers
// never issue copies, so TMA issue latency stays off their critical path.
// T: the query's element type (and the MMA's, for 16-bit caches).  KV: the caches' element
// type; with FP8 E4M3 caches the tiles are widened to f16 in registers and the MMAs run in f16.
template <typename T, int D, int BS, int G, typename KV = T>
__global__ void __launch_bounds__(MmaTraits<D, BS, G, (int)sizeof(KV)>::kThreads, 2)
    paged_decode_mma_kernel(const DecodeArgs a, const __grid_constant__ TmaMaps maps) {
  constexpr bool kFp8 = sizeof(KV) == 1;
  using Tr = MmaTraits<D, BS, G, (int)sizeof(KV)>;
  using M = MmaType<typename std::conditional<kFp8, __half, T>::type>;
  constexpr int ST = Tr::kStages;
  constexpr int NW = Tr::kWorkers;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 128-byte swizzled boxes must start on 1 KB boundaries
  unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int max_len = a.max_blocks * BS;
  ShareRecord *shares = reinterpret_cast<ShareRecord *>(smem + Tr::kShareOff);
  MailEntry *mbox = reinterpret_cast<MailEntry *>(smem + Tr::kMboxOff);
  unsigned int *mcount = reinterpret_cast<unsigned int *>(smem + Tr::kMcountOff);
  long long *step_T = reinterpret_cast<long long *>(smem + Tr::kShareOff + NW * 32);
  int *step_W = reinterpret_cast<int *>(smem + Tr::kShareOff + NW * 32 + 8);

  // ---- set-up: barriers, then every worker finds its share and publishes it ----
  if (wid < NW) {
    unsigned char *small = smem + Tr::kRingBytes + wid * Tr::kSmallBytes;
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < ST; ++i) {
        mbar_init(reinterpret_cast<uint64_t *>(small + Tr::kFullOff) + i, 1);
        mbar_init(reinterpret_cast<uint64_t *>(small + Tr::kEmptyOff) + i, 1);
      }
      fence_barrier_init();
    }
    WarpShare ws;
    ws.n = 0;
    const bool has = split_prologue<16, NW, G, D, BS, false>(a, max_len, ws);
    if (lane == 0) {
      ShareRecord r;
      r.s = has ? ws.s : -1;
      r.rem = has ? ws.rem : 0;
      r.len = has ? ws.len : 0;
      r.pad = 0;
      r.g0 = has ? ws.g0 : 0;
      r.n = has ? ws.n : 0;
      shares[wid] = r;
      mcount[wid] = 0u;
      if (wid == 0) {
        *step_T = ws.T;
        *step_W = ws.W;
      }
    }
  } else if (wid == NW && lane == 0) {
    // bring the two descriptors into the TMA unit while the workers run their prologue
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.v)) : "memory");
  }
  __syncthreads();

  if (wid == NW) {
    // ================================ producer ================================
    const int k = lane;  // the worker this lane feeds
    bool active = false;
    ChunkCursor<16, BS, Tr::kCopies, Tr::kBoxRows> cur;
    unsigned char *ring = smem + k * ST * Tr::kStageBytes;
    unsigned char *small = smem + Tr::kRingBytes + k * Tr::kSmallBytes;
    ChunkMeta *meta = reinterpret_cast<ChunkMeta *>(small + Tr::kMetaOff);
    uint64_t *full = reinterpret_cast<uint64_t *>(small + Tr::kFullOff);
    uint64_t *empty = reinterpret_cast<uint64_t *>(small + Tr::kEmptyOff);
    if (k < NW) {
      const ShareRecord r = shares[k];
      if (r.n > 0 && r.s >= 0) {
        WarpShare ws;
        ws.T = *step_T;
        ws.alpha = a.piece_cost;
        ws.W = *step_W;
        ws.g0 = r.g0;
        ws.n = r.n;
        ws.s = r.s;
        ws.rem = r.rem;
        ws.len = r.len;
        cur.init(a, ws, max_len);
        active = true;
        // Warm L2 with the first chunk while the previous grid may still run: L2 is the point
        // of coherence, so a line that grid writes afterwards is read fresh by the copies below.
#pragma unroll
        for (int c = 0; c < Tr::kCopies; ++c) {
          const int t = cur.i * 16 + c * Tr::kBoxRows;
          const int blk = cur.blk[c];
          if (t < cur.len && blk >= 0 && (long long)blk < a.num_blocks) {
            tma_prefetch_tile(&maps.k, t % BS, cur.kvh, blk);
            tma_prefetch_tile(&maps.v, t % BS, cur.kvh, blk);
          }
        }
      }
    }
    const uint64_t stream_policy = l2_evict_first_policy();
    // One stage of this lane's worker: the chunk's key and value boxes, plus the group's query
    // rows when a new (sequence, kv head) starts, all counted on the stage's full barrier.
    auto issue = [&](int slot) {
      // fused step: the chunk holding position L-1 also brings that position's new rows
      const bool new_row = a.fused && cur.i == cur.nch - 1;
      const int f = cur.flags() | (new_row ? kNewRow : 0);
      unsigned char *stage = ring + slot * Tr::kStageBytes;
      meta[slot] = cur.meta(f);
      const uint32_t bytes = 2u * cur.valid_copies() * Tr::kBoxBytes +
                             ((f & kFirst) ? (uint32_t)Tr::kQBytes : 0u) +
                             (new_row ? (uint32_t)(2 * D * 2) : 0u) +
                             ((cur.issued == 0 && test_stalls(a, blockIdx.x * NW + k)) ? 16u : 0u);
      mbar_arrive_expect_tx(full + slot, bytes);
#pragma unroll
      for (int c = 0; c < Tr::kCopies; ++c) {
        const int t = cur.i * 16 + c * Tr::kBoxRows;
        if (t < cur.len) {
          int blk = cur.blk[c];
          if (blk < 0 || (long long)blk >= a.num_blocks) {
            set_error(a.err, PA_DEVERR_BLOCK_ID);
            blk = 0;
          }
          const uint32_t off = c * Tr::kBoxBytes;
          tma_load_tile_hint(smem_u32(stage + off), &maps.k, t % BS, cur.kvh, blk, full + slot,
                             stream_policy);
          tma_load_tile_hint(smem_u32(stage + Tr::kTileBytes + off), &maps.v, t % BS, cur.kvh, blk,
                             full + slot, stream_policy);
        }
      }
      if (new_row) {
        bulk_copy_g2s(stage + Tr::kNewOff,
                      a.step.key + (long long)cur.s * a.step.k_tok + (long long)cur.kvh * a.step.k_head,
                      D * 2, full + slot);
        bulk_copy_g2s(stage + Tr::kNewOff + D * 2,
                      a.step.value + (long long)cur.s * a.step.v_tok + (long long)cur.kvh * a.step.v_head,
                      D * 2, full + slot);
      }
      if (f & kFirst) {
        const char *q = static_cast<const char *>(a.query) +
                        ((long long)cur.s * a.q_s + (long long)cur.kvh * G * a.q_h) * 2;
        if (a.q_heads_contiguous) {
          bulk_copy_g2s(stage + 2 * Tr::kTileBytes, q, Tr::kQBytes, full + slot);
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h)
            bulk_copy_g2s(stage + 2 * Tr::kTileBytes + h * D * 2, q + (long long)h * a.q_h * 2,
                          D * 2, full + slot);
        }
      }
      cur.advance(a);
      if (cur.issued >= cur.n) active = false;
    };
#if PA_EARLY_ISSUE
    // The first stages of chunks that end before the sequence's last position: the grid before
    // this one writes only that position of each sequence (the step's new token).
    while (active && cur.issued < ST && (cur.i + 1) * 16 < cur.len) issue((int)(cur.issued % ST));
#endif
    // A grid launched after this one (the separate merge) may start now and wait for us.
    if (lane == 0) allow_next_grid();
    // Everything above read only context_lens and block_tables; the caches and the query may
    // still be written by the previous grid when this one was launched to overlap it (not when
    // that grid is the shared-prefix pass: see prefix_overlap).
    if (!a.prefix_overlap) wait_for_previous_grid();
    if (a.timeline != nullptr && k < NW && blockIdx.x * NW + k < a.timeline_warps)
      a.timeline[(long long)(blockIdx.x * NW + k) * kTimelineWords + kTlIssue] = global_ns();
    long long last_progress = clock64();
    while (__any_sync(FULL_MASK, active)) {
      bool can = false;
      int slot = 0;
      if (active) {
        slot = (int)(cur.issued % ST);
        can = cur.issued < ST ||
              mbar_test(empty + slot, (uint32_t)(((cur.issued / ST) - 1) & 1));
      }
      if (can) issue(slot);
      if (__any_sync(FULL_MASK, can)) {
        last_progress = clock64();
      } else {
        if (clock64() - last_progress > a.wait_cycles) {
          // a worker stopped releasing stages: give up (the worker reports its own timeout)
          if (active) set_error(a.err, PA_DEVERR_TIMEOUT);
          break;
        }
        __nanosleep(64);
      }
    }
    if (a.prefix_overlap) wait_for_previous_grid();  // this grid completes after the prefix pass
    return;
  }

  if (wid == NW + 1) {
    // ================================ merge warp ================================
    // First, once the grid before this one (when it was launched to overlap it) has finished:
    // the out rows of empty contexts are zeroed, and in a fused decode step this grid's share
    // of the step's cache write is done.  The shared-prefix pass writes neither.
    if (!a.prefix_overlap || a.fused) wait_for_previous_grid();
    {
      const int launched_lanes = gridDim.x * 32;
      const int out_elt = a.out_dtype == PA_F32 ? 4 : 2;
      for (int s = blockIdx.x * 32 + lane; s < a.num_seqs; s += launched_lanes)
        if (clamp_len(__ldg(a.context_lens + s), max_len) == 0)
          zero_rows<D>(static_cast<char *>(a.out) + (long long)s * a.out_s * out_elt, a.out_h,
                       a.out_dtype, a.num_kv_heads * G);
      if (a.fused) {
        if constexpr (kFp8)
          fused_cache_write_fp8<T, BS>(a, max_len, blockIdx.x * 32 + lane, launched_lanes);
        else
          fused_cache_write<BS>(a, max_len, blockIdx.x * 32 + lane, launched_lanes);
      }
    }
    // Lane k follows worker k's mailbox.  For each split piece the warp makes the piece's
    // stores visible GPU-wide, takes the ticket of its (sequence, kv head) and, when the piece
    // is the last one there, merges all of them; the workers never stall on a GPU-wide fence.
    int seen = 0;
    bool fin = lane >= NW;
    long long last_progress = clock64();
    while (true) {
      const unsigned int cnt = fin ? 0u : ld_acquire_cta(mcount + lane);
      const unsigned int ready = __ballot_sync(FULL_MASK, !fin && (unsigned int)seen < cnt);
      if (ready == 0u) {
        if (__all_sync(FULL_MASK, fin)) break;
        if (clock64() - last_progress > a.wait_cycles) {
          if (!fin) set_error(a.err, PA_DEVERR_TIMEOUT);
          break;
        }
        __nanosleep(128);
        continue;
      }
      __syncwarp();
      last_progress = clock64();
      for (unsigned int r = ready; r != 0u; r &= r - 1u) {
        const int k = __ffs(r) - 1;
        const int idx = __shfl_sync(FULL_MASK, seen, k);
        const PieceInfo p = mbox[k * Tr::kMboxEntries + idx].p;
        if (p.npieces == 0) {
          if (lane == k) fin = true;
        } else {
          if (!PA_TICKET_ACQREL) __threadfence();
          __syncwarp();
          take_ticket<G, D, BS>(a, p, lane);
        }
        if (lane == k) ++seen;
      }
    }
    if (a.timeline != nullptr && lane < NW && blockIdx.x * NW + lane < a.timeline_warps)
      a.timeline[(long long)(blockIdx.x * NW + lane) * kTimelineWords + kTlMerged] = global_ns();
    return;
  }

  // ================================ workers ================================
  const ShareRecord share = shares[wid];
  MailEntry *box = mbox + wid * Tr::kMboxEntries;
  int posted = 0;
  PieceInfo done_msg;
  done_msg.pair = done_msg.first_worker = done_msg.npieces = done_msg.s = done_msg.kvh = 0;
  ChunkMeta last_piece = {};  // the share's last piece when it is split (npieces > 0)
  const int gw = blockIdx.x * NW + wid;
  // measurement aid: this warp's timeline record, or null
  unsigned long long *tl = (a.timeline != nullptr && lane == 0 && gw < a.timeline_warps)
                               ? a.timeline + (long long)gw * kTimelineWords
                               : nullptr;
  if (tl) {
    tl[kTlStart] = global_ns();
    tl[kTlSm] = sm_id();
    tl[kTlChunks] = (share.n > 0 && share.s >= 0) ? (unsigned long long)share.n : 0ull;
  }
  if (share.n <= 0 || share.s < 0) {
    mail_post(box, mcount + wid, 0, done_msg, lane);
    if (tl) tl[kTlFirst] = tl[kTlLast] = tl[kTlDone] = global_ns();
    return;
  }
  const long long n = share.n;
  const int ni = (int)n;  // below 2^31: the host bounds a step's chunks
  unsigned char *ring = smem + wid * ST * Tr::kStageBytes;
  unsigned char *small = smem + Tr::kRingBytes + wid * Tr::kSmallBytes;
  const ChunkMeta *meta = reinterpret_cast<const ChunkMeta *>(small + Tr::kMetaOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(small + Tr::kFullOff);
  uint64_t *empty = reinterpret_cast<uint64_t *>(small + Tr::kEmptyOff);

  const int g = lane >> 2;  // fragment row group
  const int c = lane & 3;   // fragment column pair
  const int h0 = 2 * c, h1 = 2 * c + 1;  // heads of this lane's logits / output columns
  // With G <= 4 the MMAs' 8 head columns have room for P's lo term: column n of P carries the
  // hi term of head n for n < 4 and the lo term of head n - 4 for n >= 4, so one P.V MMA per V
  // fragment does both terms.  The query columns follow (column n holds head n % 4, zero past
  // G): lanes c and c + 2 compute the same logits, and the two halves of O are added where a
  // piece ends.
  constexpr bool kPackLo = G <= 4;
  const int qh = kPackLo ? (g & 3) : g;     // query head of MMA column g
  const float lo_sel = (kPackLo && c >= 2) ? 1.f : 0.f;  // this lane's columns hold lo terms
  const int lm = lane >> 3;  // which 8x8 matrix this lane addresses for ldmatrix
  const int lr = lane & 7;   // row within it
  uint32_t qb[Tr::kKSteps][2];
  float o[Tr::kMTiles][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool piece_at_start = false;  // this piece begins at chunk 0 of its (sequence, kv head)
  // logit scale of this lane's two heads (base 2) and the output scale (FP8 value scale)
  float sc0 = a.scale_log2, sc1 = a.scale_log2, vsc = 1.f;

  int slot = 0;         // cc % ST
  uint32_t parity = 0;  // (cc / ST) & 1
  for (int cc = 0; cc < ni; ++cc) {
    // (one verdict for the whole warp: the paths below are warp-synchronous)
    if (!__all_sync(FULL_MASK, mbar_wait_bounded(full + slot, parity, a.wait_cycles))) {
      // a copy never completed: record it, let the copies that may be in flight land, stop.
      if (lane == 0) set_error(a.err, PA_DEVERR_TIMEOUT);
      for (long long j = cc; j < cc + ST && j < n; ++j)
        mbar_wait_bounded(full + (int)(j % ST), (uint32_t)((j / ST) & 1), a.wait_cycles);
      mail_post(box, mcount + wid, posted, done_msg, lane);
      return;
    }
    if (tl && cc == 0) tl[kTlFirst] = global_ns();
    const ChunkMeta m = meta[slot];
    unsigned char *stage = ring + slot * Tr::kStageBytes;
    if constexpr (kFp8) {
      if (m.flags & kNewRow) {
        // fused step over FP8 caches: the new token's 16-bit rows quantised as the cache write
        // quantises them (fp8_codes8), into row (L-1) % 16 of the FP8 tiles: lane l takes
        // elements 8 (l % 16) .. + 7 of the key (l < 16) or value row, which land in half
        // l % 2 of 16-byte piece (l % 16) / 2 of the swizzled row
        static_assert(D == 128, "FP8 rows of one 128-byte span");
        const int r = (m.len - 1) & 15;
        const int which = lane >> 4, j = lane & 15;
        float f[8];
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(stage + Tr::kNewOff + which * D * 2 + j * 16), f);
        const uint2 codes = fp8_codes8(f, __ldg((which ? a.v_scale : a.k_scale) + m.kvh));
        *reinterpret_cast<uint2 *>(stage + which * Tr::kTileBytes + tile_offset<Tr>(r, 0) +
                                   ((((j >> 1) ^ (r & 7)) << 4) | ((j & 1) << 3))) = codes;
        fence_proxy_async_smem();  // before the stage is copied into again
        __syncwarp();
      }
    } else {
      if (m.flags & kNewRow) {
        // fused step: position L-1 is this step's new token, read from the step's key and
        // value rather than the cache (which this kernel writes concurrently); put its rows into
        // the tiles at row (L-1) % 16, in the tiles' swizzled layout
        constexpr int kPieces = D * 2 / 16;  // 16-byte pieces of a row
        const int r = (m.len - 1) & 15;
        if (lane < 2 * kPieces) {
          const int which = lane / kPieces, c = lane % kPieces;
          const uint4 v = *reinterpret_cast<const uint4 *>(stage + Tr::kNewOff + which * D * 2 + c * 16);
          *reinterpret_cast<uint4 *>(stage + which * Tr::kTileBytes + tile_offset<Tr>(r, c / 8) +
                                     (((c % 8) ^ (r & 7)) << 4)) = v;
          fence_proxy_async_smem();  // before the stage is copied into again
        }
        __syncwarp();
      }
    }
    const uint32_t kbase = smem_u32(stage);
    const uint32_t vbase = kbase + Tr::kTileBytes;
    if (m.flags & kFirst) {
      const unsigned char *qs = stage + 2 * Tr::kTileBytes;
      if constexpr (kFp8) {
        // f16 B fragments in the dim order of the FP8 key fragments below (k-step ks holds the
        // dims 32(ks/2) + 16(ks%2) + 4c + {0,1 | 2,3}), each head scaled by a power of two
        // alpha that keeps |q * alpha| < 2^15; 1/alpha goes into that head's logit scale.
        const T *q = reinterpret_cast<const T *>(qs);
        float qv[Tr::kKSteps][4];
        float mx = 0.f;
#pragma unroll
        for (int ks = 0; ks < Tr::kKSteps; ++ks) {
          const int base = 32 * (ks >> 1) + 16 * (ks & 1) + 4 * c;
          // the 4 dims in one 8-byte load
          const uint2 u = qh < G ? *reinterpret_cast<const uint2 *>(q + qh * D + base) : make_uint2(0u, 0u);
          const T *e4 = reinterpret_cast<const T *>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qv[ks][e] = Elem<T>::to_float(e4[e]);
            mx = fmaxf(mx, fabsf(qv[ks][e]));
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, 2));
        // biased exponent of mx (0 for zero or subnormal), alpha = 2^(14 - unbiased)
        const int be = (int)((__float_as_uint(mx) >> 23) & 0xffu);
        const int ae = min(253, max(1, 127 + 14 - (be == 0 ? -126 : be - 127)));
        const float alpha = __uint_as_float((uint32_t)ae << 23);
        const float inv_alpha = __uint_as_float((uint32_t)(254 - ae) << 23);
#pragma unroll
        for (int ks = 0; ks < Tr::kKSteps; ++ks) {
          const float2 al = make_float2(alpha, alpha);
          const __half2 lo = __float22half2_rn(__fmul2_rn(make_float2(qv[ks][0], qv[ks][1]), al));
          const __half2 hi = __float22half2_rn(__fmul2_rn(make_float2(qv[ks][2], qv[ks][3]), al));
          qb[ks][0] = *reinterpret_cast<const uint32_t *>(&lo);
          qb[ks][1] = *reinterpret_cast<const uint32_t *>(&hi);
        }
        const float ks_ = a.scale_log2 * __ldg(a.k_scale + m.kvh);
        sc0 = ks_ * __shfl_sync(FULL_MASK, inv_alpha, 4 * h0);
        sc1 = ks_ * __shfl_sync(FULL_MASK, inv_alpha, 4 * h1);
        vsc = __ldg(a.v_scale + m.kvh);
      } else {
#pragma unroll
        for (int ks = 0; ks < Tr::kKSteps; ++ks) {
          if (qh < G) {
            qb[ks][0] = *reinterpret_cast<const uint32_t *>(qs + (qh * D + 16 * ks + 2 * c) * 2);
            qb[ks][1] = *reinterpret_cast<const uint32_t *>(qs + (qh * D + 16 * ks + 8 + 2 * c) * 2);
          } else {
            qb[ks][0] = 0u;
            qb[ks][1] = 0u;
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < Tr::kMTiles; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      piece_at_start = (m.flags & kPairStart) != 0;
    }

    // ---- q.K on tensor cores: s = S[token g | g+8][head 2c | 2c+1] ----
    float s[4];
    {
      // 16-bit caches: two accumulators (even / odd k-steps) halve the chain of dependent mma
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      const int row = ((lm & 1) << 3) | lr;
      if constexpr (kFp8) {
        // One ldmatrix per 32 dims (two k-steps): matrix j holds tokens 8(j&1).. of the 16-byte
        // chunk 2*s2 + (j>>1); each lane gets 4 consecutive dims of one token and widens them
        // to (a0 | a2) or (a1 | a3) of the m16n8k16 A fragment.  One accumulator: the widening
        // spaces the MMAs out, and a second chain would cost four adds per chunk (measured
        // 36.1 -> 35.8 us for the Llama-shaped FP8 step with one chain).
#pragma unroll
        for (int s2 = 0; s2 < D / 32; ++s2) {
          const int c16 = 2 * s2 + (lm >> 1);
          const uint32_t addr = kbase + tile_offset<Tr>(row, 0) + ((c16 ^ lr) << 4);
          uint32_t r[4], af[4];
          ldmatrix_x4(r, addr);
          fp8x4_to_f16x2(r[0], af[0], af[2]);
          fp8x4_to_f16x2(r[1], af[1], af[3]);
          M::mma(sa, af, qb[2 * s2][0], qb[2 * s2][1]);
          fp8x4_to_f16x2(r[2], af[0], af[2]);
          fp8x4_to_f16x2(r[3], af[1], af[3]);
          M::mma(sa, af, qb[2 * s2 + 1][0], qb[2 * s2 + 1][1]);
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < Tr::kKSteps; ++ks) {
          const int c16 = ((ks & 3) << 1) | (lm >> 1);
          const uint32_t addr = kbase + tile_offset<Tr>(row, ks >> 2) + ((c16 ^ lr) << 4);
          uint32_t af[4];
          ldmatrix_x4(af, addr);
          if (ks & 1)
            M::mma(sb, af, qb[ks][0], qb[ks][1]);
          else
            M::mma(sa, af, qb[ks][0], qb[ks][1]);
        }
      }
      // logits before their scale
#pragma unroll
      for (int i = 0; i < 4; ++i) s[i] = kFp8 ? sa[i] : sa[i] + sb[i];
    }
    const int tok0 = m.chunk * 16;
    const bool tail = tok0 + 16 > m.len;
    if (tail) {
      if (tok0 + g >= m.len) s[0] = s[1] = -INFINITY;
      if (tok0 + g + 8 >= m.len) s[2] = s[3] = -INFINITY;
    }

    // ---- online softmax in base 2: t = logit * scale - m is the exponent of a weight against
    // the reference maximum m, which moves only when some t passes 8 (m = -inf, a piece's start,
    // gives t = +inf); only then are the chunk maxima gathered across lanes ----
    float t[4] = {fmaf(s[0], sc0, -m0), fmaf(s[1], sc1, -m1), fmaf(s[2], sc0, -m0),
                  fmaf(s[3], sc1, -m1)};
    if (__any_sync(FULL_MASK, fmaxf(t[0], t[2]) > 8.f || fmaxf(t[1], t[3]) > 8.f)) {
      float cm0 = fmaxf(s[0] * sc0, s[2] * sc0), cm1 = fmaxf(s[1] * sc1, s[3] * sc1);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        cm0 = fmaxf(cm0, __shfl_xor_sync(FULL_MASK, cm0, off));
        cm1 = fmaxf(cm1, __shfl_xor_sync(FULL_MASK, cm1, off));
      }
      const float n0 = fmaxf(m0, cm0), n1 = fmaxf(m1, cm1);
      const float a0 = fast_exp2(m0 - n0), a1 = fast_exp2(m1 - n1);
      m0 = n0;
      m1 = n1;
      l0 *= a0;
      l1 *= a1;
#pragma unroll
      for (int mt = 0; mt < Tr::kMTiles; ++mt) {
        o[mt][0] *= a0;
        o[mt][1] *= a1;
        o[mt][2] *= a0;
        o[mt][3] *= a1;
      }
      t[0] = fmaf(s[0], sc0, -m0);
      t[1] = fmaf(s[1], sc1, -m1);
      t[2] = fmaf(s[2], sc0, -m0);
      t[3] = fmaf(s[3], sc1, -m1);
    }
    const float p0 = fast_exp2(t[0]), p1 = fast_exp2(t[1]);
    const float p2 = fast_exp2(t[2]), p3 = fast_exp2(t[3]);
    l0 += p0 + p2;
    l1 += p1 + p3;
    // P as the B operand of P.V, in registers: each lane packs its two columns of token rows g
    // and g + 8 (a C fragment), and movmatrix transposes each 8x8 block into the B fragment
    // (tokens 2c, 2c+1 | 2c+8, 2c+9 of column g)
    uint32_t pf[4];  // hi (tokens 0-7, 8-15), lo (tokens 0-7, 8-15); with kPackLo pf[0..1] only
    if constexpr (kPackLo) {
      pf[0] = movmatrix_trans(M::term2(p0, p1, lo_sel));
      pf[1] = movmatrix_trans(M::term2(p2, p3, lo_sel));
    } else {
      uint32_t h01, l01, h23, l23;
      M::split2(p0, p1, h01, l01);
      M::split2(p2, p3, h23, l23);
      pf[0] = movmatrix_trans(h01);
      pf[1] = movmatrix_trans(h23);
      pf[2] = movmatrix_trans(l01);
      pf[3] = movmatrix_trans(l23);
    }

    // ---- P.V on tensor cores: o[mt] = O^T[dim 16mt+g | +8][head 2c | 2c+1] (FP8 caches:
    // dims 16mt+2g | 16mt+2g+1).  Value rows past the context may hold anything (NaN included)
    // and are zeroed: only a sequence's last chunk has such rows, so that case has its own copy
    // of the loop and the others carry no masking ----
    auto pv = [&](auto masked) {
      constexpr bool kMasked = decltype(masked)::value;
      // tokens 2c, 2c+1 (the halves of vf[0], vf[1]) and 2c+8, 2c+9 (vf[2], vf[3])
      uint32_t m01 = 0xffffffffu, m89 = 0xffffffffu;
      if constexpr (kMasked) {
        m01 = (tok0 + 2 * c >= m.len ? 0u : 0x0000ffffu) | (tok0 + 2 * c + 1 >= m.len ? 0u : 0xffff0000u);
        m89 = (tok0 + 2 * c + 8 >= m.len ? 0u : 0x0000ffffu) | (tok0 + 2 * c + 9 >= m.len ? 0u : 0xffff0000u);
      }
      if constexpr (kFp8) {
        // ldmatrix.trans of 16-bit pairs: matrix j (tokens 8(j&1).., 16-byte chunk 2mp + (j>>1))
        // gives each lane tokens 2c, 2c+1 of dims 2g, 2g+1; a byte permute regroups them by dim
        // (one register per dim, the two tokens as its halves) before widening to f16.
        const int row = ((lm & 1) << 3) | lr;
#pragma unroll
        for (int mp = 0; mp < D / 32; ++mp) {
          const int c16 = 2 * mp + (lm >> 1);
          const uint32_t addr = vbase + tile_offset<Tr>(row, 0) + ((c16 ^ lr) << 4);
          uint32_t r[4];
          ldmatrix_x4_trans(r, addr);
#pragma unroll
          for (int t2 = 0; t2 < 2; ++t2) {
            uint32_t vf[4];
            fp8x4_to_f16x2(__byte_perm(r[2 * t2], 0u, 0x3120u), vf[0], vf[1]);
            fp8x4_to_f16x2(__byte_perm(r[2 * t2 + 1], 0u, 0x3120u), vf[2], vf[3]);
            if constexpr (kMasked) {
              vf[0] &= m01;
              vf[1] &= m01;
              vf[2] &= m89;
              vf[3] &= m89;
            }
            M::mma(o[2 * mp + t2], vf, pf[0], pf[1]);
            if constexpr (!kPackLo) M::mma(o[2 * mp + t2], vf, pf[2], pf[3]);
          }
        }
      } else {
        const int row = ((lm >> 1) << 3) | lr;  // token row of the V tile
#pragma unroll
        for (int mt = 0; mt < Tr::kMTiles; ++mt) {
          const int c16g = (mt << 1) | (lm & 1);
          const uint32_t addr = vbase + tile_offset<Tr>(row, c16g >> 3) + (((c16g & 7) ^ lr) << 4);
          uint32_t vf[4];
          ldmatrix_x4_trans(vf, addr);
          if constexpr (kMasked) {
            vf[0] &= m01;
            vf[1] &= m01;
            vf[2] &= m89;
            vf[3] &= m89;
          }
          M::mma(o[mt], vf, pf[0], pf[1]);
          if constexpr (!kPackLo) M::mma(o[mt], vf, pf[2], pf[3]);
        }
      }
    };
    if (tail)
      pv(std::true_type{});
    else
      pv(std::false_type{});
    // the stage is no longer needed: hand it back to the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + slot);
    if (tl && cc == ni - 1) tl[kTlLast] = global_ns();

    // ---- end of a piece ----
    if (m.flags & kLast) {
      if constexpr (kPackLo) {
        // lane c (c < 2) adds lane c + 2's lo columns to its hi ones
#pragma unroll
        for (int mt = 0; mt < Tr::kMTiles; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[mt][e] += __shfl_xor_sync(FULL_MASK, o[mt][e], 2);
      }
      float t0 = l0, t1 = l1;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        t0 += __shfl_xor_sync(FULL_MASK, t0, off);
        t1 += __shfl_xor_sync(FULL_MASK, t1, off);
      }
      float inv0 = 1.f / t0, inv1 = 1.f / t1;
      if constexpr (kFp8) {
        inv0 *= vsc;
        inv1 *= vsc;
      }
      if (a.separate_reduce && piece_at_start && lane == 0)
        a.pair_meta[m.pair] = make_int2(m.first_worker, m.npieces);
      // a (sequence, kv head) inside one share is written directly, unless it has partial
      // results of a shared prefix to merge with
      if (m.npieces == 1 && (a.prefix_lens == nullptr || prefix_pieces<BS>(a, m.s, max_len) == 0)) {
        const int out_elt = a.out_dtype == PA_F32 ? 4 : 2;
        char *row0 = static_cast<char *>(a.out) +
                     ((long long)m.s * a.out_s + (long long)(m.kvh * G + h0) * a.out_h) * out_elt;
        char *row1 = row0 + (long long)a.out_h * out_elt;
        // dims d0, d1 of one output row: adjacent with FP8 caches (one 8- or 4-byte store)
        auto put = [&](char *row, int d0, int d1, float x, float y) {
          if (a.out_dtype == PA_F32) {
            float *r = reinterpret_cast<float *>(row);
            if constexpr (kFp8) {
              *reinterpret_cast<float2 *>(r + d0) = make_float2(x, y);
            } else {
              r[d0] = x;
              r[d1] = y;
            }
          } else if (a.out_dtype == PA_BF16) {
            __nv_bfloat16 *r = reinterpret_cast<__nv_bfloat16 *>(row);
            if constexpr (kFp8) {
              *reinterpret_cast<__nv_bfloat162 *>(r + d0) = __floats2bfloat162_rn(x, y);
            } else {
              r[d0] = __float2bfloat16_rn(x);
              r[d1] = __float2bfloat16_rn(y);
            }
          } else {
            __half *r = reinterpret_cast<__half *>(row);
            if constexpr (kFp8) {
              *reinterpret_cast<__half2 *>(r + d0) = __floats2half2_rn(x, y);
            } else {
              r[d0] = __float2half_rn(x);
              r[d1] = __float2half_rn(y);
            }
          }
        };
#pragma unroll
        for (int mt = 0; mt < Tr::kMTiles; ++mt) {
          const int d0 = kFp8 ? 16 * mt + 2 * g : 16 * mt + g, d1 = kFp8 ? d0 + 1 : d0 + 8;
          if (h0 < G) put(row0, d0, d1, o[mt][0] * inv0, o[mt][2] * inv0);
          if (h1 < G) put(row1, d0, d1, o[mt][1] * inv1, o[mt][3] * inv1);
        }
      } else {
        const long long seg = (long long)m.pair + gw;
        float *o0 = a.part_o + (seg * G + h0) * D;
        float2 *ml0 = reinterpret_cast<float2 *>(a.part_ml) + seg * G + h0;
        float *o1 = o0 + D;
#pragma unroll
        for (int mt = 0; mt < Tr::kMTiles; ++mt) {
          const int d0 = kFp8 ? 16 * mt + 2 * g : 16 * mt + g, d1 = kFp8 ? d0 + 1 : d0 + 8;
          if constexpr (kFp8) {
            if (h0 < G) *reinterpret_cast<float2 *>(o0 + d0) = make_float2(o[mt][0] * inv0, o[mt][2] * inv0);
            if (h1 < G) *reinterpret_cast<float2 *>(o1 + d0) = make_float2(o[mt][1] * inv1, o[mt][3] * inv1);
          } else {
            if (h0 < G) {
              o0[d0] = o[mt][0] * inv0;
              o0[d1] = o[mt][2] * inv0;
            }
            if (h1 < G) {
              o1[d0] = o[mt][1] * inv1;
              o1[d1] = o[mt][3] * inv1;
            }
          }
        }
        if (g == 0) {
          if (h0 < G) ml0[0] = make_float2(m0, t0);
          if (h1 < G) ml0[1] = make_float2(m1, t1);
        }
        if (!a.separate_reduce) {
          PieceInfo p;
          p.pair = m.pair;
          p.first_worker = m.first_worker;
          p.npieces = m.npieces;
          p.s = m.s;
          p.kvh = m.kvh;
          if (cc == ni - 1) {
            // the share's last piece: published after the loop (nothing is left to overlap it
            // with), by this warp, so the four workers publish their last pieces in parallel
            // rather than through one merge warp
            last_piece = m;
          } else if (posted < Tr::kMboxEntries - 1) {
            // a piece that ends inside the share: the merge warp publishes it while this warp
            // goes on with its next piece
            mail_post(box, mcount + wid, posted, p, lane);
            ++posted;
          } else {
            finish_piece<G, D, BS, 1>(a, m, lane);  // mailbox full (rare): small merge rounds
          }
        }
      }
    }
    if (++slot == ST) {
      slot = 0;
      parity ^= 1u;
    }
  }
  // the loop's registers are free here: the merge takes its large rounds
  if (last_piece.npieces > 0) finish_piece<G, D, BS>(a, last_piece, lane);
  mail_post(box, mcount + wid, posted, done_msg, lane);
  if (tl) tl[kTlDone] = global_ns();
}

template <typename T, int D, int BS, int G, typename KV = T>
cudaError_t launch_decode_mma(const DecodeArgs &a, const TmaMaps *maps, int num_ctas,
                              bool overlap_previous, cudaStream_t st) {
  using Tr = MmaTraits<D, BS, G, (int)sizeof(KV)>;
  return launch_overlapping(paged_decode_mma_kernel<T, D, BS, G, KV>, num_ctas, Tr::kThreads,
                            Tr::kSmemBytes, overlap_previous, st, a, *maps);
}

template <typename T, int D, int BS, int G, typename KV = T>
bool make_decode_mma(DecodeKernel *k) {
  using Tr = MmaTraits<D, BS, G, (int)sizeof(KV)>;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(paged_decode_mma_kernel<T, D, BS, G, KV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Tr::kSmemBytes) != cudaSuccess)
      return false;
    configured[dev] = true;
  }
  k->launch = &launch_decode_mma<T, D, BS, G, KV>;
  k->launch_reduce = &launch_decode_merge<G, D, BS>;
  k->kernel = reinterpret_cast<const void *>(&paged_decode_mma_kernel<T, D, BS, G, KV>);
  k->warps_per_cta = Tr::kWorkers;
  k->threads_per_cta = Tr::kThreads;
  k->smem_bytes = Tr::kSmemBytes;
  k->chunk_tokens = 16;
  k->tma_rows = Tr::kBoxRows;
  return true;
}

// Tables over block_size {8, 16, 32} x group {1, 2, 4, 8} for one element type and head_dim.
template <typename T, int D>
bool decode_table(int block_size, int group, bool tensor_cores, DecodeKernel *k) {
#define PA_CASE(BB, GG)                                                            \
  if (block_size == BB && group == GG)                                             \
    return tensor_cores ? make_decode_mma<T, D, BB, GG>(k) : make_decode_simt<T, D, BB, GG>(k);
#define PA_GROUPS(BB) PA_CASE(BB, 1) PA_CASE(BB, 2) PA_CASE(BB, 4) PA_CASE(BB, 8)
  PA_GROUPS(8)
  PA_GROUPS(16)
  PA_GROUPS(32)
#undef PA_GROUPS
#undef PA_CASE
  return false;
}

template <int D>
bool decode_table_f32(int block_size, int group, DecodeKernel *k) {
#define PA_CASE(BB, GG) \
  if (block_size == BB && group == GG) return make_decode_simt<float, D, BB, GG>(k);
#define PA_GROUPS(BB) PA_CASE(BB, 1) PA_CASE(BB, 2) PA_CASE(BB, 4) PA_CASE(BB, 8)
  PA_GROUPS(8)
  PA_GROUPS(16)
  PA_GROUPS(32)
#undef PA_GROUPS
#undef PA_CASE
  return false;
}

}  // namespace pa

namespace pa {

// FP8 E4M3 caches (head_dim 128) with a query of element type T: block_size {8, 16, 32} x
// group {1, 2, 4, 8}.
template <typename T>
bool decode_table_fp8(int block_size, int group, DecodeKernel *k) {
#define PA_CASE(BB, GG) \
  if (block_size == BB && group == GG) return make_decode_mma<T, 128, BB, GG, __nv_fp8_e4m3>(k);
#define PA_GROUPS(BB) PA_CASE(BB, 1) PA_CASE(BB, 2) PA_CASE(BB, 4) PA_CASE(BB, 8)
  PA_GROUPS(8)
  PA_GROUPS(16)
  PA_GROUPS(32)
#undef PA_GROUPS
#undef PA_CASE
  return false;
}

}  // namespace pa

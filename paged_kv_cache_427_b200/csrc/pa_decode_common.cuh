// pa_decode_common.cuh - parts shared by the decode kernels: the stream-K work split over
// warps, the chunk cursor that walks a warp's share, and the log-sum-exp merge of pieces.
//
// What decode computes ([P4] "vLLM core architecture: model loading, PagedAttention
// principle, KV cache management", 2.2.2): for every sequence s and query head h the keys and
// values are assembled through the block table and
//     out[s,h] = softmax_t(scale * q[s,h] . K_t) . V_t  over the positions t < L_s.
// The per-block loop printed on that page adds per-block outputs and only states the principle;
// the kernels compute the full-context softmax with running rescaling and merge split contexts
// with the log-sum-exp rule.  Block tables and physical blocks follow [P2] "vLLM core
// features: PagedAttention, Continuous Batching, quantization support, distributed inference"
// 4.1 and [P4] 2.2.1.
//
// Work split (B200 design, not from the sources): the step's work is the list of chunks
// (sequence, kv head, a fixed number of key rows) in sequence-major order, C chunks in all.
// Every chunk costs one unit and every (sequence, kv head) a further `alpha` units at its start
// (what a warp spends once per piece: loading the query rows, storing and merging a partial
// result), so chunk c of pair p = s * Hkv + kvh sits at position pos(c) = c + alpha * (p + 1) of
// T = C + alpha * S * Hkv positions.  A persistent grid of W warps gives warp w the chunks with
// positions in [floor(wT/W), floor((w+1)T/W)) (W clamped to C): equal cost per warp, whatever the
// mix of lengths, and no launch size depends on context lengths.  A (sequence, kv head) inside
// one share is written directly; otherwise each share's piece stores (o, m, l) in the workspace
// and the last piece to finish (atomic ticket, no waiting) merges them.
#pragma once

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// Per-stage description written by the issuing lane before the stage's barrier arrives.
struct ChunkMeta {
  int s, kvh, chunk, len;
  int flags, first_worker, npieces, pair;
};
constexpr int kFirst = 1;      // first chunk of this warp's piece of a (sequence, kv head)
constexpr int kLast = 2;       // last chunk of the piece
constexpr int kPairStart = 4;  // chunk 0 of the (sequence, kv head)
constexpr int kNewRow = 8;     // fused step: the chunk holds position L-1, the step's new token

__device__ __forceinline__ int clamp_len(int len, int max_len) {
  return len < 0 ? 0 : (len > max_len ? max_len : len);
}

// The warp whose share of positions [floor(w*T/W), floor((w+1)*T/W)) contains position x.
__device__ __forceinline__ int worker_of(long long x, long long T, int W) {
  return (int)(((x + 1) * (long long)W + T - 1) / T - 1);
}

// Fused decode step: thread `tid` of `nthreads` moves its 16-byte pieces of the step's new
// key and value rows into their cache slots (as the cache write kernel does), and checks that
// token s is sequence s's position L-1, which the decode reads from the new rows directly: a
// slot that differs sets PA_DEVERR_SLOT.
template <int BS>
__device__ __forceinline__ void fused_cache_write(const DecodeArgs &a, int max_len, int tid,
                                                  int nthreads) {
  const CacheWriteArgs &w = a.step;
  const int vec_per_row = w.row_bytes >> 4;
  const int64_t total = w.num_tokens * w.num_kv_heads * vec_per_row;
  for (int64_t idx = tid; idx < total; idx += nthreads) {
    const int v = (int)(idx % vec_per_row);
    const int64_t th = idx / vec_per_row;
    const int h = (int)(th % w.num_kv_heads);
    const int64_t t = th / w.num_kv_heads;
    const int64_t slot = __ldg(w.slots + t);
    if (h == 0 && v == 0) {
      const int len = clamp_len(__ldg(a.context_lens + t), max_len);
      int64_t expect = -1;
      if (len > 0) {
        const int blk = __ldg(a.block_tables + t * a.bt_s + (len - 1) / BS);
        expect = (int64_t)blk * BS + (len - 1) % BS;
      }
      if (slot != expect) set_error(a.err, PA_DEVERR_SLOT);
    }
    if (slot < 0) continue;
    if (slot >= w.num_slots) {
      if (h == 0 && v == 0) set_error(a.err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t dst = (slot / w.block_size) * w.c_blk + h * w.c_head + (slot % w.block_size) * w.row_bytes + v * 16;
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(w.key + t * w.k_tok + h * w.k_head) + v);
    const uint4 vv = __ldg(reinterpret_cast<const uint4 *>(w.value + t * w.v_tok + h * w.v_head) + v);
    *reinterpret_cast<uint4 *>(w.key_cache + dst) = kv;
    *reinterpret_cast<uint4 *>(w.value_cache + dst) = vv;
  }
}

// The same for FP8 E4M3 caches: token s's 16-bit rows (element type S) are quantised with the
// cache write's arithmetic (fp8_codes16), so the codes match what that kernel would store.
// w.row_bytes is the cache row (head_dim codes).
template <typename S, int BS>
__device__ __forceinline__ void fused_cache_write_fp8(const DecodeArgs &a, int max_len, int tid,
                                                      int nthreads) {
  const CacheWriteArgs &w = a.step;
  const int vec_per_row = w.row_bytes >> 4;  // 16 codes per item
  const int64_t total = w.num_tokens * w.num_kv_heads * vec_per_row;
  for (int64_t idx = tid; idx < total; idx += nthreads) {
    const int v = (int)(idx % vec_per_row);
    const int64_t th = idx / vec_per_row;
    const int h = (int)(th % w.num_kv_heads);
    const int64_t t = th / w.num_kv_heads;
    const int64_t slot = __ldg(w.slots + t);
    if (h == 0 && v == 0) {
      const int len = clamp_len(__ldg(a.context_lens + t), max_len);
      int64_t expect = -1;
      if (len > 0) {
        const int blk = __ldg(a.block_tables + t * a.bt_s + (len - 1) / BS);
        expect = (int64_t)blk * BS + (len - 1) % BS;
      }
      if (slot != expect) set_error(a.err, PA_DEVERR_SLOT);
    }
    if (slot < 0) continue;
    if (slot >= w.num_slots) {
      if (h == 0 && v == 0) set_error(a.err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t dst = (slot / w.block_size) * w.c_blk + h * w.c_head + (slot % w.block_size) * w.row_bytes + v * 16;
    const int64_t src = (int64_t)v * 16 * (int64_t)sizeof(S);
    *reinterpret_cast<uint4 *>(w.key_cache + dst) =
        fp8_codes16<S>(w.key + t * w.k_tok + h * w.k_head + src, __ldg(a.k_scale + h));
    *reinterpret_cast<uint4 *>(w.value_cache + dst) =
        fp8_codes16<S>(w.value + t * w.v_tok + h * w.v_head + src, __ldg(a.v_scale + h));
  }
}

// The first position the decode reads of sequence s, whose context holds len positions: its
// shared prefix when the shared-prefix pass covered it (0 < prefix < len, a multiple of the block
// size, within the pass's items), else 0 (the whole context is decoded here).  A prefix that is
// not a multiple of the block size or needs more items than the workspace holds is reported.
template <int BS>
__device__ __forceinline__ int decode_start(const DecodeArgs &a, int s, int len) {
  if (a.prefix_lens == nullptr) return 0;
  const int p = __ldg(a.prefix_lens + s);
  if (p <= 0 || p >= len) return 0;
  if (p % BS != 0 || (p + a.pre_kv_tokens - 1) / a.pre_kv_tokens > a.pre_splits) {
    set_error(a.err, PA_DEVERR_PREFIX);
    return 0;
  }
  return p;
}

// The number of prefix-pass partial results sequence s merges (0 without a shared prefix).
template <int BS>
__device__ __forceinline__ int prefix_pieces(const DecodeArgs &a, int s, int max_len) {
  if (a.prefix_lens == nullptr) return 0;
  const int raw = __ldg(a.context_lens + s);
  const int len = raw < 0 ? 0 : (raw > max_len ? max_len : raw);
  const int p = decode_start<BS>(a, s, len);
  return p > 0 ? (p + a.pre_kv_tokens - 1) / a.pre_kv_tokens : 0;
}

// Test hook: whether worker warp gw's first stage waits for 16 bytes that no copy sends
// (mode 1: every worker; mode 2: the odd-numbered workers only).
__device__ __forceinline__ bool test_stalls(const DecodeArgs &a, int gw) {
  return a.test_stall == 1 || (a.test_stall == 2 && (gw & 1));
}

// Where one warp's share starts and how long it is.
struct WarpShare {
  long long T;  // positions of the split: the step's chunks plus alpha per (sequence, kv head)
  int W;        // effective number of workers
  int alpha;    // positions per (sequence, kv head) start
  long long g0, n;  // first chunk (index in the chunk list) and number of chunks
  int s, rem, len;  // first chunk: sequence, index among that sequence's Hkv*nch chunks, length
};

// Zero the `heads` output rows of a sequence with an empty context (kept out of line: rare;
// plain arguments, so the kernel parameters need no local copy).
template <int D>
__device__ __noinline__ void zero_rows(char *row0, long long out_h, int out_dtype, int heads) {
  const int out_elt = out_dtype == PA_F32 ? 4 : 2;
  const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int h = 0; h < heads; ++h)
    for (int d = 0; d < D; d += 8)
      store_row_piece(row0 + ((long long)h * out_h + d) * out_elt, out_dtype, z, 8);
}

__device__ __forceinline__ long long warp_sum(long long x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(FULL_MASK, x, off);
  return x;
}

// Warp-level prologue: every warp counts the step's chunks itself (reading context_lens
// coalesced), takes its share of positions, and finds the first chunk at or after each end of it
// with a scan over 32 sequences at a time.  No shared memory and no block-wide barrier, so warps
// start as soon as they are scheduled.  Warp gw also flags bad lengths (warp 0) and zeroes the
// rows of empty contexts s with s % (warps launched) == gw.  Returns false when this warp has no
// chunk.
template <int CH, int kWarps, int G, int D, int BS, bool kZeroEmpty = true>
__device__ __forceinline__ bool split_prologue(const DecodeArgs &a, int max_len, WarpShare &ws) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int launched = gridDim.x * kWarps;
  const int S = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  const int alpha = a.piece_cost;
  long long mine = 0;
  for (int base = 0; base < S; base += 32) {
    const int s = base + lane;
    if (s < S) {
      const int raw = __ldg(a.context_lens + s);
      const int len = clamp_len(raw, max_len);
      if (raw != len && gw == 0) set_error(a.err, PA_DEVERR_CONTEXT_LEN);
      if (kZeroEmpty && len == 0 && s % launched == gw)
        zero_rows<D>(static_cast<char *>(a.out) + (long long)s * a.out_s * (a.out_dtype == PA_F32 ? 4 : 2),
                     a.out_h, a.out_dtype, Hkv * G);
      mine += (len - decode_start<BS>(a, s, len) + CH - 1) / CH;
    }
  }
  const long long C = warp_sum(mine) * Hkv;
  const long long T = C + (long long)alpha * S * Hkv;
  const int W = (int)(C < (long long)a.num_workers ? C : (long long)a.num_workers);
  ws.T = T;
  ws.W = W;
  ws.alpha = alpha;
  if (W == 0 || gw >= W) return false;
  // the first chunk at or after position x0 (this share's start) and x1 (the next share's)
  const long long x0 = (long long)gw * T / W, x1 = (long long)(gw + 1) * T / W;
  long long c1 = C;
  bool found0 = false, found1 = false;
  long long run_cnt = 0, run_cost = 0;
  for (int base = 0; base < S && !found1; base += 32) {
    const int s = base + lane;
    const int full = s < S ? clamp_len(__ldg(a.context_lens + s), max_len) : 0;
    const int len = s < S ? full - decode_start<BS>(a, s, full) : 0;  // positions decoded here
    const int nch = (len + CH - 1) / CH;
    const long long cnt = (long long)nch * Hkv;
    const long long cost = s < S ? (long long)(nch + alpha) * Hkv : 0;
    long long incl_cnt = cnt, incl_cost = cost;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(FULL_MASK, incl_cnt, off);
      const long long z = __shfl_up_sync(FULL_MASK, incl_cost, off);
      if (lane >= off) {
        incl_cnt += y;
        incl_cost += z;
      }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j == 0 ? found0 : found1) continue;
      const long long x = j == 0 ? x0 : x1;
      // the first sequence with a chunk whose positions end after x
      const bool hit = nch > 0 && run_cost + incl_cost > x;
      const unsigned int hits = __ballot_sync(FULL_MASK, hit);
      if (hits == 0u) continue;
      const int src = __ffs(hits) - 1;
      const long long seq_cost0 = run_cost + __shfl_sync(FULL_MASK, incl_cost - cost, src);
      const long long seq_cnt0 = run_cnt + __shfl_sync(FULL_MASK, incl_cnt - cnt, src);
      const int hn = __shfl_sync(FULL_MASK, nch, src);
      const long long r = x > seq_cost0 ? x - seq_cost0 : 0;  // x may lie in an empty sequence before
      const int kvh = (int)(r / (hn + alpha));
      const int off = (int)(r - (long long)kvh * (hn + alpha));
      const int rem = kvh * hn + (off < alpha ? 0 : off - alpha);
      if (j == 0) {
        found0 = true;
        ws.s = base + src;
        ws.rem = rem;
        ws.len = __shfl_sync(FULL_MASK, len, src);
        ws.g0 = seq_cnt0 + rem;
      } else {
        found1 = true;
        c1 = seq_cnt0 + rem;
      }
    }
    run_cnt += __shfl_sync(FULL_MASK, incl_cnt, 31);
    run_cost += __shfl_sync(FULL_MASK, incl_cost, 31);
  }
  if (!found0) return false;  // no chunk lies at or after this share's start
  ws.n = c1 - ws.g0;
  return ws.n > 0;
}

// Walks one warp's share chunk by chunk in issue order.  Every lane keeps the same state.
// A chunk is CH key rows; it touches COPIES physical blocks of COPY_ROWS rows each.  The block
// ids of the next chunk to issue are loaded one chunk ahead.
template <int CH, int BS, int COPIES, int COPY_ROWS>
struct ChunkCursor {
  int s, len, nch, kvh, i, next_len;
  int start, next_start;  // first decoded position of the sequence (its shared prefix, or 0)
  long long base;  // global index of chunk 0 of the current (sequence, kv head)
  int first_worker, npieces;
  long long issued, n, T;
  int W, alpha, S, Hkv, max_len;
  int blk[COPIES];

  __device__ __forceinline__ void fetch_blocks(const DecodeArgs &a) {
#pragma unroll
    for (int k = 0; k < COPIES; ++k) {
      const int t = i * CH + k * COPY_ROWS;
      blk[k] = (t < len) ? __ldg(a.block_tables + (long long)s * a.bt_s + (start + t) / BS) : 0;
    }
  }

  // The warps whose shares hold the current (sequence, kv head): chunk c of pair p lies at
  // position c + alpha * (p + 1).
  __device__ __forceinline__ void pieces() {
    const long long shift = (long long)alpha * ((long long)s * Hkv + kvh + 1);
    first_worker = worker_of(base + shift, T, W);
    npieces = worker_of(base + nch - 1 + shift, T, W) - first_worker + 1;
  }

  __device__ __forceinline__ void init(const DecodeArgs &a, const WarpShare &ws, int max_len_) {
    S = a.num_seqs;
    Hkv = a.num_kv_heads;
    max_len = max_len_;
    T = ws.T;
    W = ws.W;
    alpha = ws.alpha;
    n = ws.n;
    issued = 0;
    s = ws.s;
    len = ws.len;
    start = decode_start<BS>(a, s, clamp_len(__ldg(a.context_lens + s), max_len));
    nch = (len + CH - 1) / CH;
    kvh = ws.rem / nch;
    i = ws.rem % nch;
    base = ws.g0 - ws.rem + (long long)kvh * nch;
    load_next(a);
    fetch_blocks(a);
    pieces();
  }

  // Decoded length and start of sequence s + 1.
  __device__ __forceinline__ void load_next(const DecodeArgs &a) {
    next_len = 0;
    next_start = 0;
    if (s + 1 < S) {
      const int full = clamp_len(__ldg(a.context_lens + s + 1), max_len);
      next_start = decode_start<BS>(a, s + 1, full);
      next_len = full - next_start;
    }
  }

  __device__ __forceinline__ int flags() const {
    int f = 0;
    if (i == 0 || issued == 0) f |= kFirst;
    if (i == nch - 1 || issued == n - 1) f |= kLast;
    if (i == 0) f |= kPairStart;
    return f;
  }

  __device__ __forceinline__ ChunkMeta meta(int f) const {
    ChunkMeta m;
    m.s = s;
    m.kvh = kvh;
    m.chunk = i;
    m.len = len;
    m.flags = f;
    m.first_worker = first_worker;
    m.npieces = npieces;
    m.pair = s * Hkv + kvh;
    return m;
  }

  // Copies of this chunk that hold context rows (the others are past the context).
  __device__ __forceinline__ int valid_copies() const {
    int v = 0;
#pragma unroll
    for (int k = 0; k < COPIES; ++k) v += (i * CH + k * COPY_ROWS < len);
    return v;
  }

  // Move to the next chunk of the share (call after issuing the current one).
  __device__ __forceinline__ void advance(const DecodeArgs &a) {
    ++issued;
    if (issued >= n) return;
    if (++i == nch) {
      i = 0;
      base += nch;
      if (++kvh == Hkv) {
        kvh = 0;
        ++s;
        len = next_len;
        start = next_start;
        while (len == 0 && s + 1 < S) {
          ++s;
          const int full = clamp_len(__ldg(a.context_lens + s), max_len);
          start = decode_start<BS>(a, s, full);
          len = full - start;
        }
        nch = (len + CH - 1) / CH;
        load_next(a);
      }
      pieces();
    }
    fetch_blocks(a);
  }
};

// Merge the pieces (o, m, l) of one (sequence, kv head) and write its G output rows.  Called by
// a whole warp; pieces live in workspace slots pair + first_worker + k, k < npieces, followed by
// the npre partial results of the shared-prefix pass (slots of the query head, item k - npieces).
// Loads are issued for many pieces at once (lane k fetches piece k's (m, l); the outputs of
// several pieces per round) so a merge costs a few memory round trips, not two per piece.  m is
// in base-2 units.
template <int G, int D, int U = (G >= 8 ? 1 : 16 / G)>
__device__ __forceinline__ void merge_pieces(const DecodeArgs &a, int pair, int first_worker,
                                             int npieces, int s, int kvh, int lane, int npre = 0) {
  const long long seg0 = (long long)pair + first_worker;
  const long long pre0 = ((long long)s * a.num_kv_heads + kvh) * G;  // first query head's slots
  const int total = npieces + npre;
  // (m, l) and output of piece k for head h
  auto ml_of = [&](int k, int h) -> const float2 * {
    return k < npieces
               ? reinterpret_cast<const float2 *>(a.part_ml + ((seg0 + k) * G + h) * 2)
               : reinterpret_cast<const float2 *>(a.pre_ml + ((pre0 + h) * a.pre_splits + (k - npieces)) * 2);
  };
  auto o_of = [&](int k, int h) -> const float4 * {
    return k < npieces
               ? reinterpret_cast<const float4 *>(a.part_o + ((seg0 + k) * G + h) * D)
               : reinterpret_cast<const float4 *>(a.pre_o + ((pre0 + h) * a.pre_splits + (k - npieces)) * D);
  };
  const bool active = lane < D / 4;  // lane j handles dims [4j, 4j+4) of every head
  float M[G], den[G];
  float4 num[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    M[h] = -INFINITY;
    den[h] = 0.f;
    num[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // Outputs: U pieces per round (U*G float4 in flight per lane), loads issued together.  The
  // first round of each group of 32 pieces is issued with the group's (m, l), since the outputs
  // do not depend on the weights: a merge of up to U pieces costs one memory round trip.
  float4 x[U][G];
  auto load_round = [&](int first, int cnt) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int h = 0; h < G; ++h)
        x[u][h] = (active && u < cnt) ? __ldcg(o_of(first + u, h) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  for (int base = 0; base < total; base += 32) {
    const int cnt = total - base < 32 ? total - base : 32;
    load_round(base, cnt);
    // lane k < cnt: (m, l) of piece base + k for every head
    float mk[G], lk[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mk[h] = -INFINITY;
      lk[h] = 0.f;
    }
    if (lane < cnt) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float2 ml = __ldcg(ml_of(base + lane, h));
        mk[h] = ml.x;
        lk[h] = ml.y;
      }
    }
    // fold this group into the running maximum and rescale what is already accumulated
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float gm = mk[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) gm = fmaxf(gm, __shfl_xor_sync(FULL_MASK, gm, off));
      const float newM = fmaxf(M[h], gm);
      const float r = (M[h] == -INFINITY) ? 0.f : fast_exp2(M[h] - newM);
      den[h] *= r;
      num[h].x *= r;
      num[h].y *= r;
      num[h].z *= r;
      num[h].w *= r;
      M[h] = newM;
      // this lane's weight for its piece
      const float w = (lane < cnt) ? lk[h] * fast_exp2(mk[h] - newM) : 0.f;
      float ws = w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(FULL_MASK, ws, off);
      den[h] += ws;
      mk[h] = w;  // reuse: the weight of piece base + lane
    }
    for (int k = 0; k < cnt; k += U) {
      if (k > 0) load_round(base + k, cnt - k);
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = __shfl_sync(FULL_MASK, mk[h], (k + u) & 31);
          if (k + u < cnt) {
            num[h].x += w * x[u][h].x;
            num[h].y += w * x[u][h].y;
            num[h].z += w * x[u][h].z;
            num[h].w += w * x[u][h].w;
          }
        }
    }
  }
  if (!active) return;
  const int out_elt = a.out_dtype == PA_F32 ? 4 : 2;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float inv = 1.f / den[h];
    const float v[4] = {num[h].x * inv, num[h].y * inv, num[h].z * inv, num[h].w * inv};
    char *dst = static_cast<char *>(a.out) +
                ((long long)s * a.out_s + (long long)(kvh * G + h) * a.out_h + lane * 4) * out_elt;
    if (a.out_dtype == PA_F32) {
      *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    } else if (a.out_dtype == PA_BF16) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t *>(&lo);
      u.y = *reinterpret_cast<uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(dst) = u;
    } else {
      __half2 lo = __floats2half2_rn(v[0], v[1]), hi = __floats2half2_rn(v[2], v[3]);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t *>(&lo);
      u.y = *reinterpret_cast<uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(dst) = u;
    }
  }
}

#ifndef PA_TICKET_ACQREL
#define PA_TICKET_ACQREL 1  // 0: a fence, then a relaxed atomic, then a fence
#endif

// Take a ticket of a merge counter.  With PA_TICKET_ACQREL the atomic has acquire-release
// semantics at GPU scope: the release orders the warp's stores of its piece (made visible to
// lane 0 by the warp barrier before it) before the increment, and the acquire orders the loads
// of the other pieces after it for the warp that takes the last ticket: one round trip in
// place of a fence followed by an atomic and a second fence.  Called by lane 0.
__device__ __forceinline__ unsigned int ticket_add(unsigned int *counter) {
#if PA_TICKET_ACQREL
  unsigned int old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(counter) : "memory");
  return old;
#else
  return atomicAdd(counter, 1u);
#endif
}

// What a worker needs to take a split piece's ticket after its (o, m, l) are stored.
struct PieceInfo {
  int pair, first_worker, npieces, s, kvh;
};

// Take the ticket of a published piece and merge when it is the last of its (sequence, kv
// head).  The caller has made the piece's stores visible GPU-wide.  Called by a whole warp.
template <int G, int D, int BS>
__device__ __forceinline__ void take_ticket(const DecodeArgs &a, const PieceInfo &p, int lane) {
  unsigned int ticket = 0;
  __syncwarp();
  // a single piece has only shared-prefix partial results to merge with: no ticket
  if (p.npieces > 1 && lane == 0) ticket = ticket_add(a.counters + p.pair);
  ticket = __shfl_sync(FULL_MASK, ticket, 0);
  if (ticket == (unsigned int)(p.npieces - 1)) {
    if (!PA_TICKET_ACQREL) __threadfence();
    __syncwarp();
    const int npre = prefix_pieces<BS>(a, p.s, a.max_blocks * BS);
    if (npre > 0) wait_for_previous_grid();  // the prefix pass's partial results are complete
    merge_pieces<G, D>(a, p.pair, p.first_worker, p.npieces, p.s, p.kvh, lane, npre);
    if (lane == 0 && p.npieces > 1) a.counters[p.pair] = 0u;
  }
}

// After a piece's (o, m, l) are stored: publish them, take a ticket, and merge when this is the
// last piece of its (sequence, kv head), U pieces per round.  Called by a whole warp.  A single
// piece (merged with shared-prefix partial results only) takes no ticket.
template <int G, int D, int BS, int U = (G >= 8 ? 1 : 16 / G)>
__device__ __forceinline__ void finish_piece(const DecodeArgs &a, const ChunkMeta &m, int lane) {
  if (a.separate_reduce) return;
  const unsigned int others = (unsigned int)(m.npieces - 1);
  if (!PA_TICKET_ACQREL) __threadfence();
  __syncwarp();
  unsigned int ticket = others;
  if (others > 0 && lane == 0) ticket = ticket_add(a.counters + m.pair);
  ticket = __shfl_sync(FULL_MASK, ticket, 0);
  if (ticket == others) {
    if (!PA_TICKET_ACQREL) __threadfence();
    __syncwarp();
    const int npre = prefix_pieces<BS>(a, m.s, a.max_blocks * BS);
    if (npre > 0) wait_for_previous_grid();  // the prefix pass's partial results are complete
    merge_pieces<G, D, U>(a, m.pair, m.first_worker, m.npieces, m.s, m.kvh, lane, npre);
    if (lane == 0 && others > 0) a.counters[m.pair] = 0u;
  }
}

// Separate merge: one warp per (sequence, kv head) that has more than one piece.  Launched to
// overlap the decode grid; it waits for that grid's pieces before reading them.
template <int G, int D, int BS>
__global__ void __launch_bounds__(128) paged_decode_merge_kernel(const DecodeArgs a) {
  const int lane = threadIdx.x & 31;
  wait_for_previous_grid();
  const long long pairs = (long long)a.num_seqs * a.num_kv_heads;
  const int max_len = a.max_blocks * BS;
  for (long long p = (long long)blockIdx.x * 4 + (threadIdx.x >> 5); p < pairs;
       p += (long long)gridDim.x * 4) {
    const int s = (int)(p / a.num_kv_heads);
    const int kvh = (int)(p % a.num_kv_heads);
    if (clamp_len(__ldg(a.context_lens + s), max_len) == 0) continue;
    const int2 pm = a.pair_meta[p];
    if (pm.y <= 1) continue;
    merge_pieces<G, D>(a, (int)p, pm.x, pm.y, s, kvh, lane);
  }
}

template <int G, int D, int BS>
cudaError_t launch_decode_merge(const DecodeArgs &a, cudaStream_t st) {
  const long long pairs = (long long)a.num_seqs * a.num_kv_heads;
  long long blocks = (pairs + 3) / 4;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, paged_decode_merge_kernel<G, D, BS>, a);
}

}  // namespace pa

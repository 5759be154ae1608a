// pa_decode.cuh - paged decode attention for sm_100a.
//
// What it computes ([P4] "vLLM core architecture: model loading, PagedAttention principle, KV
// cache management", 2.2.2): for every sequence s and query head h, the keys and values of the
// sequence are assembled through its block table and
//     out[s,h] = softmax_t(scale * q[s,h] . K_t) . V_t  over its context positions t < L_s.
// The per-block loop printed on that page adds per-block outputs, which only states the
// principle; the kernel computes the full-context softmax by rescaling running sums (online
// softmax), and merges split contexts with the log-sum-exp rule.  Block tables and physical
// blocks follow [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization
// support, distributed inference" 4.1 and [P4] 2.2.1.
//
// How the work is split (B200 design, not from the sources):
//   * The step's work is the list of chunks (sequence, kv head, 4 KB of keys = 16 rows at
//     head_dim 128 bf16) in sequence-major order.  A persistent grid of W warps gives every
//     warp an equal contiguous share of that list (stream-K), so uneven context lengths do not
//     leave SMs idle and no launch size depends on context_lens.
//   * Each warp runs its own ring of stages in shared memory.  Lane 0 issues one-dimensional
//     bulk asynchronous copies (cp.async.bulk, completion counted on an mbarrier) of each
//     chunk's key tile and value tile straight from their physical blocks, plus the query rows
//     when a new (sequence, kv head) starts; the block-table entry is resolved once per copy
//     and fetched one chunk ahead.  No other warp touches the ring, so the main loop has no
//     block-wide barrier.
//   * The query heads of a GQA group share every loaded tile.  A token row of keys is spread
//     over RL = head_dim*elt/16 lanes (16 bytes each); per-head dot products are reduced with a
//     transposed butterfly so that each lane ends up owning one (token, head) logit.  Logits
//     are kept in base-2 units (q pre-scaled by scale*log2 e).  The running maximum is only
//     moved when a chunk exceeds it by more than 2^8, which bounds every weight by 256 and
//     skips most rescaling.  P.V uses packed fp32x2 FMAs with P kept in fp32.
//   * A (sequence, kv head) covered by one warp is written directly.  Otherwise every piece
//     stores (o, m, l) in the workspace; the last piece to finish (atomic ticket, no waiting)
//     merges them, or a separate reduce kernel does so when asked.
#pragma once

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

template <typename T, int D, int BS, int G>
struct DecodeTraits {
  static constexpr int kElt = (int)sizeof(T);
  static constexpr int kRow = D * kElt;           // bytes of one key (or value) row
  static constexpr int kRL = kRow / 16;           // lanes per row
  static constexpr int kTPS = 32 / kRL;           // rows per warp step
  static constexpr int kEPL = 16 / kElt;          // elements per lane
  static constexpr int kChunk = 4096 / kRow;      // rows per chunk: 4 KB of keys
  static constexpr int kSteps = kChunk / kTPS;    // warp steps per chunk (8 for every case)
  static constexpr int kCopyRows = kChunk < BS ? kChunk : BS;
  static constexpr int kCopies = kChunk / kCopyRows;  // blocks touched per chunk
  static constexpr int kCopyBytes = kCopyRows * kRow;
  static constexpr int kQBytes = G * kRow;
  static constexpr int kStageBytes = 2 * 4096 + ((kQBytes + 127) / 128) * 128;
  static constexpr int kWarps = 4;
  static constexpr int kStages = (kWarps * 3 * kStageBytes <= 110 * 1024) ? 3 : 2;
  static constexpr int kHeadLanes = kRL / G;      // lanes sharing a head after the reduce
  static constexpr int kMetaOff = kStages * kStageBytes;
  static constexpr int kBarOff = kMetaOff + kStages * 32;
  static constexpr int kPbufOff = (kBarOff + kStages * 8 + 127) / 128 * 128;
  static constexpr int kWarpBytes = ((kPbufOff + kChunk * G * 4) + 127) / 128 * 128;
  static constexpr int kPrologueOff = kWarps * kWarpBytes;
  static constexpr int kSmemBytes = kPrologueOff + 256;
  static_assert(kRow == 128 || kRow == 256 || kRow == 512, "row of 128, 256 or 512 bytes");
  static_assert(kRL >= G, "a group must fit in one row of lanes");
  static_assert(kSteps == 8, "chunk = 8 warp steps");
  static_assert(kCopyBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
};

// Per-stage description written by the issuing lane before the stage's barrier arrives.
struct ChunkMeta {
  int s, kvh, chunk, len;
  int flags, first_worker, npieces, pair;
};
constexpr int kFirst = 1;      // first chunk of this warp's piece of a (sequence, kv head)
constexpr int kLast = 2;       // last chunk of the piece
constexpr int kPairStart = 4;  // chunk 0 of the (sequence, kv head)

__device__ __forceinline__ int clamp_len(int len, int max_len) {
  return len < 0 ? 0 : (len > max_len ? max_len : len);
}

// Transposed butterfly: v[0..N) are this lane's partial dot products for N heads over its
// slice of a row that spans the lanes differing in bits [0, log2(2*OFF)).  After the call,
// v[0] holds the full dot product of head (lane_in_row >> log2(OFF*2/N)) ... i.e. the lanes of a
// row are split into N equal ranges, range n owning head n.
template <int N, int OFF>
struct TransposeReduce {
  static __device__ __forceinline__ void run(float *v, int lane) {
    if constexpr (OFF == 0) {
      return;
    } else if constexpr (N > 1) {
      const bool upper = (lane & OFF) != 0;
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        const float send = upper ? v[k] : v[k + N / 2];
        const float keep = upper ? v[k + N / 2] : v[k];
        v[k] = keep + __shfl_xor_sync(FULL_MASK, send, OFF);
      }
      TransposeReduce<N / 2, OFF / 2>::run(v, lane);
    } else {
      v[0] += __shfl_xor_sync(FULL_MASK, v[0], OFF);
      TransposeReduce<1, OFF / 2>::run(v, lane);
    }
  }
};

// Index of the warp whose share of the chunk list contains chunk c: shares are
// [floor(w*C/W), floor((w+1)*C/W)).
__device__ __forceinline__ int worker_of(long long c, long long C, int W) {
  return (int)(((c + 1) * (long long)W + C - 1) / C - 1);
}

// Merge the pieces (o, m, l) of one (sequence, kv head) and write its G output rows.  Called by
// one whole warp; pieces live in workspace slots pair + first_worker + k, k < npieces.
template <typename Tr>
__device__ __forceinline__ void merge_pieces(const DecodeArgs &a, int pair, int first_worker,
                                             int npieces, int s, int kvh, int lane) {
  constexpr int G = Tr::kRL / Tr::kHeadLanes;
  constexpr int D = Tr::kRow / Tr::kElt;
  constexpr int EPL = Tr::kEPL;
  const int r = lane / Tr::kRL;
  const int j = lane % Tr::kRL;
  float M[G];
#pragma unroll
  for (int h = 0; h < G; ++h) M[h] = -INFINITY;
  for (int k = 0; k < npieces; ++k) {
    const long long seg = (long long)pair + first_worker + k;
#pragma unroll
    for (int h = 0; h < G; ++h) M[h] = fmaxf(M[h], __ldcg(a.part_ml + (seg * G + h) * 2));
  }
  float num[G][EPL];
  float den[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    den[h] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) num[h][e] = 0.f;
  }
  for (int k = 0; k < npieces; ++k) {
    const long long seg = (long long)pair + first_worker + k;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m = __ldcg(a.part_ml + (seg * G + h) * 2);
      const float l = __ldcg(a.part_ml + (seg * G + h) * 2 + 1);
      const float w = l * fast_exp2(m - M[h]);
      den[h] += w;
      const float4 *o = reinterpret_cast<const float4 *>(a.part_o + (seg * G + h) * D + j * EPL);
#pragma unroll
      for (int e = 0; e < EPL; e += 4) {
        const float4 x = __ldcg(o + e / 4);
        num[h][e] += w * x.x;
        num[h][e + 1] += w * x.y;
        num[h][e + 2] += w * x.z;
        num[h][e + 3] += w * x.w;
      }
    }
  }
  if (r == 0) {
    const int out_elt = a.out_dtype == PA_F32 ? 4 : 2;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v[EPL];
      const float inv = 1.f / den[h];
#pragma unroll
      for (int e = 0; e < EPL; ++e) v[e] = num[h][e] * inv;
      char *dst = static_cast<char *>(a.out) +
                  ((long long)s * a.out_s + (long long)(kvh * G + h) * a.out_h + j * EPL) * out_elt;
      store_row_piece(dst, a.out_dtype, v, EPL);
    }
  }
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(128, 1) paged_decode_kernel(const DecodeArgs a) {
  using Tr = DecodeTraits<T, D, BS, G>;
  constexpr int RL = Tr::kRL, TPS = Tr::kTPS, EPL = Tr::kEPL, CH = Tr::kChunk;
  constexpr int STEPS = Tr::kSteps, ST = Tr::kStages, HL = Tr::kHeadLanes;
  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int S = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  const int max_len = a.max_blocks * BS;

  // ---------------- prologue: size of the chunk list and where each warp starts -------------
  long long *red = reinterpret_cast<long long *>(smem + Tr::kPrologueOff);  // [kWarps]
  int4 *loc = reinterpret_cast<int4 *>(smem + Tr::kPrologueOff + 64);       // [kWarps]
  long long local = 0;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const int raw = __ldg(a.context_lens + s);
    const int len = clamp_len(raw, max_len);
    if (raw != len && blockIdx.x == 0) set_error(a.err, PA_DEVERR_CONTEXT_LEN);
    local += (len + CH - 1) / CH;
    if (len == 0 && (s % gridDim.x) == blockIdx.x) {
      // empty context: zero rows for every head of the sequence
      const int out_elt = a.out_dtype == PA_F32 ? 4 : 2;
      const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int h = 0; h < Hkv * G; ++h)
        for (int d = 0; d < D; d += 8)
          store_row_piece(static_cast<char *>(a.out) +
                              ((long long)s * a.out_s + (long long)h * a.out_h + d) * out_elt,
                          a.out_dtype, z, 8);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(FULL_MASK, local, off);
  if (lane == 0) red[wid] = local;
  if (threadIdx.x < Tr::kWarps) loc[threadIdx.x] = make_int4(-1, 0, 0, 0);
  __syncthreads();
  long long C = 0;
#pragma unroll
  for (int w = 0; w < Tr::kWarps; ++w) C += red[w];
  C *= Hkv;
  __syncthreads();
  // Never more workers than chunks, so that every worker's share is non-empty and the pieces
  // of a (sequence, kv head) belong to consecutive workers.
  const int W = (int)(C < (long long)a.num_workers ? C : (long long)a.num_workers);
  if (W == 0) return;

  // this CTA's warps' shares
  long long my_g0[Tr::kWarps];
  long long last_needed = -1;
#pragma unroll
  for (int w = 0; w < Tr::kWarps; ++w) {
    long long gw = (long long)blockIdx.x * Tr::kWarps + w;
    if (gw > W) gw = W;
    my_g0[w] = gw * C / W;
    const long long g1 = (gw + 1 > W ? W : gw + 1) * C / W;
    if (my_g0[w] < g1) last_needed = my_g0[w];
  }
  // locate each start: exclusive scan of chunk counts over sequences, 8 sequences per thread
  long long running = 0;
  for (int base = 0; base < S && running <= last_needed; base += 8 * 32 * Tr::kWarps) {
    long long cnt[8];
    long long tsum = 0;
    int lens8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int s = base + threadIdx.x * 8 + k;
      lens8[k] = s < S ? clamp_len(__ldg(a.context_lens + s), max_len) : 0;
      cnt[k] = (long long)((lens8[k] + CH - 1) / CH) * Hkv;
      tsum += cnt[k];
    }
    long long x = tsum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(FULL_MASK, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) red[wid] = x;
    __syncthreads();
    long long ex = running;
    long long tile_total = 0;
#pragma unroll
    for (int w = 0; w < Tr::kWarps; ++w) {
      if (w < wid) ex += red[w];
      tile_total += red[w];
    }
    ex += x - tsum;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
#pragma unroll
      for (int w = 0; w < Tr::kWarps; ++w)
        if (my_g0[w] <= last_needed && my_g0[w] >= ex && my_g0[w] < ex + cnt[k])
          loc[w] = make_int4(base + threadIdx.x * 8 + k, (int)(my_g0[w] - ex), lens8[k], 0);
      ex += cnt[k];
    }
    running += tile_total;
    __syncthreads();
  }

  // ---------------- per-warp pipeline -------------------------------------------------------
  const int gw = blockIdx.x * Tr::kWarps + wid;
  if (gw >= W) return;
  const long long g0 = (long long)gw * C / W;
  const long long g1 = (long long)(gw + 1) * C / W;
  const long long n = g1 - g0;
  if (n <= 0) return;
  const int4 start = loc[wid];
  if (start.x < 0) return;  // cannot happen when the scan is consistent

  unsigned char *wsm = smem + wid * Tr::kWarpBytes;
  ChunkMeta *meta = reinterpret_cast<ChunkMeta *>(wsm + Tr::kMetaOff);
  uint64_t *bars = reinterpret_cast<uint64_t *>(wsm + Tr::kBarOff);
  float *pbuf = reinterpret_cast<float *>(wsm + Tr::kPbufOff);

  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < ST; ++i) mbar_init(bars + i, 1);
    fence_barrier_init();
  }
  __syncwarp();

  // issue cursor (uniform across the warp)
  int c_s = start.x;
  int c_len = start.z;
  int c_nch = (c_len + CH - 1) / CH;
  int c_kvh = start.y / c_nch;
  int c_i = start.y % c_nch;
  long long c_base = g0 - start.y + (long long)c_kvh * c_nch;  // global index of chunk 0 of pair
  int c_next_len = (c_s + 1 < S) ? clamp_len(__ldg(a.context_lens + c_s + 1), max_len) : 0;
  int pf_blk[Tr::kCopies];
  auto fetch_blocks = [&]() {
#pragma unroll
    for (int k = 0; k < Tr::kCopies; ++k) {
      const int t = c_i * CH + k * Tr::kCopyRows;
      pf_blk[k] = (t < c_len) ? __ldg(a.block_tables + (long long)c_s * a.bt_s + t / BS) : 0;
    }
  };
  fetch_blocks();
  long long issued = 0;
  int c_first_worker = worker_of(c_base, C, W);
  int c_npieces = worker_of(c_base + c_nch - 1, C, W) - c_first_worker + 1;

  auto issue = [&](int slot) {
    int flags = 0;
    if (c_i == 0 || issued == 0) flags |= kFirst;
    if (c_i == c_nch - 1 || issued == n - 1) flags |= kLast;
    if (c_i == 0) flags |= kPairStart;
    unsigned char *stage = wsm + slot * Tr::kStageBytes;
    if (lane == 0) {
      ChunkMeta m;
      m.s = c_s;
      m.kvh = c_kvh;
      m.chunk = c_i;
      m.len = c_len;
      m.flags = flags;
      m.first_worker = c_first_worker;
      m.npieces = c_npieces;
      m.pair = c_s * Hkv + c_kvh;
      meta[slot] = m;
      int ncopy = 0;
#pragma unroll
      for (int k = 0; k < Tr::kCopies; ++k) ncopy += (c_i * CH + k * Tr::kCopyRows < c_len);
      const uint32_t bytes = 2u * ncopy * Tr::kCopyBytes +
                             ((flags & kFirst) ? (uint32_t)Tr::kQBytes : 0u) +
                             ((a.test_stall && issued == 0) ? 16u : 0u);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bars + slot, bytes);
#pragma unroll
      for (int k = 0; k < Tr::kCopies; ++k) {
        const int t = c_i * CH + k * Tr::kCopyRows;
        if (t < c_len) {
          long long blk = pf_blk[k];
          if (blk < 0 || blk >= a.num_blocks) {
            set_error(a.err, PA_DEVERR_BLOCK_ID);
            blk = 0;
          }
          const long long off =
              (blk * a.kv_blk + (long long)c_kvh * a.kv_head + (long long)(t % BS) * D) *
              Tr::kElt;
          bulk_copy_g2s(stage + k * Tr::kCopyBytes,
                        static_cast<const char *>(a.key_cache) + off, Tr::kCopyBytes, bars + slot);
          bulk_copy_g2s(stage + 4096 + k * Tr::kCopyBytes,
                        static_cast<const char *>(a.value_cache) + off, Tr::kCopyBytes,
                        bars + slot);
        }
      }
      if (flags & kFirst) {
        const char *q = static_cast<const char *>(a.query) +
                        ((long long)c_s * a.q_s + (long long)c_kvh * G * a.q_h) * Tr::kElt;
        if (a.q_heads_contiguous) {
          bulk_copy_g2s(stage + 8192, q, Tr::kQBytes, bars + slot);
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h)
            bulk_copy_g2s(stage + 8192 + h * Tr::kRow, q + (long long)h * a.q_h * Tr::kElt,
                          Tr::kRow, bars + slot);
        }
      }
    }
    ++issued;
    if (issued < n) {
      // advance the cursor and prefetch the next chunk's block ids
      if (++c_i == c_nch) {
        c_i = 0;
        c_base += c_nch;
        if (++c_kvh == Hkv) {
          c_kvh = 0;
          ++c_s;
          c_len = c_next_len;
          while (c_len == 0 && c_s + 1 < S) {
            ++c_s;
            c_len = clamp_len(__ldg(a.context_lens + c_s), max_len);
          }
          c_nch = (c_len + CH - 1) / CH;
          c_next_len = (c_s + 1 < S) ? clamp_len(__ldg(a.context_lens + c_s + 1), max_len) : 0;
        }
        c_first_worker = worker_of(c_base, C, W);
        c_npieces = worker_of(c_base + c_nch - 1, C, W) - c_first_worker + 1;
      }
      fetch_blocks();
    }
  };

  const long long prime = n < ST ? n : ST;
  for (long long i = 0; i < prime; ++i) issue((int)i);

  // per-lane roles
  const int r = lane / RL;       // row within a warp step
  const int j = lane % RL;       // 16-byte column of the row
  const int hh = j / HL;         // head this lane owns after the transposed reduce
  float2 q2[G][EPL / 2];
  float2 acc[G][EPL / 2];
  float m_ref = -INFINITY;
  float lsum = 0.f;

  for (long long c = 0; c < n; ++c) {
    const int slot = (int)(c % ST);
    const uint32_t parity = (uint32_t)((c / ST) & 1);
    if (!mbar_wait_bounded(bars + slot, parity, a.wait_cycles)) {
      // a copy never completed: record it, let the copies already issued land, and stop.
      if (lane == 0) set_error(a.err, PA_DEVERR_TIMEOUT);
      for (long long k = c; k < issued; ++k)
        mbar_wait_bounded(bars + (int)(k % ST), (uint32_t)((k / ST) & 1), a.wait_cycles);
      return;
    }
    const ChunkMeta m = meta[slot];
    const unsigned char *stage = wsm + slot * Tr::kStageBytes;
    if (m.flags & kFirst) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float qf[EPL];
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(stage + 8192 + h * Tr::kRow + j * 16), qf);
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) {
          q2[h][e] = make_float2(qf[2 * e] * a.scale_log2, qf[2 * e + 1] * a.scale_log2);
          acc[h][e] = make_float2(0.f, 0.f);
        }
      }
      m_ref = -INFINITY;
      lsum = 0.f;
    }

    // ---- logits: one (row, head) per lane after the reduce ----
    const unsigned char *Ks = stage;
    const unsigned char *Vs = stage + 4096;
    float sl[STEPS];
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const int row = st * TPS + r;
      float kf[EPL];
      Elem<T>::unpack(*reinterpret_cast<const uint4 *>(Ks + row * Tr::kRow + j * 16), kf);
      float part[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 x = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) x = ffma2(q2[h][e], make_float2(kf[2 * e], kf[2 * e + 1]), x);
        part[h] = x.x + x.y;
      }
      TransposeReduce<G, RL / 2>::run(part, lane);
      sl[st] = part[0];
    }
    const int tok0 = m.chunk * CH;
    const bool tail = tok0 + CH > m.len;
    if (tail) {
#pragma unroll
      for (int st = 0; st < STEPS; ++st)
        if (tok0 + st * TPS + r >= m.len) sl[st] = -INFINITY;
    }

    // ---- online softmax with a lazily moved reference maximum ----
    float cmax = sl[0];
#pragma unroll
    for (int st = 1; st < STEPS; ++st) cmax = fmaxf(cmax, sl[st]);
#pragma unroll
    for (int off = RL; off < 32; off <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(FULL_MASK, cmax, off));
    if (__any_sync(FULL_MASK, cmax > m_ref + 8.f)) {
      const float m_new = fmaxf(m_ref, cmax);
      const float alpha = fast_exp2(m_ref - m_new);
      m_ref = m_new;
      lsum *= alpha;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ah = __shfl_sync(FULL_MASK, alpha, h * HL);
        const float2 a2 = make_float2(ah, ah);
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) acc[h][e] = __fmul2_rn(acc[h][e], a2);
      }
    }
    float psum = 0.f;
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      sl[st] = fast_exp2(sl[st] - m_ref);
      psum += sl[st];
    }
    lsum += psum;
    if (j % HL == 0) {
#pragma unroll
      for (int st = 0; st < STEPS; ++st) pbuf[(st * TPS + r) * G + hh] = sl[st];
    }
    __syncwarp();

    // ---- P.V ----
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const int row = st * TPS + r;
      float vf[EPL];
      Elem<T>::unpack(*reinterpret_cast<const uint4 *>(Vs + row * Tr::kRow + j * 16), vf);
      if (tail && tok0 + row >= m.len) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) vf[e] = 0.f;
      }
      float pp[G];
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int h = 0; h < G; h += 4) {
          const float4 p4 = *reinterpret_cast<const float4 *>(pbuf + row * G + h);
          pp[h] = p4.x;
          pp[h + 1] = p4.y;
          pp[h + 2] = p4.z;
          pp[h + 3] = p4.w;
        }
      } else if constexpr (G == 2) {
        const float2 p2 = *reinterpret_cast<const float2 *>(pbuf + row * G);
        pp[0] = p2.x;
        pp[1] = p2.y;
      } else {
        pp[0] = pbuf[row];
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float2 p2 = make_float2(pp[h], pp[h]);
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e)
          acc[h][e] = ffma2(p2, make_float2(vf[2 * e], vf[2 * e + 1]), acc[h][e]);
      }
    }

    // ---- end of a piece: write the rows, or store the piece and maybe merge ----
    if (m.flags & kLast) {
      float lt = lsum;
#pragma unroll
      for (int off = RL; off < 32; off <<= 1) {
        lt += __shfl_xor_sync(FULL_MASK, lt, off);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e) {
            acc[h][e].x += __shfl_xor_sync(FULL_MASK, acc[h][e].x, off);
            acc[h][e].y += __shfl_xor_sync(FULL_MASK, acc[h][e].y, off);
          }
      }
      float lh[G], mh[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        lh[h] = __shfl_sync(FULL_MASK, lt, h * HL);
        mh[h] = __shfl_sync(FULL_MASK, m_ref, h * HL);
      }
      if (a.separate_reduce && (m.flags & kPairStart) && lane == 0)
        a.pair_meta[m.pair] = make_int2(m.first_worker, m.npieces);
      if (m.npieces == 1) {
        if (r == 0) {
          const int out_elt = a.out_dtype == PA_F32 ? 4 : 2;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float v[EPL];
            const float inv = 1.f / lh[h];
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) {
              v[2 * e] = acc[h][e].x * inv;
              v[2 * e + 1] = acc[h][e].y * inv;
            }
            char *dst = static_cast<char *>(a.out) +
                        ((long long)m.s * a.out_s + (long long)(m.kvh * G + h) * a.out_h + j * EPL) *
                            out_elt;
            store_row_piece(dst, a.out_dtype, v, EPL);
          }
        }
      } else {
        const long long seg = (long long)m.pair + gw;
        if (r == 0) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float inv = 1.f / lh[h];
            float4 *o = reinterpret_cast<float4 *>(a.part_o + (seg * G + h) * D + j * EPL);
#pragma unroll
            for (int e = 0; e < EPL / 2; e += 2)
              o[e / 2] = make_float4(acc[h][e].x * inv, acc[h][e].y * inv, acc[h][e + 1].x * inv,
                                     acc[h][e + 1].y * inv);
          }
        }
        if (lane < G) {
          float2 ml;
          ml.x = mh[0];
          ml.y = lh[0];
#pragma unroll
          for (int h = 1; h < G; ++h)
            if (lane == h) {
              ml.x = mh[h];
              ml.y = lh[h];
            }
          *reinterpret_cast<float2 *>(a.part_ml + (seg * G + lane) * 2) = ml;
        }
        if (!a.separate_reduce) {
          __threadfence();
          __syncwarp();
          unsigned int ticket = 0;
          if (lane == 0) ticket = atomicAdd(a.counters + m.pair, 1u);
          ticket = __shfl_sync(FULL_MASK, ticket, 0);
          if (ticket == (unsigned int)(m.npieces - 1)) {
            __threadfence();
            merge_pieces<Tr>(a, m.pair, m.first_worker, m.npieces, m.s, m.kvh, lane);
            if (lane == 0) a.counters[m.pair] = 0u;
          }
        }
      }
    }
    __syncwarp();
    if (issued < n) issue(slot);
  }
}

// Separate merge: one warp per (sequence, kv head); pairs covered by one warp were written by
// the decode kernel already.
template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(128) paged_decode_merge_kernel(const DecodeArgs a) {
  using Tr = DecodeTraits<T, D, BS, G>;
  const int lane = threadIdx.x & 31;
  const long long pairs = (long long)a.num_seqs * a.num_kv_heads;
  const int max_len = a.max_blocks * BS;
  for (long long p = (long long)blockIdx.x * 4 + (threadIdx.x >> 5); p < pairs;
       p += (long long)gridDim.x * 4) {
    const int s = (int)(p / a.num_kv_heads);
    const int kvh = (int)(p % a.num_kv_heads);
    if (clamp_len(__ldg(a.context_lens + s), max_len) == 0) continue;
    const int2 pm = a.pair_meta[p];
    if (pm.y <= 1) continue;
    merge_pieces<Tr>(a, (int)p, pm.x, pm.y, s, kvh, lane);
  }
}

template <typename T, int D, int BS, int G>
cudaError_t launch_decode(const DecodeArgs &a, int num_ctas, cudaStream_t st) {
  using Tr = DecodeTraits<T, D, BS, G>;
  paged_decode_kernel<T, D, BS, G><<<num_ctas, Tr::kWarps * 32, Tr::kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D, int BS, int G>
cudaError_t launch_decode_merge(const DecodeArgs &a, cudaStream_t st) {
  const long long pairs = (long long)a.num_seqs * a.num_kv_heads;
  long long blocks = (pairs + 3) / 4;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  paged_decode_merge_kernel<T, D, BS, G><<<(int)blocks, 128, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D, int BS, int G>
bool make_decode_kernel(DecodeKernel *k) {
  using Tr = DecodeTraits<T, D, BS, G>;
  // The shared-memory opt-in is a per-device function attribute: set it once per device.
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(paged_decode_kernel<T, D, BS, G>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Tr::kSmemBytes) != cudaSuccess)
      return false;
    configured[dev] = true;
  }
  k->launch = &launch_decode<T, D, BS, G>;
  k->launch_reduce = &launch_decode_merge<T, D, BS, G>;
  k->kernel = reinterpret_cast<const void *>(&paged_decode_kernel<T, D, BS, G>);
  k->warps_per_cta = Tr::kWarps;
  k->smem_bytes = Tr::kSmemBytes;
  k->chunk_tokens = Tr::kChunk;
  return true;
}

// Table over block_size {8, 16, 32} x group {1, 2, 4, 8} for one element type and head_dim.
template <typename T, int D>
bool decode_kernel_table(int block_size, int group, DecodeKernel *k) {
#define PA_CASE(BB, GG) \
  if (block_size == BB && group == GG) return make_decode_kernel<T, D, BB, GG>(k);
#define PA_GROUPS(BB) PA_CASE(BB, 1) PA_CASE(BB, 2) PA_CASE(BB, 4) PA_CASE(BB, 8)
  PA_GROUPS(8)
  PA_GROUPS(16)
  PA_GROUPS(32)
#undef PA_GROUPS
#undef PA_CASE
  return false;
}

}  // namespace pa

// pa_prefill_tc.cuh - causal attention of a step's new tokens over the paged cache (prefill, or
// a chunk of a prompt in a continuously batched step) on the fifth-generation tensor cores:
// tcgen05 MMAs from shared memory into tensor memory.
//
// Sources: [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization
// support, distributed inference" 4.2 (at each iteration requests join the running batch: a
// joining request's prompt tokens are that step's new tokens) and [P4] "vLLM core
// architecture: model loading, PagedAttention principle, KV cache management" 2.2.2 (attention
// assembles the whole KV sequence through the block table).  Token j of sequence s's q_len new
// tokens sits at position p = context_len - q_len + j and attends to positions 0 .. p.
//
// A tile is 128 query rows of one (sequence, kv head): 128 / G new tokens times the G query
// heads that read that kv head (head fastest), one row per tensor-memory lane.  The context is
// walked in kv tiles of 128 positions.  One persistent CTA per SM, eleven warps:
//   * warp 8 streams the tile's query rows (one 4-D box, loaded as soon as the previous tile's
//     last S = QK^T is done, so it overlaps that tile's end) and the key tiles, warp 10 the
//     value tiles (so keys run ahead of the values, which free later), through two-slot rings
//     by TMA: one box per (block, kv head) tile of the paged cache, 128-byte swizzle, in 8-row
//     groups placed one after another, which is the operand layout of the MMAs; the lanes issue
//     the boxes of a kv tile together;
//   * warp 9 (one lane) issues the MMAs: S = Q K^T (M = 128 rows, N = 128 positions, K = head
//     dim) into one of two S buffers in tensor memory, and O += P V (N = head dim, K = 128
//     positions) into the O accumulator, P split into two 16-bit terms (hi + lo) as in the
//     decode kernels so the weights keep about 16 significant bits;
//   * warps 0-7 run the softmax, two threads per row: warp w reads tensor-memory lanes
//     32 (w % 4) .. + 31 and the half w / 4 of the kv tile's columns of S.  Each thread masks
//     its columns causally (which also hides positions past the context), keeps the online
//     softmax of its half of the row in base 2 against a reference maximum the two halves
//     share (exchanged through shared memory; moved only when a logit passes it by 2^8, when O
//     is rescaled in tensor memory) and writes its part of P into tensor memory over its own S
//     columns, where the MMA reads it as the A operand; at the end of the tile the halves add
//     their row sums and each stores half of the row of O / l.
// The MMA warp issues S of kv tile j + 1 before O += P V of tile j, and S / P has two buffers,
// so the tensor cores compute the next scores and the previous products while the softmax warps
// work on the current scores.  Q, K and V are the only shared-memory operands, which leaves the
// shared-memory bandwidth to the MMAs' operand reads.  Barriers between the roles are mbarriers
// (copies: transaction bytes; MMAs: tcgen05.commit; threads: arrival counts); every wait is
// bounded and a timeout sets an error bit and winds the CTA down.
//
// Tiles differ in cost (a tile's causal prefix), so they are spread longest first: every CTA
// builds the same list of (sequence, tile) pairs sorted by cost (a histogram of costs in shared
// memory, a prefix over it, a scatter) and takes positions of the list in snake order (round r
// gives CTA i position r*P + i, or r*P + P-1-i when r is odd).  Ties land in any order: each
// tile's rows are computed by one CTA alone, so the order changes no result.  Steps too large
// for the shared list fall back to tiles in sequence order, x = blockIdx.x, += gridDim.x, each
// warp finding the (sequence, tile) of x by a scan of query_start.
#pragma once

#include "pa_decode_mma.cuh"
#include "pa_prefill_internal.h"
#include "pa_tc.cuh"

namespace pa {

// One box of a 4-D tensor map (the prefill's query rows) into shared memory.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            int c3, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

template <int D, int BS, int G>
struct PrefillTcTraits {
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
  static constexpr int kProducerWarp = 8;  // query rows and key tiles
  static constexpr int kMmaWarp = 9;
  static constexpr int kValueWarp = 10;    // value tiles
  static constexpr int kThreads = 352;
  static constexpr int kRows = 128;             // query rows of a tile (MMA M)
  static constexpr int kTokens = kRows / G;     // new tokens of a tile
  static constexpr int kKv = 128;               // context positions of a kv tile
  static constexpr int kCols = kKv / 2;         // S columns per softmax thread
  static constexpr int kSpans = D / 64;
  static constexpr int kGroup = kSpans * 1024;  // bytes between 8-row groups of K, V tiles
  static constexpr int kQBytes = kRows * D * 2; // span-major: 128 rows of a span, then the next
  static constexpr int kKvBytes = kKv * D * 2;
  static constexpr int kBoxBytes = 8 * D * 2;      // 8 positions, both spans
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kStages = 2;             // key and value rings
  static constexpr int kVOff = kKOff + kStages * kKvBytes;
  static constexpr int kBarOff = kVOff + kStages * kKvBytes;
  static constexpr int kNumBars = 28;
  static constexpr int kInfoOff = kBarOff + kNumBars * 8;  // [tmem base, abort, tile count, rounds]
  static constexpr int kXchOff = kInfoOff + 32;            // float [2 parities][2 halves][128 rows]
  static constexpr int kMaxMine = 64;                      // rounds of the sorted schedule
  static constexpr int kMineOff = kXchOff + 2 * 2 * kRows * 4;
  static constexpr int kSmemBytes = kMineOff + kMaxMine * 8 + 1024;  // + 1 KB alignment
  // the sorted schedule's scratch (histogram of costs, tile list) lives in the key and value
  // rings before the first copy
  static constexpr int kMaxBins = 2048;  // costs 0 .. 2047 (16-position steps)
  static constexpr int kMaxList = 4096;  // (sequence, tile) pairs
  // tensor memory: S0 [0, kKv), S1 [kKv, 2 kKv), O [2 kKv, 2 kKv + D).  P of a kv tile replaces
  // its S: each softmax half's kCols columns hold the hi terms of its positions (two 16-bit
  // values per column, the A operand of O += P V), then the lo terms
  static constexpr int kOCol = 2 * kKv;
  static constexpr int kTmemCols = kOCol + D <= 256 ? 256 : 512;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "1, 2, 4 or 8 query heads per kv head");
  static_assert(BS % 8 == 0 && kKv % BS == 0, "block size a multiple of the 8-position box");
  static_assert((kMaxBins + kMaxList) * 4 <= 2 * kStages * kKvBytes, "schedule scratch fits the rings");
  static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
};

// Warp-cooperative: the sequence holding tile y of the step (tiles ordered by sequence, then
// position) and the tile's index within it; s = -1 when y is past the last tile.
template <int TOK>
__device__ __forceinline__ void locate_tile_tc(const PrefillArgs &a, long long y, int &s_out,
                                               int &tau_out) {
  const int lane = threadIdx.x & 31;
  long long running = 0;
  for (int base = 0; base < a.num_seqs; base += 32) {
    const int s = base + lane;
    int cnt = 0;
    if (s < a.num_seqs) {
      const int q_len = __ldg(a.query_start + s + 1) - __ldg(a.query_start + s);
      cnt = q_len > 0 ? (q_len + TOK - 1) / TOK : 0;
    }
    long long incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long v = __shfl_up_sync(FULL_MASK, incl, off);
      if (lane >= off) incl += v;
    }
    const long long total = __shfl_sync(FULL_MASK, incl, 31);
    if (running + total > y) {
      const bool hit = running + incl - cnt <= y && y < running + incl;
      const int src = __ffs(__ballot_sync(FULL_MASK, hit)) - 1;
      s_out = base + src;
      tau_out = (int)(y - running - __shfl_sync(FULL_MASK, incl - cnt, src));
      return;
    }
    running += total;
  }
  s_out = -1;
  tau_out = 0;
}

// The per-tile quantities every role derives the same way.
struct TcTile {
  int s, tau, kvh;
  int q0, q_len, L;
  int tok0, ntok, pos0, n_kv;
  bool valid;
  int j0;          // first kv tile of the item (0 unless the shared-prefix pass splits the range)
  int slot;        // the item's slot among a (sequence, head)'s partial results (prefix pass)
  bool noncausal;  // every row sees positions 0 .. L-1 (prefix pass)
};

// Shared-prefix pass: the prefix length of group g (that of its first member, clamped to the
// block table) and its members; 0 members when the group is malformed.
__device__ __forceinline__ void prefix_group(const PrefillArgs &a, int g, int max_len, int &first,
                                             int &members, int &P) {
  first = __ldg(a.group_start + g);
  const int end = __ldg(a.group_start + g + 1);
  members = end - first;
  P = 0;
  if (first < 0 || members < 0 || (long long)end > a.num_tokens) {
    members = 0;
    return;
  }
  if (members > 0) {
    const int raw = __ldg(a.prefix_lens + first);
    P = raw < 0 ? 0 : (raw > max_len ? max_len : raw);
  }
}

// Warp-cooperative: the group holding item y of the shared-prefix pass (items ordered by
// group, then kv head, row tile, split) and y's index within the group; g = -1 past the end.
template <int TOK, int KV>
__device__ __forceinline__ void locate_prefix_item(const PrefillArgs &a, int max_len, long long y,
                                                   int &g_out, long long &rem_out) {
  const int lane = threadIdx.x & 31;
  long long running = 0;
  for (int base = 0; base < a.num_groups; base += 32) {
    const int g = base + lane;
    long long cnt = 0;
    if (g < a.num_groups) {
      int first, members, P;
      prefix_group(a, g, max_len, first, members, P);
      if (members > 0 && P > 0) {
        const int splits = ((P + KV - 1) / KV + a.pre_kv - 1) / a.pre_kv;
        cnt = (long long)((members + TOK - 1) / TOK) * a.num_kv_heads * splits;
      }
    }
    long long incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long v = __shfl_up_sync(FULL_MASK, incl, off);
      if (lane >= off) incl += v;
    }
    const long long total = __shfl_sync(FULL_MASK, incl, 31);
    if (running + total > y) {
      const bool hit = running + incl - cnt <= y && y < running + incl;
      const int src = __ffs(__ballot_sync(FULL_MASK, hit)) - 1;
      g_out = base + src;
      rem_out = y - running - __shfl_sync(FULL_MASK, incl - cnt, src);
      return;
    }
    running += total;
  }
  g_out = -1;
  rem_out = 0;
}

// Two 16-bit terms of a pair of weights: hi = round(p), lo = round(p - hi).
template <bool kBf16>
__device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo) {
  if constexpr (kBf16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
  } else {
    const __half2 h = __floats2half2_rn(x, y);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
  }
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(PrefillTcTraits<D, BS, G>::kThreads, 1)
    paged_prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  using Tr = PrefillTcTraits<D, BS, G>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Tr::kBarOff);
  // rings of kStages slots (key, value tiles) and of two (S, P buffers)
  uint64_t *k_full = bars + 0, *k_empty = bars + 3, *v_full = bars + 6, *v_empty = bars + 9;
  uint64_t *s_full = bars + 12, *s_free = bars + 14, *p_ready = bars + 16, *pv_done = bars + 18;
  uint64_t *q_full = bars + 20, *q_empty = bars + 21, *fin = bars + 22;
  uint64_t *xbar = bars + 23;  // per row quarter: the exchanges between its two softmax warps
  volatile int *info = reinterpret_cast<volatile int *>(smem + Tr::kInfoOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Tr::kInfoOff);
  int2 *mine = reinterpret_cast<int2 *>(smem + Tr::kMineOff);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int wid = tid >> 5;
  const int Hkv = a.num_kv_heads;
  const int max_len = a.max_blocks * BS;

  if (tid == 0) {
    for (int i = 0; i < Tr::kStages; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, Tr::kSoftmaxThreads);
      mbar_init(p_ready + i, Tr::kSoftmaxThreads);
      mbar_init(pv_done + i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(fin, 1);
    for (int i = 0; i < 4; ++i) mbar_init(xbar + i, 64);
    fence_barrier_init();
    info[1] = 0;
    info[2] = 0;
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.v)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.q)) : "memory");
  }
  if (wid == Tr::kMmaWarp) {
    tc::alloc(tmem_slot, Tr::kTmemCols);
    tc::relinquish();
  }
  // a grid launched after this one to overlap it (the decode after the shared-prefix pass)
  // may start: it reads nothing this grid writes before it waits for this grid to finish
  if (tid == 0) allow_next_grid();

  // ---- the longest-first schedule (scratch in the key ring) ----
  int *bins = reinterpret_cast<int *>(smem + Tr::kKOff);
  int *list = bins + Tr::kMaxBins;
  const int nbins = (max_len + 15) / 16 + 1;
  const bool prefix_pass = a.pre_o != nullptr;
  bool sorted = !prefix_pass && nbins <= Tr::kMaxBins && a.num_seqs < (1 << 19);
  if (sorted)
    for (int i = tid; i < nbins; i += Tr::kThreads) bins[i] = 0;
  __syncthreads();
  auto seq_tiles = [&](int sq, int &len_out, int &q_out) {
    const int q0s = __ldg(a.query_start + sq);
    const int qn = __ldg(a.query_start + sq + 1) - q0s;
    const int raw = __ldg(a.context_lens + sq);
    const int Ls = raw < 0 ? 0 : (raw > max_len ? max_len : raw);
    len_out = Ls;
    q_out = qn;
    if (qn > Ls || q0s < 0 || (long long)q0s + qn > a.num_tokens) return -1;  // invalid
    return qn > 0 ? (qn + Tr::kTokens - 1) / Tr::kTokens : 0;
  };
  auto tile_cost = [&](int Ls, int qn, int t) {
    const int last = min((t + 1) * Tr::kTokens, qn);  // tokens up to this tile's last one
    return (Ls - qn + last + 15) / 16;
  };
  if (sorted) {
    for (int sq = tid; sq < a.num_seqs; sq += Tr::kThreads) {
      int Ls, qn;
      const int nt = seq_tiles(sq, Ls, qn);
      if (nt < 0) {
        // new tokens outside the context, or query rows outside the query tensor: report
        set_error(a.err, PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      for (int t = 0; t < nt && t < Tr::kMaxList; ++t) atomicAdd(bins + tile_cost(Ls, qn, t), 1);
      atomicAdd((int *)info + 2, nt);
    }
  }
  __syncthreads();
  const int ntiles = sorted ? info[2] : 0;
  const long long total = (long long)ntiles * Hkv;
  sorted = sorted && ntiles <= Tr::kMaxList && total <= (long long)Tr::kMaxMine * gridDim.x;
  if (sorted && wid == 0) {
    // bins[c] <- number of tiles costing more than c: where the tiles of cost c start
    const int seg = (nbins + 31) / 32;
    const int hi = nbins - 1 - lane * seg;  // this lane's costs: hi, hi-1, .., hi-seg+1
    int sum = 0;
    for (int i = 0; i < seg; ++i)
      if (hi - i >= 0) sum += bins[hi - i];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(FULL_MASK, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
    for (int i = 0; i < seg; ++i)
      if (hi - i >= 0) {
        const int n = bins[hi - i];
        bins[hi - i] = run;
        run += n;
      }
  }
  __syncthreads();
  if (sorted) {
    for (int sq = tid; sq < a.num_seqs; sq += Tr::kThreads) {
      int Ls, qn;
      const int nt = seq_tiles(sq, Ls, qn);
      for (int t = 0; t < nt; ++t) list[atomicAdd(bins + tile_cost(Ls, qn, t), 1)] = (sq << 12) | t;
    }
  }
  __syncthreads();
  if (sorted && tid < Tr::kMaxMine) {
    const long long r = tid;
    const long long k = r * gridDim.x + ((r & 1) ? (long long)gridDim.x - 1 - blockIdx.x : (long long)blockIdx.x);
    if (k < total) mine[r] = make_int2(list[k / Hkv], (int)(k % Hkv));
  }
  if (tid == 0) {
    // every round but the last is full; in the last one this CTA's position depends on the
    // direction of the snake
    long long rounds = 0;
    if (sorted) {
      const long long full = total / gridDim.x, rem = total % gridDim.x;
      const long long at = (full & 1) ? (long long)gridDim.x - 1 - blockIdx.x : (long long)blockIdx.x;
      rounds = full + (at < rem ? 1 : 0);
    }
    info[3] = (int)rounds;
  }
  // the scratch is overwritten by copies from here on
  fence_proxy_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  const int my_rounds = info[3];

  // The tile of round `round` (whole warp calls it); false when this CTA has no more tiles.
  auto next_tile = [&](long long round, TcTile &t) -> bool {
    t.j0 = 0;
    t.slot = 0;
    t.noncausal = false;
    if (prefix_pass) {
      int g;
      long long rem;
      locate_prefix_item<Tr::kTokens, Tr::kKv>(a, max_len, blockIdx.x + round * gridDim.x, g, rem);
      if (g < 0) return false;
      int first, members, P;
      prefix_group(a, g, max_len, first, members, P);
      const int kv_tiles = (P + Tr::kKv - 1) / Tr::kKv;
      const int splits = (kv_tiles + a.pre_kv - 1) / a.pre_kv;
      const int row_tiles = (members + Tr::kTokens - 1) / Tr::kTokens;
      t.slot = (int)(rem % splits);
      rem /= splits;
      t.tau = (int)(rem % row_tiles);
      t.kvh = (int)(rem / row_tiles);
      t.s = first;  // the prefix is read through the first member's block table
      t.q0 = first;
      t.q_len = members;
      t.L = P;
      t.valid = t.slot < a.pre_splits;
      t.tok0 = t.tau * Tr::kTokens;
      t.ntok = min(Tr::kTokens, members - t.tok0);
      t.pos0 = 0;
      t.j0 = t.slot * a.pre_kv;
      t.n_kv = t.valid ? min(a.pre_kv, kv_tiles - t.j0) : 0;
      t.noncausal = true;
      return true;
    }
    if (sorted) {
      if (round >= my_rounds) return false;
      const int2 e = mine[round];
      t.s = e.x >> 12;
      t.tau = e.x & 4095;
      t.kvh = e.y;
    } else {
      const long long x = blockIdx.x + round * gridDim.x;
      int ls, lt;
      locate_tile_tc<Tr::kTokens>(a, x / Hkv, ls, lt);
      if (ls < 0) return false;
      t.s = ls;
      t.tau = lt;
      t.kvh = (int)(x % Hkv);
    }
    t.q0 = __ldg(a.query_start + t.s);
    t.q_len = __ldg(a.query_start + t.s + 1) - t.q0;
    const int raw = __ldg(a.context_lens + t.s);
    t.L = raw < 0 ? 0 : (raw > max_len ? max_len : raw);
    t.valid = !(t.q_len > t.L || t.q0 < 0 || (long long)t.q0 + t.q_len > a.num_tokens);
    t.tok0 = t.tau * Tr::kTokens;
    t.ntok = min(Tr::kTokens, t.q_len - t.tok0);
    t.pos0 = t.L - t.q_len + t.tok0;
    t.n_kv = t.valid ? (t.pos0 + t.ntok + Tr::kKv - 1) / Tr::kKv : 0;
    return true;
  };
  // A bounded wait that also gives up once another role has aborted.
  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
      if (mbar_try_wait(bar, parity)) return true;
      if (info[1] != 0) return false;
      if (clock64() - t0 > a.wait_cycles) {
        set_error(a.err, PA_DEVERR_TIMEOUT);
        info[1] = 1;
        return false;
      }
    }
  };

  const uint32_t q_s = smem_u32(smem + Tr::kQOff);
  const uint32_t k_s = smem_u32(smem + Tr::kKOff);
  const uint32_t v_s = smem_u32(smem + Tr::kVOff);

  if (wid == Tr::kProducerWarp || wid == Tr::kValueWarp) {
    // ======= producers: query rows and key tiles (warp 8), value tiles (warp 10), by TMA =======
    const int which = wid == Tr::kValueWarp ? 1 : 0;
    long long kv_base = 0, qt = 0;
    long long k_issued = 0, v_issued = 0;
    bool ok = true;
    TcTile t;
    for (long long round = 0; ok && next_tile(round, t); ++round) {
      if (!t.valid) {
        if (lane == 0 && t.tau == 0 && t.kvh == 0)
          set_error(a.err, t.noncausal ? PA_DEVERR_PREFIX : PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      if (which == 0) {
        // the tile's query rows: tokens q0 + tok0 .. + 128/G of heads kvh*G .. + G (rows past
        // the tensor read as zeros, rows of the next sequence are computed and dropped), once
        // the previous tile's S = QK^T are all done
        bool q_ok = true;
        if (lane == 0) {
          q_ok = qt < 1 || wait(q_empty, (uint32_t)((qt - 1) & 1));
          if (q_ok) {
            mbar_arrive_expect_tx(q_full, Tr::kQBytes);
            tma_load_4d(q_s, &maps.q, 0, t.kvh * G, t.q0 + t.tok0, 0, q_full);
          }
        }
        if (__shfl_sync(FULL_MASK, q_ok ? 1 : 0, 0) == 0) {
          ok = false;
          break;
        }
        ++qt;
      }
      // Block ids of a kv tile: lane i holds the tile's i-th block (at most 16 blocks).  The
      // ids of tile j + 1 are fetched before the waits of tile j, so their latency is hidden.
      const int32_t *row = a.block_tables + (long long)t.s * a.bt_s;
      auto fetch_ids = [&](int j) {
        const int p0 = (t.j0 + j) * Tr::kKv;
        const int nblk = (min(p0 + Tr::kKv, t.L) - p0 + BS - 1) / BS;
        int blk = 0;
        if (lane < nblk) {
          blk = __ldg(row + p0 / BS + lane);
          if (blk < 0 || (long long)blk >= a.num_blocks) {
            set_error(a.err, PA_DEVERR_BLOCK_ID);
            blk = 0;
          }
        }
        return blk;
      };
      int cur = fetch_ids(0);
      for (int j = 0; j < t.n_kv && ok; ++j) {
        const int nxt = j + 1 < t.n_kv ? fetch_ids(j + 1) : 0;
        const long long it = kv_base + j;
        const int b = (int)(it % Tr::kStages);
        const long long use = it / Tr::kStages;
        const int p0 = (t.j0 + j) * Tr::kKv;
        const int pend = min(p0 + Tr::kKv, t.L);
        const int nblk = (pend - p0 + BS - 1) / BS;
        const uint32_t bytes = (uint32_t)(a.grouped_maps ? nblk * (BS / 8) : (pend - p0 + 7) / 8) * Tr::kBoxBytes;
        {
          uint64_t *full = which ? v_full + b : k_full + b;
          uint64_t *empty = which ? v_empty + b : k_empty + b;
          bool w_ok = true;
          if (lane == 0) {
            w_ok = use < 1 || wait(empty, (uint32_t)((use - 1) & 1));
            if (w_ok) mbar_arrive_expect_tx(full, bytes);
          }
          if (__shfl_sync(FULL_MASK, w_ok ? 1 : 0, 0) == 0) {
            ok = false;
            continue;
          }
          const uint32_t dst = (which ? v_s : k_s) + b * Tr::kKvBytes;
          const CUtensorMap *map = which ? &maps.v : &maps.k;
          if (a.grouped_maps) {
            // lane i copies the tile's i-th (block, kv head) tile, rows past the context
            // included: the copies of one kv tile are issued together
            if (lane < nblk)
              tma_load_tile(dst + (lane * BS / 8) * Tr::kBoxBytes, map, 0, 0, cur * Hkv + t.kvh, full);
          } else {
            for (int bi = 0; bi < nblk; ++bi) {
              const int blk = __shfl_sync(FULL_MASK, cur, bi);
              if (lane == 0) {
                const int p = p0 + bi * BS;
                for (int y = 0; y < BS && p + y < pend; y += 8)
                  tma_load_tile(dst + ((p + y - p0) / 8) * Tr::kBoxBytes, map, y, t.kvh, blk, full);
              }
            }
          }
          if (which) ++v_issued; else ++k_issued;
        }
        cur = nxt;
      }
      ok = __shfl_sync(FULL_MASK, ok ? 1 : 0, 0) != 0;
      if (t.noncausal && which == 1 && t.kvh == 0) {
        // shared-prefix pass: the members of this tile must name the first member's prefix
        // length and, over this item's positions, its physical blocks (kv head 0's items check,
        // once their value copies are issued: the check only reports)
        const int32_t *row0 = a.block_tables + (long long)t.s * a.bt_s;
        const int b0 = t.j0 * Tr::kKv / BS;
        const int b1 = (min((t.j0 + t.n_kv) * Tr::kKv, t.L) + BS - 1) / BS;
        bool bad = false;
        for (int m = t.tok0 + lane; m < t.tok0 + t.ntok; m += 32) {
          const int sq = t.q0 + m;
          if (sq == t.s) continue;
          if (__ldg(a.prefix_lens + sq) != __ldg(a.prefix_lens + t.s)) bad = true;
          const int32_t *row = a.block_tables + (long long)sq * a.bt_s;
          for (int b = b0; b < b1; ++b)
            if (__ldg(row + b) != __ldg(row0 + b)) bad = true;
        }
        if (bad) set_error(a.err, PA_DEVERR_PREFIX);
        if (lane == 0 && t.L % BS != 0) set_error(a.err, PA_DEVERR_PREFIX);
      }
      kv_base += t.n_kv;
    }
    if (lane == 0 && !ok) {
      // let the copies in flight land before the CTA leaves
      if (qt > 0) mbar_wait_bounded(q_full, (uint32_t)((qt - 1) & 1), a.wait_cycles);
      constexpr int S = Tr::kStages;
      for (long long i = k_issued > S ? k_issued - S : 0; i < k_issued; ++i)
        mbar_wait_bounded(k_full + (int)(i % S), (uint32_t)((i / S) & 1), a.wait_cycles);
      for (long long i = v_issued > S ? v_issued - S : 0; i < v_issued; ++i)
        mbar_wait_bounded(v_full + (int)(i % S), (uint32_t)((i / S) & 1), a.wait_cycles);
    }
  } else if (wid == Tr::kMmaWarp) {
    // ================= MMA issue =================
    constexpr uint32_t kIdS = tc::idesc_f16(kBf16, 128, Tr::kKv, false);
    constexpr uint32_t kIdO = tc::idesc_f16(kBf16, 128, D, true);
    long long kv_base = 0;
    long long qt = 0;
    bool ok = true;
    TcTile t;
    auto pv = [&](int j) -> bool {
      const long long it = kv_base + j;
      const int b = (int)(it & 1);               // P buffer
      const int vs = (int)(it % Tr::kStages);    // value slot
      if (!wait(p_ready + b, (uint32_t)((it >> 1) & 1)) ||
          !wait(v_full + vs, (uint32_t)((it / Tr::kStages) & 1)))
        return false;
      tc::fence_after();
      const uint32_t vb = v_s + vs * Tr::kKvBytes;
#pragma unroll
      for (int kt = 0; kt < Tr::kKv / 16; ++kt) {
        const uint64_t vd = tc::smem_desc(vb + kt * 2 * Tr::kGroup, 1024, Tr::kGroup);
        // positions 16 kt .. + 15 belong to the softmax half h, offset o within it: their hi
        // terms sit at column kCols h + o / 2 of S buffer b, the lo terms kCols / 2 further
        const int h = (16 * kt) / Tr::kCols, o = 16 * kt - h * Tr::kCols;
        const uint32_t pc = tmem + Tr::kKv * b + Tr::kCols * h + o / 2;
        tc::mma_ts(tmem + Tr::kOCol, pc, vd, kIdO, (j > 0 || kt > 0) ? 1u : 0u);
        tc::mma_ts(tmem + Tr::kOCol, pc + Tr::kCols / 2, vd, kIdO, 1u);
      }
      tc::commit(pv_done + b);
      tc::commit(v_empty + vs);
      return true;
    };
    for (long long round = 0; ok && next_tile(round, t); ++round) {
      if (!t.valid) continue;
      const uint32_t qbuf = q_s;
      if (lane == 0) {
        ok = wait(q_full, (uint32_t)(qt & 1));
        tc::fence_after();
        for (int j = 0; j < t.n_kv && ok; ++j) {
          const long long it = kv_base + j;
          const int b = (int)(it & 1);              // S buffer
          const int ks_ = (int)(it % Tr::kStages);  // key slot
          if (!wait(k_full + ks_, (uint32_t)((it / Tr::kStages) & 1)) ||
              (it >= 2 && !wait(s_free + b, (uint32_t)(((it >> 1) - 1) & 1)))) {
            ok = false;
            break;
          }
          tc::fence_after();
          const uint32_t kb = k_s + ks_ * Tr::kKvBytes;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            // query rows span-major (128 rows of a 64-element span, then the next span), keys
            // in 8-row groups of both spans
            const uint32_t inner = (ks & 3) * 32;
            tc::mma(tmem + Tr::kKv * b, tc::smem_desc(qbuf + (ks >> 2) * (Tr::kRows * 128) + inner, 16, 1024),
                    tc::smem_desc(kb + (ks >> 2) * 1024 + inner, 16, Tr::kGroup), kIdS, ks > 0 ? 1u : 0u);
          }
          tc::commit(s_full + b);
          tc::commit(k_empty + ks_);
          if (j == t.n_kv - 1) tc::commit(q_empty);
          if (j > 0) ok = pv(j - 1);
        }
        if (ok) ok = pv(t.n_kv - 1);
      }
      ok = __shfl_sync(FULL_MASK, ok ? 1 : 0, 0) != 0;
      kv_base += t.n_kv;
      ++qt;
    }
    if (lane == 0) {
      // every MMA issued has completed before tensor memory is released
      tc::commit(fin);
      mbar_wait_bounded(fin, 0, a.wait_cycles);
    }
    __syncwarp();
  } else {
    // ================= softmax, two threads per row =================
    const int quarter = wid & 3, half = wid >> 2;
    const int r = 32 * quarter + lane;  // row = tensor-memory lane
    const int lt = r / G, hh = r % G;
    const uint32_t lane_base = tc::taddr(tmem, 32 * quarter, 0);
    float *xch = reinterpret_cast<float *>(smem + Tr::kXchOff);  // [parity][half][row]
    // The two threads of a row swap a value through shared memory; the two warps of a row
    // quarter meet at their own mbarrier (bounded wait), exchanges alternate between two slots.
    long long nx = 0;  // exchanges so far (the same count in both warps of a quarter)
    auto swap_with_other_half = [&](float mine_v, float &other) -> bool {
      float *xs = xch + (nx & 1) * 2 * Tr::kRows;
      xs[half * Tr::kRows + r] = mine_v;
      mbar_arrive(xbar + quarter);
      const bool got = __all_sync(FULL_MASK, wait(xbar + quarter, (uint32_t)(nx & 1)));
      other = xs[(half ^ 1) * Tr::kRows + r];
      ++nx;
      return got;
    };
    long long kv_base = 0;
    bool ok = true;
    TcTile t;
    for (long long round = 0; ok && next_tile(round, t); ++round) {
      if (!t.valid) continue;
      const bool row_ok = lt < t.ntok;
      const int prow = row_ok ? (t.noncausal ? t.L - 1 : t.pos0 + lt) : -1;
      float m_ref = -INFINITY, l_part = 0.f;
      for (int j = 0; j < t.n_kv; ++j) {
        const long long it = kv_base + j;
        const int b = (int)(it & 1);
        if (!__all_sync(FULL_MASK, wait(s_full + b, (uint32_t)((it >> 1) & 1)))) {
          ok = false;
          break;
        }
        tc::fence_after();
        // this thread's S columns and, later, its P: the hi terms of its kCols positions in the
        // first kCols / 2 of its columns, the lo terms in the rest
        const uint32_t my_cols = lane_base + Tr::kKv * b + Tr::kCols * half;
        const int jj = t.j0 + j;  // the kv tile's index in the context
        const int c_lim = prow - jj * Tr::kKv - Tr::kCols * half;  // this thread's visible columns
        // t = logit * scale_log2 + nm on the visible columns (-inf elsewhere); returns the
        // largest t; with exps leaves 2^t as two 16-bit terms in hw / lw, their sum in l_t
        uint32_t hw[Tr::kCols / 2], lw[Tr::kCols / 2];
        // Only kv tiles that reach past a row's position need the causal mask; when every row
        // of the warp sees all of its columns the pass runs without it
        const bool unmasked = __all_sync(FULL_MASK, c_lim >= Tr::kCols - 1);
        auto pass_as = [&](auto masked, float nm, bool exps, float &l_t) -> float {
          constexpr bool kMasked = decltype(masked)::value;
          float tmax = -INFINITY;
          l_t = 0.f;
#pragma unroll
          for (int q = 0; q < Tr::kCols / 32; ++q) {
            uint32_t sr[32];
            __syncwarp();
            tc::ld32x32(my_cols + 32 * q, sr);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c0 = 32 * q + 2 * i;
              float t0 = fmaf(__uint_as_float(sr[2 * i]), a.scale_log2, nm);
              float t1 = fmaf(__uint_as_float(sr[2 * i + 1]), a.scale_log2, nm);
              if constexpr (kMasked) {
                t0 = c0 <= c_lim ? t0 : -INFINITY;
                t1 = c0 + 1 <= c_lim ? t1 : -INFINITY;
              }
              tmax = fmaxf(tmax, fmaxf(t0, t1));
              if (exps) {
                const float p0 = fast_exp2(t0), p1 = fast_exp2(t1);
                l_t += p0 + p1;
                split2<kBf16>(p0, p1, hw[16 * q + i], lw[16 * q + i]);
              }
            }
          }
          return tmax;
        };
        auto pass = [&](float nm, bool exps, float &l_t) -> float {
          return unmasked ? pass_as(std::false_type{}, nm, exps, l_t) : pass_as(std::true_type{}, nm, exps, l_t);
        };
        // the row's largest t over both halves
        auto row_max = [&](float mine_t, float &both) -> bool {
          float other;
          const bool got = swap_with_other_half(mine_t, other);
          both = fmaxf(mine_t, other);
          return got;
        };
        float l_t, alpha = 1.f;
        bool rescale = false;
        // S may be released once both passes that can read it are behind: the first tile reads
        // it twice (maximum, then weights), a later one once, and a second time on a move
        auto release_s = [&]() {
          tc::fence_before();
          mbar_arrive(s_free + b);
        };
        if (j == 0) {
          // first kv tile: the maximum first, then the weights
          if (!row_max(pass(0.f, false, l_t), m_ref)) {
            ok = false;
            break;
          }
          pass(m_ref == -INFINITY ? 0.f : -m_ref, true, l_t);
          l_part = l_t;
        } else {
          // later tiles: weights against the current reference; a row whose logits pass it by
          // more than 2^8 moves its reference (both halves alike) and takes the pass again
          float tmax;
          if (!row_max(pass(m_ref == -INFINITY ? 0.f : -m_ref, true, l_t), tmax)) {
            ok = false;
            break;
          }
          const bool move = tmax > 8.f;
          if (__any_sync(FULL_MASK, move)) {
            if (move) {
              alpha = fast_exp2(-tmax);
              rescale = true;
              m_ref += tmax;
            }
            pass(m_ref == -INFINITY ? 0.f : -m_ref, true, l_t);
          }
          l_part = l_part * alpha + l_t;
        }
        // P over this thread's own S columns in tensor memory
        release_s();
#pragma unroll
        for (int g = 0; g < Tr::kCols / 32; ++g)
          tc::st32x16x2(my_cols + 16 * g, *reinterpret_cast<const uint32_t(*)[16]>(hw + 16 * g),
                        my_cols + Tr::kCols / 2 + 16 * g, *reinterpret_cast<const uint32_t(*)[16]>(lw + 16 * g));
        // O of rows whose reference moved is rescaled (by the first half's warps) once the
        // previous O += P V is done
        if (half == 0 && __any_sync(FULL_MASK, rescale)) {
          const long long pit = it - 1;
          if (!__all_sync(FULL_MASK, wait(pv_done + (int)(pit & 1), (uint32_t)((pit >> 1) & 1)))) {
            ok = false;
            break;
          }
          tc::fence_after();
          const float f = rescale ? alpha : 1.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc::ld32x32(lane_base + Tr::kOCol + 32 * c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tc::st32x32(lane_base + Tr::kOCol + 32 * c, o);
          }
        }
        if (half == 0 && j == t.n_kv - 1 && (jj + 1) * Tr::kKv > t.L) {
          // positions past the context may hold anything (NaN included) and would meet a zero
          // weight in the MMA: zero the value rows there once their copy has landed
          const int vs = (int)(it % Tr::kStages);
          if (!__all_sync(FULL_MASK, wait(v_full + vs, (uint32_t)((it / Tr::kStages) & 1)))) {
            ok = false;
            break;
          }
          if (r < Tr::kKv && r >= t.L - jj * Tr::kKv) {
            const uint32_t vrow = v_s + vs * Tr::kKvBytes + (r >> 3) * Tr::kGroup + (r & 7) * 128;
#pragma unroll
            for (int h = 0; h < Tr::kSpans; ++h)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + h * 1024 + c * 16),
                             "r"(0u)
                             : "memory");
          }
          fence_proxy_async_smem();
        }
        tc::fence_before();
        mbar_arrive(p_ready + b);
      }
      if (!ok) break;
      // ---- epilogue: the halves add their sums; each stores half of the row of O / l ----
      float l_other;
      if (!swap_with_other_half(l_part, l_other)) {
        ok = false;
        break;
      }
      const float l_row = l_part + l_other;
      const long long last = kv_base + t.n_kv - 1;
      if (!__all_sync(FULL_MASK, wait(pv_done + (int)(last & 1), (uint32_t)((last >> 1) & 1)))) {
        ok = false;
        break;
      }
      tc::fence_after();
      const float inv = row_ok ? 1.f / l_row : 0.f;
      if (prefix_pass) {
        // this item's partial result of (member sequence, query head): O / l and (m, l); the
        // tensor-memory loads are warp-wide, only the stores depend on the row
        const long long slot = ((long long)(t.q0 + t.tok0 + (row_ok ? lt : 0)) * (Hkv * G) +
                                t.kvh * G + hh) * a.pre_splits + t.slot;
        float *dst = a.pre_o + slot * D;
#pragma unroll
        for (int c2 = 0; c2 < D / 64; ++c2) {
          const int c = (D / 64) * half + c2;
          uint32_t o[32];
          __syncwarp();
          tc::ld32x32(lane_base + Tr::kOCol + 32 * c, o);
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<float4 *>(dst + 32 * c)[i] =
                  make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                              __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          }
        }
        if (row_ok && half == 0) *reinterpret_cast<float2 *>(a.pre_ml + slot * 2) = make_float2(m_ref, l_row);
        kv_base += t.n_kv;
        continue;
      }
      const long long ob = (long long)(t.q0 + t.tok0 + (row_ok ? lt : 0)) * a.out_t +
                           (long long)(t.kvh * G + hh) * a.out_h;
#pragma unroll
      for (int c2 = 0; c2 < D / 64; ++c2) {
        const int c = (D / 64) * half + c2;  // 32-column chunk of O
        uint32_t o[32];
        __syncwarp();
        tc::ld32x32(lane_base + Tr::kOCol + 32 * c, o);
        if (!row_ok) {
        } else if (a.out_dtype == PA_F32) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + ob + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                 __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<T *>(a.out) + ob + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(o[8 * i + 2 * e]) * inv;
              const float x1 = __uint_as_float(o[8 * i + 2 * e + 1]) * inv;
              if constexpr (kBf16) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
                w[e] = *reinterpret_cast<const uint32_t *>(&h);
              } else {
                const __half2 h = __floats2half2_rn(x0, x1);
                w[e] = *reinterpret_cast<const uint32_t *>(&h);
              }
            }
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      kv_base += t.n_kv;
    }
  }

  // ---- teardown: every role done, tensor memory released by the warp that allocated it ----
  tc::fence_before();
  __syncthreads();
  if (wid == Tr::kMmaWarp) {
    tc::fence_after();
    tc::dealloc(tmem, Tr::kTmemCols);
  }
}

template <typename T, int D, int BS, int G>
cudaError_t launch_prefill_tc(const PrefillArgs &a, const PrefillMaps *maps, int num_ctas, cudaStream_t st) {
  using Tr = PrefillTcTraits<D, BS, G>;
  paged_prefill_tc_kernel<T, D, BS, G><<<num_ctas, Tr::kThreads, Tr::kSmemBytes, st>>>(a, *maps);
  return cudaGetLastError();
}

template <typename T, int D, int BS, int G>
bool make_prefill_tc(PrefillKernel *k) {
  using Tr = PrefillTcTraits<D, BS, G>;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(paged_prefill_tc_kernel<T, D, BS, G>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Tr::kSmemBytes) != cudaSuccess)
      return false;
    configured[dev] = true;
  }
  k->launch = &launch_prefill_tc<T, D, BS, G>;
  k->kernel = reinterpret_cast<const void *>(&paged_prefill_tc_kernel<T, D, BS, G>);
  k->threads_per_cta = Tr::kThreads;
  k->smem_bytes = Tr::kSmemBytes;
  k->tokens_per_tile = Tr::kTokens;
  k->tma_rows = 8;
  return true;
}

// Tables over head_dim {64, 128} x block_size {8, 16, 32} x group {1, 2, 4, 8}.
template <typename T>
bool prefill_tc_table(int head_dim, int block_size, int group, PrefillKernel *k) {
#define PA_CASE(DD, BB, GG) \
  if (head_dim == DD && block_size == BB && group == GG) return make_prefill_tc<T, DD, BB, GG>(k);
#define PA_GROUPS(DD, BB) PA_CASE(DD, BB, 1) PA_CASE(DD, BB, 2) PA_CASE(DD, BB, 4) PA_CASE(DD, BB, 8)
  PA_GROUPS(64, 8)
  PA_GROUPS(64, 16)
  PA_GROUPS(64, 32)
  PA_GROUPS(128, 8)
  PA_GROUPS(128, 16)
  PA_GROUPS(128, 32)
#undef PA_GROUPS
#undef PA_CASE
  return false;
}

}  // namespace pa

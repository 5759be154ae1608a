// pa_prefill_pp.cuh - the prefill kernel with two query tiles in flight per CTA (ping-pong):
// causal attention of a step's new tokens over the paged cache on the fifth-generation tensor
// cores, and the shared-prefix pass of pa_decode_shared_prefix.
//
// Sources: [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization
// support, distributed inference" 4.2 (requests join the running batch with their prompt
// tokens) and [P4] "vLLM core architecture: model loading, PagedAttention principle, KV cache
// management" 2.2.2 (attention assembles the whole KV sequence through the block table).  Token
// j of sequence s's q_len new tokens sits at position p = context_len - q_len + j and attends
// to positions 0 .. p.
//
// Work unit: two consecutive 128-row query tiles of one (sequence, kv head) (the second may be
// absent), each tile 128/G new tokens x G heads, one row per tensor-memory lane.  Both tiles
// read the same key/value tiles, which stream once per unit; the second tile's causal prefix
// is at least as long as the first's.  One persistent CTA per SM, eleven warps:
//   * warps 0-3 run the softmax of tile slot 0, warps 4-7 that of slot 1, one thread per row
//     (all 128 positions of a kv tile), so a row's maximum and sum never leave its thread;
//   * warp 8 loads the units' query tiles and the key tiles, warp 10 the value tiles, by TMA
//     into two-slot rings, one box per (block, kv head) tile as in the single-tile kernel;
//   * warp 9 (one lane) issues the MMAs in ping-pong order: S0 = Q0 K^T and S1 = Q1 K^T of kv
//     tile 0, then for each kv tile j: O0 += P0 V(j), S0 of tile j+1, O1 += P1 V(j), S1 of tile
//     j+1, so that one slot's MMAs run while the other slot's softmax works.
// Tensor memory (512 columns): slot x owns S/P at [256 x, 256 x + 128) and O at
// [256 x + 128, 256 x + 128 + D).  P replaces S in place, 32 positions at a time: for each
// block of 16 positions the hi terms (bf16 or fp16 pairs) fill its first 8 columns and the lo
// terms (p - hi) the next 8, so the columns written are those of the S values just read, and
// O += P V reads each block's hi and lo terms as two A operands.  An MMA reading P precedes the
// next S of the same slot in issue order, and tcgen05 MMAs complete in order, so S never
// overwrites P that is still to be read; by the same order, when S of tile j is complete the
// previous O += P V of that slot is complete too, and the softmax may rescale O in place.
// The online softmax is in base 2 against a reference maximum kept at whole numbers: it moves
// (by a whole number of units, to the ceiling of the new maximum) only when a logit passes it
// by more than 2^8, and the P terms already written for the kv tile, O and the running sum
// are then scaled by that power of two, which is exact.
#pragma once

#include "pa_prefill_tc.cuh"

namespace pa {

template <int D, int BS, int G>
struct PrefillPpTraits {
  static constexpr int kThreads = 352;
  static constexpr int kProducerWarp = 8;  // query tiles and key tiles
  static constexpr int kMmaWarp = 9;
  static constexpr int kValueWarp = 10;    // value tiles
  static constexpr int kRows = 128;
  static constexpr int kTokens = kRows / G;
  static constexpr int kKv = 128;
  static constexpr int kSpans = D / 64;
  static constexpr int kGroup = kSpans * 1024;  // bytes between 8-row groups of K, V tiles
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kKvBytes = kKv * D * 2;
  static constexpr int kBoxBytes = 8 * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kQOff = 0;                              // two query tiles
  static constexpr int kKOff = kQOff + 2 * kQBytes;
  static constexpr int kVOff = kKOff + kStages * kKvBytes;
  static constexpr int kBarOff = kVOff + kStages * kKvBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kInfoOff = kBarOff + kNumBars * 8;     // [tmem base, abort, count, rounds]
  static constexpr int kMaxMine = 64;
  static constexpr int kMineOff = kInfoOff + 32;
  static constexpr int kSmemBytes = kMineOff + kMaxMine * 8 + 1024;
  static constexpr int kMaxBins = 2048;
  static constexpr int kMaxList = 4096;
  static constexpr int kSlotCols = 256;                        // S/P 128 + O D (<= 128)
  static constexpr int kTmemCols = 512;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "1, 2, 4 or 8 query heads per kv head");
  static_assert(BS % 8 == 0 && kKv % BS == 0, "block size a multiple of the 8-position box");
  static_assert((kMaxBins + kMaxList) * 4 <= kStages * kKvBytes, "schedule scratch fits the key ring");
  static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
};

// A unit: up to two consecutive query tiles of one (sequence or group, kv head).
struct PpUnit {
  TcTile t[2];
  bool two;  // the second tile exists
  int n;     // kv tiles the unit streams (the longer tile's)
};

// 32 weights of one row -> their hi and lo 16-bit terms in the column order of one 32-position
// chunk of P: [hi of positions 0-15 | lo of 0-15 | hi of 16-31 | lo of 16-31], two per column.
template <bool kBf16>
__device__ __forceinline__ void pack_chunk(const float (&p)[32], uint32_t (&r)[32]) {
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int i = 0; i < 8; ++i) split2<kBf16>(p[16 * b + 2 * i], p[16 * b + 2 * i + 1], r[16 * b + i], r[16 * b + 8 + i]);
}

// 2^k for a whole number k <= 0 (0 below the normal range).
__device__ __forceinline__ float pow2_int(float k) {
  const int e = (int)k + 127;
  return e > 0 ? __int_as_float(e << 23) : 0.f;
}

// Multiply two packed 16-bit values by a power of two f: exact while the results stay normal.
template <bool kBf16>
__device__ __forceinline__ uint32_t scale_pair(uint32_t v, float f) {
  if constexpr (kBf16) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
    const __nv_bfloat162 y = __floats2bfloat162_rn(x.x * f, x.y * f);
    return *reinterpret_cast<const uint32_t *>(&y);
  } else {
    const float2 x = __half22float2(*reinterpret_cast<const __half2 *>(&v));
    const __half2 y = __floats2half2_rn(x.x * f, x.y * f);
    return *reinterpret_cast<const uint32_t *>(&y);
  }
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(PrefillPpTraits<D, BS, G>::kThreads, 1)
    paged_prefill_pp_kernel(const PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  using Tr = PrefillPpTraits<D, BS, G>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Tr::kBarOff);
  uint64_t *k_full = bars + 0, *k_empty = bars + 2, *v_full = bars + 4, *v_empty = bars + 6;
  uint64_t *q_full = bars + 8, *q_empty = bars + 10;    // per slot
  uint64_t *s_full = bars + 12, *p_ready = bars + 14;   // per slot
  uint64_t *o_ready = bars + 16, *o_free = bars + 18;   // per slot
  uint64_t *fin = bars + 20;
  volatile int *info = reinterpret_cast<volatile int *>(smem + Tr::kInfoOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Tr::kInfoOff);
  int2 *mine = reinterpret_cast<int2 *>(smem + Tr::kMineOff);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int wid = tid >> 5;
  const int Hkv = a.num_kv_heads;
  const int max_len = a.max_blocks * BS;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(p_ready + i, 128);
      mbar_init(o_ready + i, 1);
      mbar_init(o_free + i, 128);
    }
    mbar_init(fin, 1);
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

  // ---- the longest-first schedule of units (scratch in the key ring) ----
  int *bins = reinterpret_cast<int *>(smem + Tr::kKOff);
  int *list = bins + Tr::kMaxBins;
  const int nbins = (max_len + 15) / 16 + 1;
  const bool prefix_pass = a.pre_o != nullptr;
  bool sorted = !prefix_pass && nbins <= Tr::kMaxBins && a.num_seqs < (1 << 19);
  if (sorted)
    for (int i = tid; i < nbins; i += Tr::kThreads) bins[i] = 0;
  __syncthreads();
  auto seq_units = [&](int sq, int &len_out, int &q_out) {
    const int q0s = __ldg(a.query_start + sq);
    const int qn = __ldg(a.query_start + sq + 1) - q0s;
    const int raw = __ldg(a.context_lens + sq);
    const int Ls = raw < 0 ? 0 : (raw > max_len ? max_len : raw);
    len_out = Ls;
    q_out = qn;
    if (qn > Ls || q0s < 0 || (long long)q0s + qn > a.num_tokens) return -1;  // invalid
    const int tiles = qn > 0 ? (qn + Tr::kTokens - 1) / Tr::kTokens : 0;
    return (tiles + 1) / 2;
  };
  // cost of unit u: the causal prefix of its last token, in 16-position steps
  auto unit_cost = [&](int Ls, int qn, int u) {
    const int last = min((2 * u + 2) * Tr::kTokens, qn);
    return (Ls - qn + last + 15) / 16;
  };
  if (sorted) {
    for (int sq = tid; sq < a.num_seqs; sq += Tr::kThreads) {
      int Ls, qn;
      const int nu = seq_units(sq, Ls, qn);
      if (nu < 0) {
        set_error(a.err, PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      for (int u = 0; u < nu && u < Tr::kMaxList; ++u) atomicAdd(bins + unit_cost(Ls, qn, u), 1);
      atomicAdd((int *)info + 2, nu);
    }
  }
  __syncthreads();
  const int nunits = sorted ? info[2] : 0;
  const long long total = (long long)nunits * Hkv;
  sorted = sorted && nunits <= Tr::kMaxList && total <= (long long)Tr::kMaxMine * gridDim.x;
  if (sorted && wid == 0) {
    // bins[c] <- number of units costing more than c: where the units of cost c start
    const int seg = (nbins + 31) / 32;
    const int hi = nbins - 1 - lane * seg;
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
      const int nu = seq_units(sq, Ls, qn);
      for (int u = 0; u < nu; ++u) list[atomicAdd(bins + unit_cost(Ls, qn, u), 1)] = (sq << 12) | u;
    }
  }
  __syncthreads();
  if (sorted && tid < Tr::kMaxMine) {
    const long long r = tid;
    const long long k = r * gridDim.x + ((r & 1) ? (long long)gridDim.x - 1 - blockIdx.x : (long long)blockIdx.x);
    if (k < total) mine[r] = make_int2(list[k / Hkv], (int)(k % Hkv));
  }
  if (tid == 0) {
    long long rounds = 0;
    if (sorted) {
      const long long full = total / gridDim.x, rem = total % gridDim.x;
      const long long at = (full & 1) ? (long long)gridDim.x - 1 - blockIdx.x : (long long)blockIdx.x;
      rounds = full + (at < rem ? 1 : 0);
    }
    info[3] = (int)rounds;
  }
  fence_proxy_async_smem();  // the scratch is overwritten by copies from here on
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  const int my_rounds = info[3];

  // Tile tau (0-based) of (sequence s, kv head), causal: its tokens, positions and kv tiles.
  auto causal_tile = [&](int s, int tau, int kvh, TcTile &t) {
    t.s = s;
    t.tau = tau;
    t.kvh = kvh;
    t.q0 = __ldg(a.query_start + s);
    t.q_len = __ldg(a.query_start + s + 1) - t.q0;
    const int raw = __ldg(a.context_lens + s);
    t.L = raw < 0 ? 0 : (raw > max_len ? max_len : raw);
    t.valid = !(t.q_len > t.L || t.q0 < 0 || (long long)t.q0 + t.q_len > a.num_tokens) &&
              tau * Tr::kTokens < t.q_len;
    t.tok0 = tau * Tr::kTokens;
    t.ntok = min(Tr::kTokens, t.q_len - t.tok0);
    t.pos0 = t.L - t.q_len + t.tok0;
    t.n_kv = t.valid ? (t.pos0 + t.ntok + Tr::kKv - 1) / Tr::kKv : 0;
    t.j0 = 0;
    t.slot = 0;
    t.noncausal = false;
  };
  // The unit of round `round` (whole warp calls it); false when this CTA has no more units.
  auto next_unit = [&](long long round, PpUnit &u) -> bool {
    if (prefix_pass) {
      int g;
      long long rem;
      locate_prefix_item<2 * Tr::kTokens, Tr::kKv>(a, max_len, blockIdx.x + round * gridDim.x, g, rem);
      if (g < 0) return false;
      int first, members, P;
      prefix_group(a, g, max_len, first, members, P);
      const int kv_tiles = (P + Tr::kKv - 1) / Tr::kKv;
      const int splits = (kv_tiles + a.pre_kv - 1) / a.pre_kv;
      const int pairs = (members + 2 * Tr::kTokens - 1) / (2 * Tr::kTokens);
      const int slot = (int)(rem % splits);
      rem /= splits;
      const int up = (int)(rem % pairs);
      const int kvh = (int)(rem / pairs);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        TcTile &t = u.t[x];
        t.s = first;
        t.tau = 2 * up + x;
        t.kvh = kvh;
        t.q0 = first;
        t.q_len = members;
        t.L = P;
        t.tok0 = t.tau * Tr::kTokens;
        t.ntok = min(Tr::kTokens, members - t.tok0);
        t.pos0 = 0;
        t.slot = slot;
        t.j0 = slot * a.pre_kv;
        t.valid = slot < a.pre_splits && t.tok0 < members;
        t.n_kv = t.valid ? min(a.pre_kv, kv_tiles - t.j0) : 0;
        t.noncausal = true;
      }
      u.two = u.t[1].valid;
      u.n = u.t[0].n_kv;
      return true;
    }
    int s, up, kvh;
    if (sorted) {
      if (round >= my_rounds) return false;
      const int2 e = mine[round];
      s = e.x >> 12;
      up = e.x & 4095;
      kvh = e.y;
    } else {
      const long long x = blockIdx.x + round * gridDim.x;
      int ls, lu;
      locate_tile_tc<2 * Tr::kTokens>(a, x / Hkv, ls, lu);
      if (ls < 0) return false;
      s = ls;
      up = lu;
      kvh = (int)(x % Hkv);
    }
    causal_tile(s, 2 * up, kvh, u.t[0]);
    causal_tile(s, 2 * up + 1, kvh, u.t[1]);
    u.two = u.t[1].valid;
    u.n = u.two ? max(u.t[0].n_kv, u.t[1].n_kv) : u.t[0].n_kv;
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
    // ======= producers: query tiles and key tiles (warp 8), value tiles (warp 10), by TMA =======
    const int which = wid == Tr::kValueWarp ? 1 : 0;
    long long kv_base = 0;
    long long qt[2] = {0, 0};  // query tiles loaded per slot
    long long k_issued = 0, v_issued = 0;
    bool ok = true;
    PpUnit u;
    for (long long round = 0; ok && next_unit(round, u); ++round) {
      if (!u.t[0].valid) {
        if (lane == 0 && u.t[0].tau == 0 && u.t[0].kvh == 0)
          set_error(a.err, u.t[0].noncausal ? PA_DEVERR_PREFIX : PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      const TcTile &t = u.t[0];
      if (t.noncausal && which == 1 && t.kvh == 0) {
        // shared-prefix pass: the members of this unit must name the first member's prefix
        // length and, over this item's positions, its physical blocks (kv head 0's items check)
        const int32_t *row0 = a.block_tables + (long long)t.s * a.bt_s;
        const int b0 = t.j0 * Tr::kKv / BS;
        const int b1 = (min((t.j0 + t.n_kv) * Tr::kKv, t.L) + BS - 1) / BS;
        const int mend = u.two ? u.t[1].tok0 + u.t[1].ntok : t.tok0 + t.ntok;
        bool bad = false;
        for (int m = t.tok0 + lane; m < mend; m += 32) {
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
      if (which == 0) {
        // the unit's query tiles, each once its slot's previous S = QK^T are all done
        bool q_ok = true;
        if (lane == 0) {
          for (int x = 0; x < 2 && q_ok; ++x) {
            if (x == 1 && !u.two) break;
            q_ok = qt[x] < 1 || wait(q_empty + x, (uint32_t)((qt[x] - 1) & 1));
            if (q_ok) {
              mbar_arrive_expect_tx(q_full + x, Tr::kQBytes);
              tma_load_4d(q_s + x * Tr::kQBytes, &maps.q, 0, u.t[x].kvh * G, u.t[x].q0 + u.t[x].tok0,
                          0, q_full + x);
            }
          }
        }
        if (__shfl_sync(FULL_MASK, q_ok ? 1 : 0, 0) == 0) {
          ok = false;
          break;
        }
        ++qt[0];
        if (u.two) ++qt[1];
      }
      // Block ids of a kv tile: lane i holds the tile's i-th block (at most 16 blocks); the ids
      // of tile j + 1 are fetched before the waits of tile j.
      const int32_t *row = a.block_tables + (long long)t.s * a.bt_s;
      const int Lu = u.two ? u.t[1].L : t.L;  // the same context for both tiles
      auto fetch_ids = [&](int j) {
        const int p0 = (t.j0 + j) * Tr::kKv;
        const int nblk = (min(p0 + Tr::kKv, Lu) - p0 + BS - 1) / BS;
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
      for (int j = 0; j < u.n && ok; ++j) {
        const int nxt = j + 1 < u.n ? fetch_ids(j + 1) : 0;
        const long long it = kv_base + j;
        const int b = (int)(it % Tr::kStages);
        const long long use = it / Tr::kStages;
        const int p0 = (t.j0 + j) * Tr::kKv;
        const int pend = min(p0 + Tr::kKv, Lu);
        const int nblk = (pend - p0 + BS - 1) / BS;
        const uint32_t bytes = (uint32_t)(a.grouped_maps ? nblk * (BS / 8) : (pend - p0 + 7) / 8) * Tr::kBoxBytes;
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
        cur = nxt;
      }
      ok = __shfl_sync(FULL_MASK, ok ? 1 : 0, 0) != 0;
      kv_base += u.n;
    }
    if (lane == 0 && !ok) {
      // let the copies in flight land before the CTA leaves
      for (int x = 0; x < 2; ++x)
        if (qt[x] > 0) mbar_wait_bounded(q_full + x, (uint32_t)((qt[x] - 1) & 1), a.wait_cycles);
      constexpr int S = Tr::kStages;
      for (long long i = k_issued > S ? k_issued - S : 0; i < k_issued; ++i)
        mbar_wait_bounded(k_full + (int)(i % S), (uint32_t)((i / S) & 1), a.wait_cycles);
      for (long long i = v_issued > S ? v_issued - S : 0; i < v_issued; ++i)
        mbar_wait_bounded(v_full + (int)(i % S), (uint32_t)((i / S) & 1), a.wait_cycles);
    }
  } else if (wid == Tr::kMmaWarp) {
    // ================= MMA issue, ping-pong between the two slots =================
    constexpr uint32_t kIdS = tc::idesc_f16(kBf16, 128, Tr::kKv, false);
    constexpr uint32_t kIdO = tc::idesc_f16(kBf16, 128, D, true);
    long long kv_base = 0;
    long long qt[2] = {0, 0};  // units per slot (q_full, o_ready, o_free phases)
    long long sp[2] = {0, 0};  // S rounds per slot (s_full, p_ready phases)
    bool ok = true;
    PpUnit u;
    auto s_mma = [&](int x, int j) -> bool {  // S of slot x, kv tile j
      const long long it = kv_base + j;
      if (!wait(k_full + (int)(it % Tr::kStages), (uint32_t)((it / Tr::kStages) & 1))) return false;
      tc::fence_after();
      const uint32_t kb = k_s + (int)(it % Tr::kStages) * Tr::kKvBytes;
      const uint32_t qb = q_s + x * Tr::kQBytes;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t inner = (ks & 3) * 32;
        tc::mma(tmem + x * Tr::kSlotCols, tc::smem_desc(qb + (ks >> 2) * (Tr::kRows * 128) + inner, 16, 1024),
                tc::smem_desc(kb + (ks >> 2) * 1024 + inner, 16, Tr::kGroup), kIdS, ks > 0 ? 1u : 0u);
      }
      tc::commit(s_full + x);
      return true;
    };
    auto pv_mma = [&](int x, int j) -> bool {  // O of slot x += P V(j)
      const long long it = kv_base + j;
      if (!wait(p_ready + x, (uint32_t)(sp[x] & 1))) return false;
      ++sp[x];
      if (!wait(v_full + (int)(it % Tr::kStages), (uint32_t)((it / Tr::kStages) & 1))) return false;
      if (j == 0 && qt[x] > 0 && !wait(o_free + x, (uint32_t)((qt[x] - 1) & 1))) return false;
      tc::fence_after();
      const uint32_t vb = v_s + (int)(it % Tr::kStages) * Tr::kKvBytes;
      const uint32_t pc = tmem + x * Tr::kSlotCols;
#pragma unroll
      for (int kt = 0; kt < Tr::kKv / 16; ++kt) {
        const uint64_t vd = tc::smem_desc(vb + kt * 2 * Tr::kGroup, 1024, Tr::kGroup);
        tc::mma_ts(pc + 128, pc + 16 * kt, vd, kIdO, (j > 0 || kt > 0) ? 1u : 0u);
        tc::mma_ts(pc + 128, pc + 16 * kt + 8, vd, kIdO, 1u);
      }
      return true;
    };
    for (long long round = 0; ok && next_unit(round, u); ++round) {
      if (!u.t[0].valid) continue;
      if (lane == 0) {
        const int nx = u.two ? 2 : 1;
        int nk[2] = {u.t[0].n_kv, u.two ? u.t[1].n_kv : 0};
        for (int x = 0; x < nx && ok; ++x) ok = wait(q_full + x, (uint32_t)(qt[x] & 1));
        tc::fence_after();
        // prologue: S of kv tile 0 for both slots
        for (int x = 0; x < nx && ok; ++x) {
          if (nk[x] > 0) {
            ok = s_mma(x, 0);
            if (nk[x] == 1) tc::commit(q_empty + x);
          }
        }
        if (ok) tc::commit(k_empty + (int)(kv_base % Tr::kStages));
        for (int j = 0; j < u.n && ok; ++j) {
          bool next_s = false;
          for (int x = 0; x < nx && ok; ++x) {
            if (j >= nk[x]) continue;
            ok = pv_mma(x, j);
            if (!ok) break;
            if (j == nk[x] - 1) tc::commit(o_ready + x);
            if (j + 1 < nk[x]) {
              ok = s_mma(x, j + 1);
              next_s = true;
              if (j + 2 == nk[x]) tc::commit(q_empty + x);
            }
          }
          if (!ok) break;
          tc::commit(v_empty + (int)((kv_base + j) % Tr::kStages));
          if (next_s) tc::commit(k_empty + (int)((kv_base + j + 1) % Tr::kStages));
        }
        ++qt[0];
        if (u.two) ++qt[1];
      }
      ok = __shfl_sync(FULL_MASK, ok ? 1 : 0, 0) != 0;
      qt[0] = __shfl_sync(FULL_MASK, qt[0], 0);
      qt[1] = __shfl_sync(FULL_MASK, qt[1], 0);
      sp[0] = __shfl_sync(FULL_MASK, sp[0], 0);
      sp[1] = __shfl_sync(FULL_MASK, sp[1], 0);
      kv_base += u.n;
    }
    if (lane == 0) {
      // every MMA issued has completed before tensor memory is released
      tc::commit(fin);
      mbar_wait_bounded(fin, 0, a.wait_cycles);
    }
    __syncwarp();
  } else {
    // ================= softmax: warpgroup x owns slot x, one thread per row =================
    const int x = wid >> 2;
    const int quarter = wid & 3;
    const int r = 32 * quarter + lane;  // row = tensor-memory lane
    const int lt = r / G, hh = r % G;
    const uint32_t s_base = tc::taddr(tmem, 32 * quarter, x * Tr::kSlotCols);  // S/P of the slot
    const uint32_t o_base = s_base + 128;
    long long kv_base = 0;
    long long units = 0, sp = 0;
    bool ok = true;
    PpUnit u;
    for (long long round = 0; ok && next_unit(round, u); ++round) {
      if (!u.t[0].valid) continue;
      const int n_all = u.n;
      if (x == 1 && !u.two) {
        kv_base += n_all;
        continue;
      }
      const TcTile &t = u.t[x];
      const bool row_ok = lt < t.ntok;
      const int prow = row_ok ? (t.noncausal ? t.L - 1 : t.pos0 + lt) : -1;
      float m_ref = -INFINITY, l_row = 0.f;
      for (int j = 0; j < t.n_kv; ++j) {
        const long long it = kv_base + j;
        if (!__all_sync(FULL_MASK, wait(s_full + x, (uint32_t)(sp & 1)))) {
          ok = false;
          break;
        }
        ++sp;
        tc::fence_after();
        const int jj = t.j0 + j;
        const int c_lim = prow - jj * Tr::kKv;  // this row sees columns 0 .. c_lim of the tile
        float alpha = 1.f;                      // factor for what the tile had before
#pragma unroll 1
        for (int q = 0; q < Tr::kKv / 32; ++q) {
          uint32_t sr[32];
          __syncwarp();
          tc::ld32x32(s_base + 32 * q, sr);
          float tv[32];
          float cmax = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            tv[i] = 32 * q + i <= c_lim ? __uint_as_float(sr[i]) * a.scale_log2 : -INFINITY;
            cmax = fmaxf(cmax, tv[i]);
          }
          // move the reference (to a whole number at or above the chunk's maximum) when a
          // logit passes it by more than 2^8
          float mv = 1.f;
          if (cmax > m_ref + 8.f) {
            const float m_new = ceilf(cmax);
            mv = m_ref == -INFINITY ? 0.f : pow2_int(m_ref - m_new);
            m_ref = m_new;
          }
          if (__any_sync(FULL_MASK, mv != 1.f)) {
            // rescale the P terms this tile already holds (exact: a power of two), the sum
            // and (below, once per tile) O
            for (int q2 = 0; q2 < q; ++q2) {
              uint32_t pr[32];
              tc::ld32x32(s_base + 32 * q2, pr);
#pragma unroll
              for (int i = 0; i < 32; ++i) pr[i] = scale_pair<kBf16>(pr[i], mv);
              tc::st32x32(s_base + 32 * q2, pr);
            }
            l_row *= mv;
            alpha *= mv;
          }
          float p[32];
          const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            p[i] = fast_exp2(tv[i] + nm);
            l_row += p[i];
          }
          uint32_t pk[32];
          pack_chunk<kBf16>(p, pk);
          tc::st32x32(s_base + 32 * q, pk);
        }
        if (__any_sync(FULL_MASK, alpha != 1.f) && j > 0) {
          // O of rows whose reference moved: the previous O += P V of this slot completed before
          // this tile's S did (issue order), and the next one waits for p_ready
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc::ld32x32(o_base + 32 * c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tc::st32x32(o_base + 32 * c, o);
          }
        }
        // Only the unit's last kv tile can reach past the context; its value rows there are
        // zeroed by the slot whose O += P V reads that tile first (slot 0 when its causal
        // prefix reaches the tile, else slot 1).
        const bool zero_here = (x == 0) == (u.t[0].n_kv == u.n);
        if (zero_here && j == u.n - 1 && (jj + 1) * Tr::kKv > t.L) {
          // positions past the context may hold anything (NaN included) and would meet a zero
          // weight in the MMA: zero those value rows once their copy has landed
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
                asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + h * 1024 + c * 16), "r"(0u)
                             : "memory");
          }
          fence_proxy_async_smem();
        }
        tc::fence_before();
        mbar_arrive(p_ready + x);
      }
      if (!ok) break;
      // ---- epilogue: O / l of this slot's rows, once its last O += P V is done ----
      if (!__all_sync(FULL_MASK, wait(o_ready + x, (uint32_t)(units & 1)))) {
        ok = false;
        break;
      }
      tc::fence_after();
      const float inv = row_ok ? 1.f / l_row : 0.f;
      if (t.noncausal) {
        const long long slot = ((long long)(t.q0 + t.tok0 + (row_ok ? lt : 0)) * (Hkv * G) +
                                t.kvh * G + hh) * a.pre_splits + t.slot;
        float *dst = a.pre_o + slot * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          __syncwarp();
          tc::ld32x32(o_base + 32 * c, o);
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<float4 *>(dst + 32 * c)[i] =
                  make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                              __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          }
        }
        if (row_ok) *reinterpret_cast<float2 *>(a.pre_ml + slot * 2) = make_float2(m_ref, l_row);
      } else {
        const long long ob = (long long)(t.q0 + t.tok0 + (row_ok ? lt : 0)) * a.out_t +
                             (long long)(t.kvh * G + hh) * a.out_h;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          __syncwarp();
          tc::ld32x32(o_base + 32 * c, o);
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
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
                  w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                } else {
                  const __half2 h2 = __floats2half2_rn(x0, x1);
                  w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
              }
              dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc::fence_before();
      mbar_arrive(o_free + x);
      ++units;
      kv_base += n_all;
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
cudaError_t launch_prefill_pp(const PrefillArgs &a, const PrefillMaps *maps, int num_ctas, cudaStream_t st) {
  using Tr = PrefillPpTraits<D, BS, G>;
  paged_prefill_pp_kernel<T, D, BS, G><<<num_ctas, Tr::kThreads, Tr::kSmemBytes, st>>>(a, *maps);
  return cudaGetLastError();
}

template <typename T, int D, int BS, int G>
bool make_prefill_pp(PrefillKernel *k) {
  using Tr = PrefillPpTraits<D, BS, G>;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(paged_prefill_pp_kernel<T, D, BS, G>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::kSmemBytes) != cudaSuccess)
      return false;
    configured[dev] = true;
  }
  k->launch = &launch_prefill_pp<T, D, BS, G>;
  k->kernel = reinterpret_cast<const void *>(&paged_prefill_pp_kernel<T, D, BS, G>);
  k->threads_per_cta = Tr::kThreads;
  k->smem_bytes = Tr::kSmemBytes;
  k->tokens_per_tile = Tr::kTokens;
  k->tma_rows = 8;
  return true;
}

// Tables over head_dim {64, 128} x block_size {8, 16, 32} x group {1, 2, 4, 8}.
template <typename T>
bool prefill_pp_table(int head_dim, int block_size, int group, PrefillKernel *k) {
#define PA_CASE(DD, BB, GG) \
  if (head_dim == DD && block_size == BB && group == GG) return make_prefill_pp<T, DD, BB, GG>(k);
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

// pa_prefill.cuh - causal attention of a step's new tokens over the paged cache (prefill, or a
// chunk of a prompt in a continuously batched step), on tensor cores.
//
// Sources: [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization
// support, distributed inference" 4.2 (at each iteration requests join the running batch: a
// joining request's prompt tokens are that step's new tokens) and [P4] "vLLM core
// architecture: model loading, PagedAttention principle, KV cache management" 2.2.2 (attention
// assembles the whole KV sequence through the block table).  Token j of sequence s's q_len new
// tokens sits at position p = context_len - q_len + j and attends to positions 0 .. p.
//
// One CTA of four warps takes a tile of 64 query rows: 64 / G tokens of one sequence times
// the G query heads that read one kv head, 16 rows per warp (head fastest).  The K and V tiles
// of 16 context positions stream through a three-stage ring by TMA (the decode kernel's 5-D
// view of the cache, 128-byte swizzle); every warp reads each stage, so a K/V tile read from
// L2/HBM serves all 64 rows.  Per warp and chunk:
//   * S = Q K^T: mma.sync m16n8k16, the warp's 16 query rows as M (A fragments held in
//     registers for the whole tile), the chunk's 16 positions as N (two n-tiles), head_dim as K;
//     B comes from the key tile by ldmatrix.
//   * causal mask (position > p of the row, which also covers positions past the context),
//     online softmax in base 2 per row (4 lanes share a row; maxima and sums by shuffles).
//   * O += P V: the S accumulators are already laid out as the A fragment of the next MMA
//     (16 rows x 16 positions); P is split into two 16-bit terms (hi + lo) as in the decode
//     kernel; V fragments come from the value tile by ldmatrix.trans, head_dim as N.
// Tiles differ in cost (a tile's causal prefix), so they are spread longest first: every CTA
// builds the same list of (sequence, tile) pairs sorted by cost (a histogram of costs in shared
// memory, a prefix over it, a scatter) and takes positions of the list in snake order (round r
// gives CTA i position r*P + i, or r*P + P-1-i when r is odd), which keeps the heaviest tiles on
// different CTAs and evens out the sums.  Ties land in any order: each tile's rows are computed
// by one CTA alone, so the order changes no result.  Steps too large for the shared list fall
// back to tiles in sequence order, x = blockIdx.x, += gridDim.x, warp 0 finding the (sequence,
// tile) of x by a scan of query_start.
#pragma once

#include "pa_decode_mma.cuh"

namespace pa {

template <int D, int BS, int G>
struct PrefillTraits {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kRows = 64;                      // query rows of a tile
  static constexpr int kTokens = kRows / G;             // query tokens of a tile
  static constexpr int kBoxRows = BS < 16 ? BS : 16;    // rows per TMA box
  static constexpr int kCopies = 16 / kBoxRows;
  static constexpr int kBoxBytes = kBoxRows * D * 2;
  static constexpr int kTileBytes = 16 * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = 3;
  static constexpr int kKSteps = D / 16;
  static constexpr int kNTiles = D / 8;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kInfoOff = kBarOff + kStages * 16;
  // longest-first schedule: a histogram of tile costs (chunks) and the sorted tile list
  static constexpr int kMaxBins = 2048;  // costs 0 .. 2047 chunks (contexts up to 32K tokens)
  static constexpr int kMaxList = 4096;  // (sequence, tile) pairs
  static constexpr int kBinsOff = kInfoOff + 32;
  static constexpr int kListOff = kBinsOff + kMaxBins * 4;
  static constexpr int kSmemBytes = kListOff + kMaxList * 4 + 1024;  // + 1 KB alignment
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "1, 2, 4 or 8 query heads per kv head");
};

// Warp-cooperative: the sequence holding tile y of the step (tiles ordered by sequence, then
// position) and the tile's index within it; s = -1 when y is past the last tile.
template <int TOK>
__device__ __forceinline__ void locate_tile(const PrefillArgs &a, long long y, int &s_out,
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

__device__ __forceinline__ uint32_t pack_split(float x, float y, bool lo_part, bool bf16) {
  if (bf16) {
    const __nv_bfloat16 hx = __float2bfloat16_rn(x), hy = __float2bfloat16_rn(y);
    if (!lo_part) {
      const __nv_bfloat162 h = __halves2bfloat162(hx, hy);
      return *reinterpret_cast<const uint32_t *>(&h);
    }
    const __nv_bfloat162 l = __halves2bfloat162(__float2bfloat16_rn(x - __bfloat162float(hx)),
                                                __float2bfloat16_rn(y - __bfloat162float(hy)));
    return *reinterpret_cast<const uint32_t *>(&l);
  }
  const __half hx = __float2half_rn(x), hy = __float2half_rn(y);
  if (!lo_part) {
    const __half2 h = __halves2half2(hx, hy);
    return *reinterpret_cast<const uint32_t *>(&h);
  }
  const __half2 l = __halves2half2(__float2half_rn(x - __half2float(hx)),
                                   __float2half_rn(y - __half2float(hy)));
  return *reinterpret_cast<const uint32_t *>(&l);
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(PrefillTraits<D, BS, G>::kThreads)
    paged_prefill_kernel(const PrefillArgs a, const __grid_constant__ TmaMaps maps) {
  using Tr = PrefillTraits<D, BS, G>;
  using M = MmaType<T>;
  constexpr int ST = Tr::kStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Tr::kBarOff);
  uint64_t *empty = full + ST;
  int *info = reinterpret_cast<int *>(smem + Tr::kInfoOff);  // [s, tau, abort, tile count]

  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int lm = lane >> 3, lr = lane & 7;
  const int Hkv = a.num_kv_heads;
  const int max_len = a.max_blocks * BS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, Tr::kWarps);
    }
    fence_barrier_init();
    info[2] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.v)) : "memory");
  }

  // ---- the longest-first schedule ----
  int *bins = reinterpret_cast<int *>(smem + Tr::kBinsOff);
  int *list = reinterpret_cast<int *>(smem + Tr::kListOff);
  const int nbins = (max_len + 15) / 16 + 1;
  bool sorted = nbins <= Tr::kMaxBins && a.num_seqs < (1 << 19);
  if (sorted) {
    for (int i = threadIdx.x; i < nbins; i += Tr::kThreads) bins[i] = 0;
    if (threadIdx.x == 0) info[3] = 0;
  }
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
    for (int sq = threadIdx.x; sq < a.num_seqs; sq += Tr::kThreads) {
      int Ls, qn;
      const int nt = seq_tiles(sq, Ls, qn);
      if (nt < 0) {
        // new tokens outside the context, or query rows outside the query tensor: report
        set_error(a.err, PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      for (int t = 0; t < nt && t < Tr::kMaxList; ++t) atomicAdd(bins + tile_cost(Ls, qn, t), 1);
      atomicAdd(info + 3, nt);
    }
  }
  __syncthreads();
  const int ntiles = sorted ? info[3] : 0;
  sorted = sorted && ntiles <= Tr::kMaxList;
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
    for (int sq = threadIdx.x; sq < a.num_seqs; sq += Tr::kThreads) {
      int Ls, qn;
      const int nt = seq_tiles(sq, Ls, qn);
      for (int t = 0; t < nt; ++t) list[atomicAdd(bins + tile_cost(Ls, qn, t), 1)] = (sq << 12) | t;
    }
  }
  __syncthreads();

  long long pos = 0;  // ring items used so far by this CTA (every thread keeps the same count)
  const long long total = (long long)ntiles * Hkv;
  for (long long round = 0;; ++round) {
    int s, tau, kvh;
    if (sorted) {
      const long long k = round * gridDim.x +
                          ((round & 1) ? (long long)gridDim.x - 1 - blockIdx.x : (long long)blockIdx.x);
      if (k >= total || info[2] != 0) break;
      const int e = list[k / Hkv];
      s = e >> 12;
      tau = e & 4095;
      kvh = (int)(k % Hkv);
    } else {
      const long long x = blockIdx.x + round * gridDim.x;
      if (wid == 0) {
        int ls, lt_;
        locate_tile<Tr::kTokens>(a, x / Hkv, ls, lt_);
        if (lane == 0) {
          info[0] = ls;
          info[1] = lt_;
        }
      }
      __syncthreads();
      s = info[0];
      tau = info[1];
      const bool aborted = info[2] != 0;
      __syncthreads();  // info is rewritten for the next tile only after every thread read it
      if (s < 0 || aborted) break;
      kvh = (int)(x % Hkv);
    }
    const int q0 = __ldg(a.query_start + s);
    const int q_len = __ldg(a.query_start + s + 1) - q0;
    const int raw_len = __ldg(a.context_lens + s);
    const int L = raw_len < 0 ? 0 : (raw_len > max_len ? max_len : raw_len);
    if (q_len > L || q0 < 0 || (long long)q0 + q_len > a.num_tokens) {
      // new tokens outside the context, or query rows outside the query tensor: report, skip
      if (threadIdx.x == 0 && tau == 0 && kvh == 0) set_error(a.err, PA_DEVERR_CONTEXT_LEN);
      continue;
    }
    const int tok0 = tau * Tr::kTokens;                      // first new token of the tile
    const int ntok = min(Tr::kTokens, q_len - tok0);
    const int pos0 = L - q_len + tok0;                       // its position
    const int nchunks = (pos0 + ntok + 15) / 16;             // positions 0 .. pos0 + ntok - 1

    // this lane's two rows (g, g+8 of the warp's 16): token, head, position (-1: no row)
    int lt[2], hh[2], prow[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = 16 * wid + g + 8 * i;
      lt[i] = r / G;
      hh[i] = r % G;
      prow[i] = lt[i] < ntok ? pos0 + lt[i] : -1;
    }
    // query A fragments of the warp's 16 rows
    uint32_t qa[Tr::kKSteps][4];
    {
      const T *q = static_cast<const T *>(a.query);
      const T *row0 = q + (long long)(q0 + tok0 + lt[0]) * a.q_t + (long long)(kvh * G + hh[0]) * a.q_h;
      const T *row1 = q + (long long)(q0 + tok0 + lt[1]) * a.q_t + (long long)(kvh * G + hh[1]) * a.q_h;
#pragma unroll
      for (int ks = 0; ks < Tr::kKSteps; ++ks) {
        const int d = 16 * ks + 2 * c;
        qa[ks][0] = prow[0] >= 0 ? *reinterpret_cast<const uint32_t *>(row0 + d) : 0u;
        qa[ks][1] = prow[1] >= 0 ? *reinterpret_cast<const uint32_t *>(row1 + d) : 0u;
        qa[ks][2] = prow[0] >= 0 ? *reinterpret_cast<const uint32_t *>(row0 + d + 8) : 0u;
        qa[ks][3] = prow[1] >= 0 ? *reinterpret_cast<const uint32_t *>(row1 + d + 8) : 0u;
      }
    }
    float o[Tr::kNTiles][4];
#pragma unroll
    for (int nt = 0; nt < Tr::kNTiles; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

    // thread 0 keeps up to ST - 1 chunks ahead of the one being computed
    int issued = 0;
    auto issue = [&](int chunk) {
      const long long item = pos + chunk;
      const int slot = (int)(item % ST);
      if (item >= ST &&
          !mbar_wait_bounded(empty + slot, (uint32_t)(((item / ST) - 1) & 1), a.wait_cycles)) {
        set_error(a.err, PA_DEVERR_TIMEOUT);
        info[2] = 1;
        return false;
      }
      unsigned char *stage = smem + slot * Tr::kStageBytes;
      int valid = 0;
#pragma unroll
      for (int k = 0; k < Tr::kCopies; ++k) valid += chunk * 16 + k * Tr::kBoxRows < L;
      mbar_arrive_expect_tx(full + slot, 2u * valid * Tr::kBoxBytes);
#pragma unroll
      for (int k = 0; k < Tr::kCopies; ++k) {
        const int t = chunk * 16 + k * Tr::kBoxRows;
        if (t < L) {
          int blk = __ldg(a.block_tables + (long long)s * a.bt_s + t / BS);
          if (blk < 0 || (long long)blk >= a.num_blocks) {
            set_error(a.err, PA_DEVERR_BLOCK_ID);
            blk = 0;
          }
          tma_load_tile(smem_u32(stage + k * Tr::kBoxBytes), &maps.k, t % BS, kvh, blk, full + slot);
          tma_load_tile(smem_u32(stage + Tr::kTileBytes + k * Tr::kBoxBytes), &maps.v, t % BS, kvh,
                        blk, full + slot);
        }
      }
      ++issued;
      return true;
    };
    bool ok = true;
    if (threadIdx.x == 0)
      for (int i = 0; i < ST - 1 && i < nchunks && ok; ++i) ok = issue(i);

    for (int i = 0; i < nchunks; ++i) {
      if (threadIdx.x == 0 && ok && i + ST - 1 < nchunks) ok = issue(i + ST - 1);
      const long long item = pos + i;
      const int slot = (int)(item % ST);
      if (!__all_sync(FULL_MASK, mbar_wait_bounded(full + slot, (uint32_t)((item / ST) & 1),
                                                    a.wait_cycles))) {
        if (lane == 0) {
          set_error(a.err, PA_DEVERR_TIMEOUT);
          info[2] = 1;
        }
        break;
      }
      const uint32_t kb = smem_u32(smem + slot * Tr::kStageBytes);
      const uint32_t vb = kb + Tr::kTileBytes;
      const int t0 = i * 16;

      // ---- S = Q K^T (rows g | g+8, positions t0 + 8nt + 2c | +1) ----
      float sc[2][4];
      {
        // four independent accumulator chains (n-tile x even/odd k-step), summed at the end
        float sx[2][2][4] = {};
        const int row = ((lm >> 1) << 3) | lr;
#pragma unroll
        for (int ks = 0; ks < Tr::kKSteps; ++ks) {
          const int c16 = ((ks & 3) << 1) | (lm & 1);
          uint32_t r[4];
          ldmatrix_x4(r, kb + tile_offset<Tr>(row, ks >> 2) + ((c16 ^ lr) << 4));
          M::mma(sx[0][ks & 1], qa[ks], r[0], r[1]);
          M::mma(sx[1][ks & 1], qa[ks], r[2], r[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = sx[nt][0][e] + sx[nt][1][e];
      }
      // ---- causal mask, online softmax per row: the reference maximum of a row moves only
      // when a logit passes it by more than 8 (base 2), so weights stay <= 256 and most
      // chunks skip the rescale of O ----
      float cmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ri = e >> 1;
          const int t = t0 + 8 * nt + 2 * c + (e & 1);
          sc[nt][e] = t <= prow[ri] ? sc[nt][e] * a.scale_log2 : -INFINITY;
          cmax[ri] = fmaxf(cmax[ri], sc[nt][e]);
        }
      if (__any_sync(FULL_MASK, cmax[0] > mrow[0] + 8.f || cmax[1] > mrow[1] + 8.f)) {
        float alpha[2];
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          cmax[ri] = fmaxf(cmax[ri], __shfl_xor_sync(FULL_MASK, cmax[ri], 1));
          cmax[ri] = fmaxf(cmax[ri], __shfl_xor_sync(FULL_MASK, cmax[ri], 2));
          const float mnew = fmaxf(mrow[ri], cmax[ri]);
          alpha[ri] = mnew == -INFINITY ? 1.f : fast_exp2(mrow[ri] - mnew);
          mrow[ri] = mnew;
          lrow[ri] *= alpha[ri];
        }
#pragma unroll
        for (int nt = 0; nt < Tr::kNTiles; ++nt) {
          o[nt][0] *= alpha[0];
          o[nt][1] *= alpha[0];
          o[nt][2] *= alpha[1];
          o[nt][3] *= alpha[1];
        }
      }
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ri = e >> 1;
          p[nt][e] = mrow[ri] == -INFINITY ? 0.f : fast_exp2(sc[nt][e] - mrow[ri]);
          lrow[ri] += p[nt][e];
        }
      // ---- O += P V: P (16 rows x 16 positions) as the A fragment, hi and lo terms ----
      uint32_t ph[4], pl[4];
      ph[0] = pack_split(p[0][0], p[0][1], false, kBf16);
      ph[1] = pack_split(p[0][2], p[0][3], false, kBf16);
      ph[2] = pack_split(p[1][0], p[1][1], false, kBf16);
      ph[3] = pack_split(p[1][2], p[1][3], false, kBf16);
      pl[0] = pack_split(p[0][0], p[0][1], true, kBf16);
      pl[1] = pack_split(p[0][2], p[0][3], true, kBf16);
      pl[2] = pack_split(p[1][0], p[1][1], true, kBf16);
      pl[3] = pack_split(p[1][2], p[1][3], true, kBf16);
      const bool tail = t0 + 16 > L;
      const bool mlo = tail && t0 + 2 * c >= L, mhi = tail && t0 + 2 * c + 1 >= L;
      const bool mlo8 = tail && t0 + 2 * c + 8 >= L, mhi8 = tail && t0 + 2 * c + 9 >= L;
      {
        const int row = ((lm & 1) << 3) | lr;  // matrices 0, 2: positions 0-7; 1, 3: 8-15
#pragma unroll
        for (int j2 = 0; j2 < D / 16; ++j2) {
          const int c16 = ((j2 & 3) << 1) | (lm >> 1);
          uint32_t r[4];
          ldmatrix_x4_trans(r, vb + tile_offset<Tr>(row, j2 >> 2) + ((c16 ^ lr) << 4));
          if (tail) {
            // positions past the context may hold anything (NaN included): zero them
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              if (mlo) r[2 * h2] &= 0xffff0000u;
              if (mhi) r[2 * h2] &= 0x0000ffffu;
              if (mlo8) r[2 * h2 + 1] &= 0xffff0000u;
              if (mhi8) r[2 * h2 + 1] &= 0x0000ffffu;
            }
          }
          M::mma(o[2 * j2], ph, r[0], r[1]);
          M::mma(o[2 * j2 + 1], ph, r[2], r[3]);
          M::mma(o[2 * j2], pl, r[0], r[1]);
          M::mma(o[2 * j2 + 1], pl, r[2], r[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + slot);
    }
    __syncthreads();
    if (info[2] != 0) {
      // a wait timed out: let this tile's last copies land before the CTA leaves, then stop
      if (threadIdx.x == 0)
        for (int i = issued > ST ? issued - ST : 0; i < issued; ++i)
          mbar_wait_bounded(full + (int)((pos + i) % ST), (uint32_t)(((pos + i) / ST) & 1),
                            a.wait_cycles);
      break;
    }
    pos += nchunks;

    // ---- epilogue: O / l of the valid rows ----
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      lrow[ri] += __shfl_xor_sync(FULL_MASK, lrow[ri], 1);
      lrow[ri] += __shfl_xor_sync(FULL_MASK, lrow[ri], 2);
    }
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      if (prow[ri] < 0) continue;
      const float inv = 1.f / lrow[ri];
      const long long base = (long long)(q0 + tok0 + lt[ri]) * a.out_t + (long long)(kvh * G + hh[ri]) * a.out_h;
#pragma unroll
      for (int nt = 0; nt < Tr::kNTiles; ++nt) {
        const int d = 8 * nt + 2 * c;
        const float x0 = o[nt][2 * ri] * inv, x1 = o[nt][2 * ri + 1] * inv;
        if (a.out_dtype == PA_F32) {
          *reinterpret_cast<float2 *>(static_cast<float *>(a.out) + base + d) = make_float2(x0, x1);
        } else if (a.out_dtype == PA_BF16) {
          *reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(a.out) + base + d) =
              __floats2bfloat162_rn(x0, x1);
        } else {
          *reinterpret_cast<__half2 *>(static_cast<__half *>(a.out) + base + d) = __floats2half2_rn(x0, x1);
        }
      }
    }
  }
}

template <typename T, int D, int BS, int G>
cudaError_t launch_prefill(const PrefillArgs &a, const TmaMaps *maps, int num_ctas, cudaStream_t st) {
  using Tr = PrefillTraits<D, BS, G>;
  paged_prefill_kernel<T, D, BS, G><<<num_ctas, Tr::kThreads, Tr::kSmemBytes, st>>>(a, *maps);
  return cudaGetLastError();
}

template <typename T, int D, int BS, int G>
bool make_prefill(PrefillKernel *k) {
  using Tr = PrefillTraits<D, BS, G>;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(paged_prefill_kernel<T, D, BS, G>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Tr::kSmemBytes) != cudaSuccess)
      return false;
    configured[dev] = true;
  }
  k->launch = &launch_prefill<T, D, BS, G>;
  k->kernel = reinterpret_cast<const void *>(&paged_prefill_kernel<T, D, BS, G>);
  k->threads_per_cta = Tr::kThreads;
  k->smem_bytes = Tr::kSmemBytes;
  k->tokens_per_tile = Tr::kTokens;
  k->tma_rows = Tr::kBoxRows;
  return true;
}

// Tables over head_dim {64, 128} x block_size {8, 16, 32} x group {1, 2, 4, 8}.
template <typename T>
bool prefill_table(int head_dim, int block_size, int group, PrefillKernel *k) {
#define PA_CASE(DD, BB, GG) \
  if (head_dim == DD && block_size == BB && group == GG) return make_prefill<T, DD, BB, GG>(k);
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

// pa_decode.cuh - the CUDA-core decode kernel (any element type; the one used for fp32
// caches).  q.K and P.V run on fp32 CUDA cores with packed fp32x2 FMAs.  The work split, the
// chunk cursor and the merge are shared with the tensor-core kernel (pa_decode_common.cuh).
//
//   * Each warp runs its own ring of stages in shared memory.  Lane 0 issues one-dimensional
//     bulk asynchronous copies (cp.async.bulk, completion counted on an mbarrier) of each
//     chunk's key tile and value tile straight from their physical blocks, plus the query rows
//     when a new (sequence, kv head) starts.  No other warp touches the ring, so the main loop
//     has no block-wide barrier.
//   * A token row of keys is spread over RL = head_dim*elt/16 lanes (16 bytes each); per-head
//     dot products are reduced with a transposed butterfly so that each lane ends up owning one
//     (token, head) logit.  Logits are kept in base-2 units (q pre-scaled by scale*log2 e).  The
//     running maximum only moves when a chunk exceeds it by more than 2^8, which bounds every
//     weight by 256 and skips most rescaling.
#pragma once

#include "pa_decode_common.cuh"

namespace pa {

template <typename T, int D, int BS, int G>
struct SimtTraits {
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

// Transposed butterfly: v[0..N) are this lane's partial dot products for N heads over its
// slice of a row spread over the lanes that differ in the bits below 2*OFF.  Each level keeps
// half of the heads and sends the other half to the partner lane, so after the call v[0] holds
// the full dot product of one head: the row's lanes are split into N equal ranges, range n
// owning head n.
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

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(128, 1) paged_decode_kernel(const DecodeArgs a) {
  using Tr = SimtTraits<T, D, BS, G>;
  constexpr int RL = Tr::kRL, TPS = Tr::kTPS, EPL = Tr::kEPL, CH = Tr::kChunk;
  constexpr int STEPS = Tr::kSteps, ST = Tr::kStages, HL = Tr::kHeadLanes;
  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int max_len = a.max_blocks * BS;

  WarpShare share;
  if (!split_prologue<CH, Tr::kWarps, G, D, BS>(a, max_len, share)) return;
  const int gw = blockIdx.x * Tr::kWarps + wid;

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

  ChunkCursor<CH, BS, Tr::kCopies, Tr::kCopyRows> cur;
  cur.init(a, share, max_len);
  const long long n = share.n;

  auto issue = [&](int slot) {
    const int f = cur.flags();
    unsigned char *stage = wsm + slot * Tr::kStageBytes;
    if (lane == 0) {
      meta[slot] = cur.meta(f);
      const uint32_t bytes = 2u * cur.valid_copies() * Tr::kCopyBytes +
                             ((f & kFirst) ? (uint32_t)Tr::kQBytes : 0u) +
                             ((cur.issued == 0 && test_stalls(a, gw)) ? 16u : 0u);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bars + slot, bytes);
#pragma unroll
      for (int k = 0; k < Tr::kCopies; ++k) {
        const int t = cur.i * CH + k * Tr::kCopyRows;
        if (t < cur.len) {
          long long blk = cur.blk[k];
          if (blk < 0 || blk >= a.num_blocks) {
            set_error(a.err, PA_DEVERR_BLOCK_ID);
            blk = 0;
          }
          const long long off =
              (blk * a.kv_blk + (long long)cur.kvh * a.kv_head + (long long)(t % BS) * D) * Tr::kElt;
          bulk_copy_g2s(stage + k * Tr::kCopyBytes, static_cast<const char *>(a.key_cache) + off,
                        Tr::kCopyBytes, bars + slot);
          bulk_copy_g2s(stage + 4096 + k * Tr::kCopyBytes,
                        static_cast<const char *>(a.value_cache) + off, Tr::kCopyBytes, bars + slot);
        }
      }
      if (f & kFirst) {
        const char *q = static_cast<const char *>(a.query) +
                        ((long long)cur.s * a.q_s + (long long)cur.kvh * G * a.q_h) * Tr::kElt;
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
    cur.advance(a);
  };

  // Everything above read only context_lens and block_tables; the caches and the query may
  // still be written by the previous grid when this one was launched to overlap it.
  wait_for_previous_grid();
  const long long prime = n < ST ? n : ST;
  for (long long i = 0; i < prime; ++i) issue((int)i);

  const int r = lane / RL;  // row within a warp step
  const int j = lane % RL;  // 16-byte column of the row
  const int hh = j / HL;    // head this lane owns after the transposed reduce
  float2 q2[G][EPL / 2];
  float2 acc[G][EPL / 2];
  float m_ref = -INFINITY;
  float lsum = 0.f;
  bool piece_at_start = false;  // this piece begins at chunk 0 of its (sequence, kv head)

  for (long long c = 0; c < n; ++c) {
    const int slot = (int)(c % ST);
    const uint32_t parity = (uint32_t)((c / ST) & 1);
    if (!mbar_wait_bounded(bars + slot, parity, a.wait_cycles)) {
      // a copy never completed: record it, let the copies already issued land, and stop.
      if (lane == 0) set_error(a.err, PA_DEVERR_TIMEOUT);
      for (long long k = c; k < cur.issued; ++k)
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
      piece_at_start = (m.flags & kPairStart) != 0;
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
      if (a.separate_reduce && piece_at_start && lane == 0)
        a.pair_meta[m.pair] = make_int2(m.first_worker, m.npieces);
      // a (sequence, kv head) inside one share is written directly, unless it has partial
      // results of a shared prefix to merge with
      if (m.npieces == 1 && (a.prefix_lens == nullptr || prefix_pieces<BS>(a, m.s, max_len) == 0)) {
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
          float2 ml = make_float2(mh[0], lh[0]);
#pragma unroll
          for (int h = 1; h < G; ++h)
            if (lane == h) ml = make_float2(mh[h], lh[h]);
          *reinterpret_cast<float2 *>(a.part_ml + (seg * G + lane) * 2) = ml;
        }
        finish_piece<G, D, BS>(a, m, lane);
      }
    }
    __syncwarp();
    if (cur.issued < n) issue(slot);
  }
}

// Launch with or without programmatic dependent launch on the previous grid of the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapping(void (*kernel)(KArgs...), int ctas, int threads, int smem,
                               bool overlap_previous, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap_previous ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename T, int D, int BS, int G>
cudaError_t launch_decode_simt(const DecodeArgs &a, const TmaMaps *, int num_ctas,
                               bool overlap_previous, cudaStream_t st) {
  using Tr = SimtTraits<T, D, BS, G>;
  return launch_overlapping(paged_decode_kernel<T, D, BS, G>, num_ctas, Tr::kWarps * 32,
                            Tr::kSmemBytes, overlap_previous, st, a);
}

template <typename T, int D, int BS, int G>
bool make_decode_simt(DecodeKernel *k) {
  using Tr = SimtTraits<T, D, BS, G>;
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
  k->launch = &launch_decode_simt<T, D, BS, G>;
  k->launch_reduce = &launch_decode_merge<G, D, BS>;
  k->kernel = reinterpret_cast<const void *>(&paged_decode_kernel<T, D, BS, G>);
  k->warps_per_cta = Tr::kWarps;
  k->threads_per_cta = Tr::kWarps * 32;
  k->smem_bytes = Tr::kSmemBytes;
  k->chunk_tokens = Tr::kChunk;
  k->tma_rows = 0;
  return true;
}

}  // namespace pa

// pa_device.cuh - device helpers shared by the sm_100a kernels of the paged-attention library:
// shared-memory barriers and bulk asynchronous copies (inline PTX), element conversions and
// the error word.  Written for sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <type_traits>

#include "pa.h"

namespace pa {

constexpr unsigned FULL_MASK = 0xffffffffu;

// ------------------------------------------------------------------------------------------
// Element types.  Every kernel moves elements as 16-byte vectors; Elem<T>::kPerVec elements
// fit one vector and unpack() widens them to fp32.
// ------------------------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPerVec = 4;
  static __device__ __forceinline__ void unpack(const uint4 &v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  static __device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
  // A bf16 is the upper half of an fp32: widening is a shift (low element) or a mask (high).
  static __device__ __forceinline__ void unpack(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

template <>
struct Elem<__half> {
  static constexpr int kPerVec = 8;
  static __device__ __forceinline__ float to_float(__half x) { return __half2float(x); }
  static __device__ __forceinline__ void unpack(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
      float2 x = __half22float2(h);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
};

// ------------------------------------------------------------------------------------------
// FP8 E4M3 cache codes.  A value x of kv head h is stored as code(x / scale[h]): the division in
// fp32 (IEEE, round to nearest), the conversion rounding to nearest even and saturating to
// +-448 (NaN kept).  The cache write kernel and the fused decode step both quantise with these,
// so a position holds the same code whichever of them wrote it.
// ------------------------------------------------------------------------------------------
// Two fp32 values -> two codes, x0 in the low byte.
__device__ __forceinline__ uint16_t f32x2_to_fp8x2(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// Eight values -> eight codes (element i in byte i).
__device__ __forceinline__ uint2 fp8_codes8(const float (&f)[8], float scale) {
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
    w[i] = (uint32_t)f32x2_to_fp8x2(__fdiv_rn(f[4 * i], scale), __fdiv_rn(f[4 * i + 1], scale)) |
           ((uint32_t)f32x2_to_fp8x2(__fdiv_rn(f[4 * i + 2], scale), __fdiv_rn(f[4 * i + 3], scale)) << 16);
  return make_uint2(w[0], w[1]);
}

// Sixteen consecutive elements of type S at p (16-byte aligned) -> sixteen codes.
template <typename S>
__device__ __forceinline__ uint4 fp8_codes16(const char *p, float scale) {
  float a[8], b[8];
  if constexpr (sizeof(S) == 4) {
    float g[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      Elem<float>::unpack(__ldg(reinterpret_cast<const uint4 *>(p) + i), g);
#pragma unroll
      for (int j = 0; j < 4; ++j) (i < 2 ? a[4 * i + j] : b[4 * (i - 2) + j]) = g[j];
    }
  } else {
    Elem<S>::unpack(__ldg(reinterpret_cast<const uint4 *>(p)), a);
    Elem<S>::unpack(__ldg(reinterpret_cast<const uint4 *>(p) + 1), b);
  }
  const uint2 lo = fp8_codes8(a, scale), hi = fp8_codes8(b, scale);
  return make_uint4(lo.x, lo.y, hi.x, hi.y);
}

// Store n (= 4 or 8) fp32 values to `dst` in the given output element type, as 16-byte
// vectors (dst is 16-byte aligned).
__device__ __forceinline__ void store_row_piece(void *dst, int out_dtype, const float *v, int n) {
  if (out_dtype == PA_F32) {
    for (int i = 0; i < n; i += 4)
      *reinterpret_cast<float4 *>(static_cast<float *>(dst) + i) =
          make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  } else if (out_dtype == PA_BF16) {
    for (int i = 0; i < n; i += 8) {
      uint4 u;
      uint32_t *w = reinterpret_cast<uint32_t *>(&u);
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[i + 2 * k], v[i + 2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t *>(&b);
      }
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(dst) + i) = u;
    }
  } else {
    for (int i = 0; i < n; i += 8) {
      uint4 u;
      uint32_t *w = reinterpret_cast<uint32_t *>(&u);
      for (int k = 0; k < 4; ++k) {
        __half2 b = __floats2half2_rn(v[i + 2 * k], v[i + 2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t *>(&b);
      }
      *reinterpret_cast<uint4 *>(static_cast<__half *>(dst) + i) = u;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Shared-memory barriers and bulk copies (PTX ISA: mbarrier, cp.async.bulk).
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the asynchronous proxy (the bulk-copy engine).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier shared-memory accesses before later asynchronous-proxy writes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of a barrier, giving up after about `limit_cycles` SM clocks.
// Returns false on timeout.  Every lane of the warp calls it (the result is warp-uniform
// because every lane observes the same barrier).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long limit_cycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit_cycles) return false;
  }
}

// Bulk copy global -> this CTA's shared memory, completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2^x on the SFU (ex2.approx.ftz.f32: relative error about 2^-22; results below 2^-126 flush to
// zero, which only drops weights that are negligible next to the running maximum).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32x2 FMA (sm_100): d = a * b + c on both halves.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Programmatic dependent launch: wait until the grid this one depends on has completed and its
// memory is visible (returns at once when the launch had no such dependency) ...
__device__ __forceinline__ void wait_for_previous_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// ... and let the grid launched after this one start early.
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;"); }

// Global nanosecond timer and the SM this thread runs on (decode timelines).
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ unsigned int sm_id() {
  unsigned int r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void set_error(unsigned int *err, unsigned int bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace pa

// pa_probe.cu - a read-only HBM bandwidth probe: the ceiling a read stream such as decode
// attention can reach, next to the copy bandwidth (which counts read and written bytes).
//
// Two ways to read a buffer once, each a persistent grid over all SMs:
//   mode 0: 16-byte vector loads that skip L1 (eight independent loads in flight per thread,
//           2048 threads per SM), folded into one word so that the loads are kept;
//   mode 1: 1-D bulk asynchronous copies (the copy engine the decode kernels use) of 32 KB
//           chunks into a six-slot shared-memory ring per SM, each completion counted on an
//           mbarrier; nothing reads the landed bytes.
// Every wait is bounded; a wait that runs out stops the CTA and sets bit 1 of the sink word's
// companion flag (sink[1]).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace {

constexpr int kLdThreads = 512;
constexpr int kLdUnroll = 8;
constexpr uint32_t kBulkChunk = 32768;
constexpr int kBulkStages = 6;
constexpr long long kBulkWaitCycles = 2000000000ll;  // about one second

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kLdThreads) hbm_read_ld_kernel(const uint4 *__restrict__ p,
                                                                 unsigned long long n16,
                                                                 unsigned int *sink) {
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (kLdUnroll - 1) * stride < n16; i += kLdUnroll * stride) {
    uint4 v[kLdUnroll];
#pragma unroll
    for (int k = 0; k < kLdUnroll; ++k) v[k] = ld_stream(p + i + k * stride);
#pragma unroll
    for (int k = 0; k < kLdUnroll; ++k) acc ^= v[k].x ^ v[k].y ^ v[k].z ^ v[k].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ld_stream(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc ^= __shfl_xor_sync(pa::FULL_MASK, acc, off);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

// One warp per CTA; lane 0 keeps kBulkStages chunks in flight.  CTA b reads chunks
// b, b + gridDim.x, b + 2 gridDim.x, ...
__global__ void __launch_bounds__(32) hbm_read_bulk_kernel(const char *__restrict__ p,
                                                           unsigned long long chunks,
                                                           unsigned int *sink) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBulkStages * kBulkChunk);
  if (threadIdx.x != 0) return;
  for (int s = 0; s < kBulkStages; ++s) pa::mbar_init(full + s, 1);
  pa::fence_barrier_init();
  const unsigned long long mine =
      chunks > blockIdx.x ? (chunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0ull;
  auto issue = [&](unsigned long long j) {
    const int slot = (int)(j % kBulkStages);
    pa::mbar_arrive_expect_tx(full + slot, kBulkChunk);
    pa::bulk_copy_g2s(smem + (size_t)slot * kBulkChunk,
                      p + (blockIdx.x + j * gridDim.x) * (unsigned long long)kBulkChunk,
                      kBulkChunk, full + slot);
  };
  for (unsigned long long j = 0; j < mine && j < (unsigned long long)kBulkStages; ++j) issue(j);
  for (unsigned long long j = 0; j < mine; ++j) {
    const int slot = (int)(j % kBulkStages);
    if (!pa::mbar_wait_bounded(full + slot, (uint32_t)((j / kBulkStages) & 1), kBulkWaitCycles)) {
      atomicOr(sink + 1, 1u);
      // let the copies still in flight land before the CTA's shared memory goes away
      for (unsigned long long r = j + 1; r < mine && r < j + kBulkStages; ++r)
        pa::mbar_wait_bounded(full + (int)(r % kBulkStages), (uint32_t)((r / kBulkStages) & 1),
                              kBulkWaitCycles);
      return;
    }
    if (j + kBulkStages < mine) issue(j + kBulkStages);
  }
}

thread_local char g_probe_msg[256];

}  // namespace

extern "C" int pa_hbm_read_probe(const void *buf, size_t bytes, int32_t mode, void *sink,
                                 void *stream) {
  auto refuse = [](int code, const char *msg) {
    snprintf(g_probe_msg, sizeof(g_probe_msg), "pa_hbm_read_probe: %s", msg);
    pa::set_last_error(g_probe_msg);
    return code;
  };
  if (!buf || !sink) return refuse(PA_ERR_INVALID_ARG, "NULL buffer or sink");
  if (((uintptr_t)buf & 127u) != 0 || ((uintptr_t)sink & 7u) != 0)
    return refuse(PA_ERR_LAYOUT, "buffer must be 128-byte aligned and sink 8-byte aligned");
  if (mode != 0 && mode != 1) return refuse(PA_ERR_INVALID_ARG, "mode must be 0 or 1");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return refuse(PA_ERR_CUDA, "cudaGetDevice failed");
  cudaPointerAttributes at;
  for (const void *q : {buf, static_cast<const void *>(sink)}) {
    if (cudaPointerGetAttributes(&at, q) != cudaSuccess || at.type != cudaMemoryTypeDevice ||
        at.device != dev) {
      cudaGetLastError();
      return refuse(PA_ERR_LAYOUT, "buffer and sink must be device memory of the current device");
    }
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return refuse(PA_ERR_CUDA, "cudaDeviceGetAttribute failed");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (mode == 0) {
    hbm_read_ld_kernel<<<sms * 4, kLdThreads, 0, st>>>(static_cast<const uint4 *>(buf), bytes / 16,
                                                       static_cast<unsigned int *>(sink));
    e = cudaGetLastError();
  } else {
    const size_t smem = (size_t)kBulkStages * kBulkChunk + kBulkStages * 8;
    static bool configured[64] = {};
    if (dev < 64 && !configured[dev]) {
      if (cudaFuncSetAttribute(hbm_read_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem) != cudaSuccess)
        return refuse(PA_ERR_CUDA, "cudaFuncSetAttribute failed");
      configured[dev] = true;
    }
    hbm_read_bulk_kernel<<<sms, 32, smem, st>>>(static_cast<const char *>(buf), bytes / kBulkChunk,
                                                static_cast<unsigned int *>(sink));
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    snprintf(g_probe_msg, sizeof(g_probe_msg), "pa_hbm_read_probe: launch failed: %s",
             cudaGetErrorString(e));
    pa::set_last_error(g_probe_msg);
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

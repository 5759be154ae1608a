// pa_noalloc.cu - decode with its scratch in a fixed device array, for callers that cannot
// allocate device memory (graph capture, engines that own all memory, latency-critical loops).
//
// The array below is the decode scratch of pa_decode_noalloc: merge counters, pair records and
// partial results, laid out exactly as a pa_decode_ex workspace.  Host code may not use the
// array's name as a device address (in host code it names a host-side stand-in), so every call
// looks the address up with cudaGetSymbolAddress, with the caller's device current, and passes
// it to the kernels.  The lookup allocates nothing; when the address differs from the one seen
// before on that device (the first call, or the module reloaded after a device reset) the
// array is cleared on the call's stream.  Nothing here allocates.
//
// After a decode that ran out of its wait limit (PA_DEVERR_TIMEOUT) the merge counters in the
// array may be partly counted; reading the error word with pa_get_device_error marks every
// workspace the library knows, this array included, so that the next call zeroes its counters
// again (on its stream, with cudaMemsetAsync, which allocates nothing).
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr size_t kScratchBytes = PA_NOALLOC_SCRATCH_BYTES;

// One instance per device that loads the library, zero at module load, kept until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch[64];  // device address of g_noalloc_scratch last cleared, per device id

}  // namespace

extern "C" int pa_decode_noalloc(const pa_tensor *out, const pa_tensor *query,
                                 const pa_tensor *key_cache, const pa_tensor *value_cache,
                                 const pa_tensor *block_tables, const pa_tensor *context_lens,
                                 float scale, int32_t block_size, int32_t num_kv_heads,
                                 void *stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    pa::set_last_error("pa_decode_noalloc: cudaGetDevice failed");
    return PA_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) {
    pa::set_last_error("pa_decode_noalloc: device id out of range (at most 64 devices)");
    return PA_ERR_INVALID_ARG;
  }
  void *scratch = nullptr;
  e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
  if (e != cudaSuccess || !scratch) {
    char msg[160];
    snprintf(msg, sizeof(msg), "pa_decode_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    pa::set_last_error(msg);
    return PA_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch[dev] != scratch) {
      // The merge counters must start at zero: clear the array on the caller's stream.
      const int rc = pa_workspace_init(scratch, kScratchBytes, stream);
      if (rc != PA_OK) return rc;
      g_scratch[dev] = scratch;
    }
  }
  const size_t need = pa::decode_scratch_need(query, key_cache, block_size, num_kv_heads);
  if (need > kScratchBytes) {
    char msg[240];
    snprintf(msg, sizeof(msg),
             "pa_decode_noalloc: these shapes need %zu bytes of scratch, more than the %zu-byte "
             "static scratch; use pa_decode or pa_decode_ex",
             need, kScratchBytes);
    pa::set_last_error(msg);
    return PA_ERR_WORKSPACE;
  }
  return pa::decode_into(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                         block_size, num_kv_heads, scratch, kScratchBytes, stream);
}

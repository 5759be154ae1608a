// Prefill kernels (tcgen05) for f16 caches: head_dim 64/128, block sizes 8/16/32, 1/2/4/8 query heads
// per kv head.
#include "pa_prefill_tc.cuh"

namespace pa {
bool prefill_kernel_f16(int head_dim, int block_size, int group, PrefillKernel *k) {
  return prefill_tc_table<__half>(head_dim, block_size, group, k);
}
}  // namespace pa

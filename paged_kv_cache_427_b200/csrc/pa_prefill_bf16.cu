// Prefill kernels (tcgen05) for bf16 caches: head_dim 64/128, block sizes 8/16/32, 1/2/4/8 query heads
// per kv head.
#include "pa_prefill_tc.cuh"
#ifndef PA_PREFILL_PP
#define PA_PREFILL_PP 0  // 1: the two-tile (ping-pong) kernel
#endif
#if PA_PREFILL_PP
#include "pa_prefill_pp.cuh"
#endif

namespace pa {
bool prefill_kernel_bf16(int head_dim, int block_size, int group, PrefillKernel *k) {
#if PA_PREFILL_PP
  return prefill_pp_table<__nv_bfloat16>(head_dim, block_size, group, k);
#else
  return prefill_tc_table<__nv_bfloat16>(head_dim, block_size, group, k);
#endif
}
}  // namespace pa

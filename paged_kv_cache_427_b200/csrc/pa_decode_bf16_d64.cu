// Decode kernels for bf16 caches with head_dim 64 (block sizes 8/16/32, groups 1/2/4/8).
#include "pa_decode.cuh"

namespace pa {
bool decode_kernel_bf16_d64(int block_size, int group, DecodeKernel *k) {
  return decode_kernel_table<__nv_bfloat16, 64>(block_size, group, k);
}
}  // namespace pa

// Decode kernels for bf16 caches with head_dim 64: tensor-core and CUDA-core variants for
// block sizes 8/16/32 and 1/2/4/8 query heads per kv head.
#include "pa_decode_mma.cuh"

namespace pa {
bool decode_kernel_bf16_d64(int block_size, int group, bool tensor_cores, DecodeKernel *k) {
  return decode_table<__nv_bfloat16, 64>(block_size, group, tensor_cores, k);
}
}  // namespace pa

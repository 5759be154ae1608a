// Decode kernels for fp32 caches with head_dim 128 (CUDA-core; block sizes 8/16/32, 1/2/4/8
// query heads per kv head).
#include "pa_decode_mma.cuh"

namespace pa {
bool decode_kernel_f32_d128(int block_size, int group, bool, DecodeKernel *k) {
  return decode_table_f32<128>(block_size, group, k);
}
}  // namespace pa

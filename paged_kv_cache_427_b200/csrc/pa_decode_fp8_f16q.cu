// Decode kernels for FP8 E4M3 caches (head_dim 128) read with a f16 query: tensor-core
// variants for block sizes 8/16/32 and 1/2/4/8 query heads per kv head.
#include "pa_decode_mma.cuh"

namespace pa {
bool decode_kernel_fp8_f16q(int block_size, int group, DecodeKernel *k) {
  return decode_table_fp8<__half>(block_size, group, k);
}
}  // namespace pa

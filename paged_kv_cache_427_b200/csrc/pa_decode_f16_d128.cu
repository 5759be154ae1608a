// Decode kernels for f16 caches with head_dim 128 (block sizes 8/16/32, groups 1/2/4/8).
#include "pa_decode.cuh"

namespace pa {
bool decode_kernel_f16_d128(int block_size, int group, DecodeKernel *k) {
  return decode_kernel_table<__half, 128>(block_size, group, k);
}
}  // namespace pa

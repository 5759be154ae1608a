// Decode kernel selection by element type and head_dim (the instantiations live in one
// translation unit per (element type, head_dim) so they compile in parallel).
#include "pa_internal.h"

namespace pa {
bool decode_kernel_f32_d64(int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_f32_d128(int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_bf16_d64(int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_bf16_d128(int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_f16_d64(int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_f16_d128(int block_size, int group, bool tensor_cores, DecodeKernel *k);
bool decode_kernel_fp8_bf16q(int block_size, int group, DecodeKernel *k);
bool decode_kernel_fp8_f16q(int block_size, int group, DecodeKernel *k);

bool decode_kernel_fp8(int q_dtype, int head_dim, int block_size, int group, DecodeKernel *k) {
  if (head_dim != 128) return false;
  if (q_dtype == PA_BF16) return decode_kernel_fp8_bf16q(block_size, group, k);
  if (q_dtype == PA_F16) return decode_kernel_fp8_f16q(block_size, group, k);
  return false;
}

bool decode_kernel_f32(int head_dim, int block_size, int group, bool tensor_cores, DecodeKernel *k) {
  if (head_dim == 64) return decode_kernel_f32_d64(block_size, group, tensor_cores, k);
  if (head_dim == 128) return decode_kernel_f32_d128(block_size, group, tensor_cores, k);
  return false;
}
bool decode_kernel_bf16(int head_dim, int block_size, int group, bool tensor_cores, DecodeKernel *k) {
  if (head_dim == 64) return decode_kernel_bf16_d64(block_size, group, tensor_cores, k);
  if (head_dim == 128) return decode_kernel_bf16_d128(block_size, group, tensor_cores, k);
  return false;
}
bool decode_kernel_f16(int head_dim, int block_size, int group, bool tensor_cores, DecodeKernel *k) {
  if (head_dim == 64) return decode_kernel_f16_d64(block_size, group, tensor_cores, k);
  if (head_dim == 128) return decode_kernel_f16_d128(block_size, group, tensor_cores, k);
  return false;
}
}  // namespace pa

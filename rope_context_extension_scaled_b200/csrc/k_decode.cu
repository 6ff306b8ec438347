// Launchers of the decode kernels (attn_decode.cuh) and of the int8 KV-cache
// kernels (kv_int8.cuh).
#include "launch.h"
#include "kv_int8.cuh"

namespace rcx {

int decode_launch(const DecodeArgs& a, int G, bool tensor_core, dim3 grid, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_DECODE, stream);
  if (tensor_core) {
    // tensor-core form: 16-byte rows of k and v for cp.async
    auto kern = G == 1 ? attn_decode_mma_kernel<1>
              : G == 2 ? attn_decode_mma_kernel<2>
              : G == 4 ? attn_decode_mma_kernel<4>
                       : attn_decode_mma_kernel<8>;
    if (allow_smem(kern, kDmSmem)) return RCX_ERR_CUDA;
    kern<<<grid, kDmWarps * 32, kDmSmem, stream>>>(a);
  } else {
    switch (G) {
      case 1: attn_decode_kernel<1><<<grid, kDecThreads, 0, stream>>>(a); break;
      case 2: attn_decode_kernel<2><<<grid, kDecThreads, 0, stream>>>(a); break;
      case 4: attn_decode_kernel<4><<<grid, kDecThreads, 0, stream>>>(a); break;
      default: attn_decode_kernel<8><<<grid, kDecThreads, 0, stream>>>(a); break;
    }
  }
  return launch_status();
}

int decode_i8_launch(const DecodeArgs& a, int G, const float* k_scale, const float* v_scale, dim3 grid,
                     cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_DECODE, stream);
  auto kern = G == 1 ? attn_decode_i8_kernel<1>
            : G == 2 ? attn_decode_i8_kernel<2>
            : G == 4 ? attn_decode_i8_kernel<4>
                     : attn_decode_i8_kernel<8>;
  if (allow_smem(kern, kDqSmem)) return RCX_ERR_CUDA;
  kern<<<grid, kDqWarps * 32, kDqSmem, stream>>>(a, k_scale, v_scale);
  return launch_status();
}

int decode_combine_launch(const DecodeArgs& a, int out_dtype, int grid, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_DECODE, stream);
  if (out_dtype == RCX_BF16)
    decode_combine_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a);
  else
    decode_combine_kernel<float><<<grid, 256, 0, stream>>>(a);
  return launch_status();
}

int quantize_i8_launch(const QuantArgs& a, bool rows16, int grid, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_DECODE, stream);
  if (rows16)
    kv_quantize_int8_r8_kernel<<<grid, 256, 0, stream>>>(a);
  else
    kv_quantize_int8_kernel<<<grid, 256, 0, stream>>>(a);
  return launch_status();
}

}  // namespace rcx

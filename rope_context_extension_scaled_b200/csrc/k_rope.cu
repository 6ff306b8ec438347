// Launchers of the RoPE rotation kernels (rope_apply.cuh).
#include "launch.h"
#include "rope_apply.cuh"

namespace rcx {

int rope_bulk_launch(const RopeBulkArgs& b, int dtype, int grid, size_t smem, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_ROPE, stream);
  if (dtype == RCX_BF16) {
    if (allow_smem(rope_bulk_kernel<__nv_bfloat16>, smem)) return RCX_ERR_CUDA;
    rope_bulk_kernel<__nv_bfloat16><<<grid, kRopeThreads, smem, stream>>>(b);
  } else {
    if (allow_smem(rope_bulk_kernel<float>, smem)) return RCX_ERR_CUDA;
    rope_bulk_kernel<float><<<grid, kRopeThreads, smem, stream>>>(b);
  }
  return launch_status();
}

int rope_apply_launch(const RopeArgs& a, int dtype, bool same_layout, int grid, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_ROPE, stream);
  if (dtype == RCX_BF16) {
    if (same_layout) rope_apply_kernel<__nv_bfloat16, true><<<grid, kRopeThreads, 0, stream>>>(a);
    else rope_apply_kernel<__nv_bfloat16, false><<<grid, kRopeThreads, 0, stream>>>(a);
  } else {
    if (same_layout) rope_apply_kernel<float, true><<<grid, kRopeThreads, 0, stream>>>(a);
    else rope_apply_kernel<float, false><<<grid, kRopeThreads, 0, stream>>>(a);
  }
  return launch_status();
}

int status_exchange_rope(cudaStream_t stream, int* status) { return device_status_exchange(stream, status); }

}  // namespace rcx

// Launchers of the RoPE rotation kernels (rope_apply.cuh).
#include "launch.h"
#include "rope_apply.cuh"

namespace rcx {

int rope_apply_launch(const RopeArgs& a, int dtype, int grid, int block, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_ROPE, stream);
  if (dtype == RCX_BF16) rope_apply_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(a);
  else rope_apply_kernel<float><<<grid, block, 0, stream>>>(a);
  return launch_status();
}

int status_exchange_rope(cudaStream_t stream, int* status) { return device_status_exchange(stream, status); }

}  // namespace rcx

// Launcher of the LSE merge kernel (merge.cuh).
#include "launch.h"
#include "merge.cuh"

namespace rcx {

int merge_launch(const MergeArgs& a, int out_dtype, int grid, cudaStream_t stream) {
  LaunchScope scope(RCX_KERNEL_MERGE, stream);
  if (out_dtype == RCX_BF16)
    merge_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a);
  else
    merge_kernel<float><<<grid, 256, 0, stream>>>(a);
  return launch_status();
}

}  // namespace rcx

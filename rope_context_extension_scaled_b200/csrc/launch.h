// Host-side interface between the C-ABI translation unit (rcx_api.cu) and the
// kernel translation units (k_*.cu), which are compiled separately and in
// parallel.  Each k_*.cu file holds one family of kernels and the functions
// that launch them; rcx_api.cu holds argument checking, planning and the C
// entry points.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/rcx.h"

namespace rcx {

struct AttnArgs;
struct RopeArgs;
struct MergeArgs;
struct DecodeArgs;
struct QuantArgs;

// Counts a launch of `kind` (rcx_kernel_kind); with timing on, records CUDA
// events around it on `stream`.  Defined in rcx_api.cu.
class LaunchScope {
 public:
  LaunchScope(int kind, cudaStream_t stream);
  ~LaunchScope();
  LaunchScope(const LaunchScope&) = delete;
  LaunchScope& operator=(const LaunchScope&) = delete;

 private:
  int kind_;
  cudaStream_t stream_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

int sm_count();            // SMs of the current device (read once)
int launch_status();       // RCX_OK, or RCX_ERR_CUDA after printing the launch error

// Opt a kernel into more than 48 KB of dynamic shared memory.
template <typename K>
inline int allow_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess
             ? RCX_OK
             : RCX_ERR_CUDA;
}

// ---- k_rope.cu
int rope_apply_launch(const RopeArgs& a, int dtype, int grid, int block, cudaStream_t stream);

// ---- k_merge.cu
int merge_launch(const MergeArgs& a, int out_dtype, int grid, cudaStream_t stream);

// ---- k_attn_simt_*.cu (one unit per input/output dtype pair)
int attn_simt_launch_f32_f32(const AttnArgs& a, cudaStream_t stream);
int attn_simt_launch_f32_bf16(const AttnArgs& a, cudaStream_t stream);
int attn_simt_launch_bf16_f32(const AttnArgs& a, cudaStream_t stream);
int attn_simt_launch_bf16_bf16(const AttnArgs& a, cudaStream_t stream);

// ---- k_attn_tc.cu
int attn_tc_launch(const AttnArgs& a, const rcx_tensor& q, const rcx_tensor& k, const rcx_tensor& v,
                   const rcx_tensor& o, cudaStream_t stream);
void attn_tc_set_inject(int64_t spins);

// ---- k_decode.cu
int decode_launch(const DecodeArgs& a, int G, bool tensor_core, dim3 grid, cudaStream_t stream);
int decode_i8_launch(const DecodeArgs& a, int G, const float* k_scale, const float* v_scale, dim3 grid,
                     cudaStream_t stream);
int decode_combine_launch(const DecodeArgs& a, int out_dtype, int grid, cudaStream_t stream);
// rows16: bf16 rows and code rows both 16-byte aligned (eight-lanes-per-row kernel)
int quantize_i8_launch(const QuantArgs& a, bool rows16, int grid, cudaStream_t stream);

// Device status words: every translation unit whose kernels have bounded
// waits keeps its own word; these read one into *status and clear it
// (stream-ordered, synchronising `stream`).
int status_exchange_attn_tc(cudaStream_t stream, int* status);
int status_exchange_rope(cudaStream_t stream, int* status);

}  // namespace rcx

// SIMT attention launcher, __nv_bfloat16 inputs and float output.
#include <cuda_bf16.h>
#define RCX_SIMT_IN __nv_bfloat16
#define RCX_SIMT_OUT float
#define RCX_SIMT_NAME attn_simt_launch_bf16_f32
#include "k_attn_simt.inc"

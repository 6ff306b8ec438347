// SIMT attention launcher, __nv_bfloat16 inputs and __nv_bfloat16 output.
#include <cuda_bf16.h>
#define RCX_SIMT_IN __nv_bfloat16
#define RCX_SIMT_OUT __nv_bfloat16
#define RCX_SIMT_NAME attn_simt_launch_bf16_bf16
#include "k_attn_simt.inc"

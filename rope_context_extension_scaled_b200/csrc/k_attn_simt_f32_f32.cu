// SIMT attention launcher, float inputs and float output.
#include <cuda_bf16.h>
#define RCX_SIMT_IN float
#define RCX_SIMT_OUT float
#define RCX_SIMT_NAME attn_simt_launch_f32_f32
#include "k_attn_simt.inc"

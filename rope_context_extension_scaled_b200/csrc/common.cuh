// Shared device helpers of librcx: views, bf16 packing, precise RoPE angles.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/rcx.h"

namespace rcx {

// Launch parameters of a [B, N, H, d] view (element strides, stride[3] == 1).
struct View4 {
  void* ptr;
  int64_t B, N, H, D;
  int64_t sb, sn, sh;
};

inline View4 make_view(const rcx_tensor& t) {
  View4 v;
  v.ptr = t.ptr;
  v.B = t.shape[0]; v.N = t.shape[1]; v.H = t.shape[2]; v.D = t.shape[3];
  v.sb = t.stride[0]; v.sn = t.stride[1]; v.sh = t.stride[2];
  return v;
}

// Up to 128 pairs of rotation frequencies, passed by value in kernel params.
constexpr int kMaxPairs = 128;
struct Freqs {
  double theta[kMaxPairs];
};

// cos/sin of the rotation angle phi = m * theta for pair frequency theta.
// "Context Extension" concept page, Technical principles: pair (2i, 2i+1) at
// position m turns by m * theta_i.  The product and the reduction modulo 2 pi
// are done in float64 (|m * theta| reaches ~1e6 rad at m = 2^20, where fp32
// spacing is 0.06 rad); the reduced angle in [-pi, pi] then goes through the
// fp32 sincosf of the CUDA math library.  Angle error <= ~5e-7 rad for m < 2^24.
__device__ __forceinline__ void rope_cos_sin(int64_t m, double theta, float& c, float& s) {
  const double kTwoPi = 6.283185307179586476925;
  const double kInvTwoPi = 0.159154943091895335769;
  double phi = (double)m * theta;
  double k = rint(phi * kInvTwoPi);
  double r = fma(-k, kTwoPi, phi);
  sincosf((float)r, &s, &c);
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  float2 r;
  r.x = __uint_as_float(u << 16);
  r.y = __uint_as_float(u & 0xffff0000u);
  return r;
}

__device__ __forceinline__ uint32_t f2_to_bf2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Device status word (RCX_OK or the first RCX_ERR_DEVICE_TIMEOUT recorded).
// The kernels are compiled in several translation units without relocatable
// device code, so each unit that includes this header has its own word;
// device_status_exchange() reads and clears the word of the calling unit.
static __device__ int g_device_status = 0;

__device__ __forceinline__ void record_device_error(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// Reads this translation unit's status word into *status and clears it,
// ordered on `stream` (synchronises the stream).
static inline int device_status_exchange(cudaStream_t stream, int* status) {
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
      cudaSuccess)
    return RCX_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return RCX_ERR_CUDA;
  *status = v;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
      return RCX_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return RCX_ERR_CUDA;
  }
  return RCX_OK;
}

}  // namespace rcx

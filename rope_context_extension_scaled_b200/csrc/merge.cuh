// merge_partials: LSE-weighted merge of two partial attention results.
//
// "Context window extension: 4K to 1M" 5.3 accumulates each ring step's block
// output into the running output; kwkr.cn 2.2 aggregates online.  With softmax
// partials that sum needs the weights w = exp(lse - max):
//   o = (w_a o_a + w_b o_b) / (w_a + w_b),  lse = max + ln(w_a + w_b).
// Memory-bound: each thread merges 4 consecutive fp32 values of one
// (b, n, h) row; the row's two LSEs are read by every thread of the row
// (L1 hits).  Rows of two empty partials give o = 0, lse = -inf.
#pragma once
#include "common.cuh"

namespace rcx {

struct MergeArgs {
  View4 oa, ob, oo;         // oo: output view (may alias oa)
  float* la; const float* lb; float* lo;
  int64_t la_sb, la_sh, lb_sb, lb_sh, lo_sb, lo_sh;   // lse strides ([B, H, N], unit on N)
  int64_t rows;             // B * N * H
  int d4;                   // d / 4
};

template <typename Tout>
__device__ __forceinline__ void store4(Tout* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(f2_to_bf2(v.x, v.y), f2_to_bf2(v.z, v.w));
}

template <typename Tout>
__global__ void __launch_bounds__(256) merge_kernel(const MergeArgs a) {
  // d4 divides 32: a warp covers 32 / d4 whole rows per iteration, and the
  // loop trip count is uniform across the warp, so the in-place LSE write can
  // wait for every lane's LSE read with __syncwarp().
  const int rows_per_warp = 32 / a.d4;
  const int lane = threadIdx.x & 31;
  const int sub = lane / a.d4, c = lane % a.d4;
  const int64_t H = a.oa.H, N = a.oa.N;
  const int64_t nwarps = (int64_t)gridDim.x * blockDim.x / 32;
  for (int64_t rg = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; rg * rows_per_warp < a.rows;
       rg += nwarps) {
    const int64_t row = rg * rows_per_warp + sub;
    const bool valid = row < a.rows;
    const int64_t h = row % H;
    const int64_t bn = row / H;
    const int64_t n = bn % N, b = bn / N;
    float lse = -INFINITY;
    if (valid) {
      // Issue every load before any arithmetic so they are all in flight.
      const float lsa = a.la[b * a.la_sb + h * a.la_sh + n];
      const float lsb = a.lb[b * a.lb_sb + h * a.lb_sh + n];
      const float4 x = *reinterpret_cast<const float4*>(
          reinterpret_cast<const float*>(a.oa.ptr) + b * a.oa.sb + n * a.oa.sn + h * a.oa.sh + 4 * c);
      const float4 y = *reinterpret_cast<const float4*>(
          reinterpret_cast<const float*>(a.ob.ptr) + b * a.ob.sb + n * a.ob.sn + h * a.ob.sh + 4 * c);
      const float m = fmaxf(lsa, lsb);
      float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m != -INFINITY) {
        const float wa = (lsa == -INFINITY) ? 0.f : expf(lsa - m);
        const float wb = (lsb == -INFINITY) ? 0.f : expf(lsb - m);
        const float inv = 1.f / (wa + wb);
        const float ca = wa * inv, cb = wb * inv;
        r = make_float4(ca * x.x + cb * y.x, ca * x.y + cb * y.y, ca * x.z + cb * y.z, ca * x.w + cb * y.w);
        lse = m + logf(wa + wb);
      }
      store4<Tout>(reinterpret_cast<Tout*>(a.oo.ptr) + b * a.oo.sb + n * a.oo.sn + h * a.oo.sh + 4 * c, r);
    }
    __syncwarp();
    if (valid && c == 0) a.lo[b * a.lo_sb + h * a.lo_sh + n] = lse;
  }
}

}  // namespace rcx

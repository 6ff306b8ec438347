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
  // A warp walks tokens (b, n) and, per token, all heads: 32 / d4 heads per
  // step, each lane owning 4 consecutive values of one row.  The token index
  // is divided once per token, not per element.  Loop trip counts are uniform
  // across the warp, so the in-place LSE write can wait for every lane's LSE
  // read with __syncwarp().
  const int rows_per_warp = 32 / a.d4;
  const int lane = threadIdx.x & 31;
  const int sub = lane / a.d4, c = lane % a.d4;
  const int64_t H = a.oa.H, N = a.oa.N;
  const int64_t ntok = a.rows / H;
  const int64_t nwarps = (int64_t)gridDim.x * blockDim.x / 32;
  const float* oa = reinterpret_cast<const float*>(a.oa.ptr);
  const float* ob = reinterpret_cast<const float*>(a.ob.ptr);
  Tout* oo = reinterpret_cast<Tout*>(a.oo.ptr);
  for (int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; tok < ntok; tok += nwarps) {
    const int64_t b = tok / N, n = tok - b * N;
    const float* pa = oa + b * a.oa.sb + n * a.oa.sn + 4 * c;
    const float* pb = ob + b * a.ob.sb + n * a.ob.sn + 4 * c;
    Tout* po = oo + b * a.oo.sb + n * a.oo.sn + 4 * c;
    const float* la = a.la + b * a.la_sb + n;
    const float* lb = a.lb + b * a.lb_sb + n;
    float* lo = a.lo + b * a.lo_sb + n;
    // Four rows per lane per step: every load of the step is issued before
    // any arithmetic, so 8 x 16 bytes per lane are in flight.
    constexpr int kU = 4;
    for (int64_t h0 = 0; h0 < H; h0 += (int64_t)kU * rows_per_warp) {
      float lsa[kU], lsb[kU];
      float4 x[kU], y[kU];
      bool valid[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t h = h0 + (int64_t)u * rows_per_warp + sub;
        valid[u] = h < H;
        if (valid[u]) {
          lsa[u] = la[h * a.la_sh];
          lsb[u] = lb[h * a.lb_sh];
          x[u] = *reinterpret_cast<const float4*>(pa + h * a.oa.sh);
          y[u] = *reinterpret_cast<const float4*>(pb + h * a.ob.sh);
        }
      }
      float lse[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t h = h0 + (int64_t)u * rows_per_warp + sub;
        lse[u] = -INFINITY;
        if (valid[u]) {
          const float m = fmaxf(lsa[u], lsb[u]);
          float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
          if (m != -INFINITY) {
            const float wa = (lsa[u] == -INFINITY) ? 0.f : expf(lsa[u] - m);
            const float wb = (lsb[u] == -INFINITY) ? 0.f : expf(lsb[u] - m);
            const float inv = 1.f / (wa + wb);
            const float ca = wa * inv, cb = wb * inv;
            r = make_float4(ca * x[u].x + cb * y[u].x, ca * x[u].y + cb * y[u].y, ca * x[u].z + cb * y[u].z,
                            ca * x[u].w + cb * y[u].w);
            lse[u] = m + logf(wa + wb);
          }
          store4<Tout>(po + h * a.oo.sh, r);
        }
      }
      __syncwarp();
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t h = h0 + (int64_t)u * rows_per_warp + sub;
        if (valid[u] && c == 0) lo[h * a.lo_sh] = lse[u];
      }
    }
  }
}

}  // namespace rcx

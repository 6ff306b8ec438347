// rope_apply: rotate Q and K by R(m) -- memory-bound elementwise kernel.
//
// "Context Extension" concept page, Technical principles: q_m = R(m) W_q x_m,
// k_n = R(n) W_k x_n with R(m) turning each pair (2i, 2i+1) by m * theta_i.
//
// Layout: [B, N, H, d] views, unit stride on d.  Each CTA takes kTok tokens at
// a time: it computes the d/2 (cos, sin) pairs of each token once into shared
// memory (float64 angle reduction, see rope_cos_sin), then every thread
// rotates 16-byte chunks (8 bf16 or 4 fp32 values) of all Q and K heads of
// those tokens.  Algorithmic traffic: read + write of every element once.
#pragma once
#include "common.cuh"

namespace rcx {

struct RopeArgs {
  View4 q_in, q_out, k_in, k_out;   // ptr == nullptr: operand skipped
  const int64_t* positions;         // nullptr: m = n
  int64_t n_tok;                    // B * N
  int64_t N;
  int pairs;                        // d / 2
  Freqs f;
};

constexpr int kRopeTok = 8;
constexpr int kRopeThreads = 256;

template <typename T>
__device__ __forceinline__ void rope_chunk(const T* src, T* dst, const float2* cs);

// 8 bf16 = 4 pairs per 16-byte chunk
template <>
__device__ __forceinline__ void rope_chunk<__nv_bfloat16>(const __nv_bfloat16* src, __nv_bfloat16* dst,
                                                          const float2* cs) {
  uint4 u = *reinterpret_cast<const uint4*>(src);
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    float2 x = bf2_to_f2(w[p]);
    float2 a = cs[p];  // (cos, sin)
    w[p] = f2_to_bf2(x.x * a.x - x.y * a.y, x.x * a.y + x.y * a.x);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// 4 fp32 = 2 pairs per 16-byte chunk
template <>
__device__ __forceinline__ void rope_chunk<float>(const float* src, float* dst, const float2* cs) {
  float4 u = *reinterpret_cast<const float4*>(src);
  float2 a = cs[0], b = cs[1];
  float4 r;
  r.x = u.x * a.x - u.y * a.y;
  r.y = u.x * a.y + u.y * a.x;
  r.z = u.z * b.x - u.w * b.y;
  r.w = u.z * b.y + u.w * b.x;
  *reinterpret_cast<float4*>(dst) = r;
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads) rope_apply_kernel(const RopeArgs a) {
  constexpr int kElems = 16 / sizeof(T);       // elements per chunk
  constexpr int kPairsPerChunk = kElems / 2;
  __shared__ float2 cs[kRopeTok][kMaxPairs];
  const int pairs = a.pairs;
  const int chunks_per_head = (2 * pairs) / kElems;
  const int hq = a.q_in.ptr ? (int)a.q_in.H : 0;
  const int hk = a.k_in.ptr ? (int)a.k_in.H : 0;
  const int chunks_per_tok = (hq + hk) * chunks_per_head;

  for (int64_t tok0 = (int64_t)blockIdx.x * kRopeTok; tok0 < a.n_tok; tok0 += (int64_t)gridDim.x * kRopeTok) {
    const int ntok = (int)(a.n_tok - tok0 < kRopeTok ? a.n_tok - tok0 : kRopeTok);
    for (int e = threadIdx.x; e < ntok * pairs; e += blockDim.x) {
      const int t = e / pairs, i = e % pairs;
      const int64_t n = (tok0 + t) % a.N;
      const int64_t m = a.positions ? a.positions[n] : n;
      float c, s;
      rope_cos_sin(m, a.f.theta[i], c, s);
      cs[t][i] = make_float2(c, s);
    }
    __syncthreads();
    const int total = ntok * chunks_per_tok;
#pragma unroll 4
    for (int e = threadIdx.x; e < total; e += blockDim.x) {
      const int t = e / chunks_per_tok;
      int r = e - t * chunks_per_tok;
      const int h = r / chunks_per_head;
      const int c = r - h * chunks_per_head;
      const int64_t tok = tok0 + t;
      const int64_t b = tok / a.N, n = tok - b * a.N;
      const View4& vi = (h < hq) ? a.q_in : a.k_in;
      const View4& vo = (h < hq) ? a.q_out : a.k_out;
      const int hh = (h < hq) ? h : h - hq;
      const int64_t off_i = b * vi.sb + n * vi.sn + hh * vi.sh + (int64_t)c * kElems;
      const int64_t off_o = b * vo.sb + n * vo.sn + hh * vo.sh + (int64_t)c * kElems;
      rope_chunk<T>(reinterpret_cast<const T*>(vi.ptr) + off_i, reinterpret_cast<T*>(vo.ptr) + off_o,
                    &cs[t][c * kPairsPerChunk]);
    }
    __syncthreads();
  }
}

}  // namespace rcx

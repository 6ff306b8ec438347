// rope_apply: rotate Q and K by R(m) -- memory-bound elementwise kernel.
//
// "Context Extension" concept page, Technical principles: q_m = R(m) W_q x_m,
// k_n = R(n) W_k x_n with R(m) turning each pair (2i, 2i+1) by m * theta_i.
//
// Layout: [B, N, H, d] views with unit stride on d and 16-byte aligned rows.
// The unit of work is (token n, 16-byte piece j of a head): a piece holds 8
// bf16 or 4 fp32 values, i.e. 4 or 2 pairs, and the same pairs of every Q and
// K head of token n turn by the same angles.  So a thread computes the angles
// of its unit once (float64 product and reduction modulo 2 pi, see
// rope_cos_sin) and applies them to that piece of all Hq + Hk heads, with the
// loads of kRopeGroup heads in flight at a time.  No shared memory and no
// barrier: the angle work is 4 (or 2) exact sincos per Hq + Hk pieces, small
// beside the 32 bytes of HBM traffic each piece costs.  A CTA's threads take
// tokens in rows of d-pieces (blockDim = tokens x pieces-per-head), so a
// thread keeps its piece j, and with it its pair frequencies, for the whole
// grid-stride loop, and a warp's loads of one head cover whole 16-byte
// pieces of consecutive tokens.  Algorithmic traffic: one read and one write
// of every element.
#pragma once
#include "common.cuh"

namespace rcx {

struct RopeArgs {
  View4 q_in, q_out, k_in, k_out;   // ptr == nullptr: operand skipped
  const int64_t* positions;         // nullptr: m = n
  int64_t n_tok;                    // B * N
  int64_t N;
  int d_chunks;                     // 16-byte pieces per head: d * element size / 16
  Freqs f;
};

constexpr int kRopeThreads = 256;   // upper bound of blockDim (tokens per pass x d_chunks)
constexpr int kRopeGroup = 8;       // heads whose pieces one thread has in flight at once
constexpr int kRopeCtasPerSm = 8;   // grid = SMs x 8 (about three resident per SM)

template <typename T>
__device__ __forceinline__ void rope_chunk_regs(uint4& u, const float2* cs);

// 8 bf16 = 4 pairs per 16-byte chunk
template <>
__device__ __forceinline__ void rope_chunk_regs<__nv_bfloat16>(uint4& u, const float2* cs) {
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 x = bf2_to_f2(w[p]);
    const float2 a = cs[p];  // (cos, sin)
    w[p] = f2_to_bf2(x.x * a.x - x.y * a.y, x.x * a.y + x.y * a.x);
  }
  u = make_uint4(w[0], w[1], w[2], w[3]);
}

// 4 fp32 = 2 pairs per 16-byte chunk
template <>
__device__ __forceinline__ void rope_chunk_regs<float>(uint4& u, const float2* cs) {
  const float x0 = __uint_as_float(u.x), y0 = __uint_as_float(u.y);
  const float x1 = __uint_as_float(u.z), y1 = __uint_as_float(u.w);
  const float2 a = cs[0], b = cs[1];
  u.x = __float_as_uint(x0 * a.x - y0 * a.y);
  u.y = __float_as_uint(x0 * a.y + y0 * a.x);
  u.z = __float_as_uint(x1 * b.x - y1 * b.y);
  u.w = __float_as_uint(x1 * b.y + y1 * b.x);
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads, 3) rope_apply_kernel(const RopeArgs a) {
  constexpr int kElems = 16 / sizeof(T);        // elements per piece
  constexpr int kPairsPerChunk = kElems / 2;
  const int dch = a.d_chunks;
  const int tpb = blockDim.x / dch;             // tokens per CTA pass
  const int j = threadIdx.x % dch;              // this thread's piece of a head, fixed
  double th[kPairsPerChunk];
#pragma unroll
  for (int q = 0; q < kPairsPerChunk; ++q) th[q] = a.f.theta[j * kPairsPerChunk + q];
  const int hq = a.q_in.ptr ? (int)a.q_in.H : 0;
  const int H = hq + (a.k_in.ptr ? (int)a.k_in.H : 0);
  const T* qi = static_cast<const T*>(a.q_in.ptr);
  const T* ki = static_cast<const T*>(a.k_in.ptr);
  T* qo = static_cast<T*>(a.q_out.ptr);
  T* ko = static_cast<T*>(a.k_out.ptr);
  const int64_t step = (int64_t)gridDim.x * tpb;
  for (int64_t n = (int64_t)blockIdx.x * tpb + threadIdx.x / dch; n < a.n_tok; n += step) {
    const int64_t b = a.N == a.n_tok ? 0 : n / a.N;
    const int64_t nn = n - b * a.N;
    const int64_t e = (int64_t)j * kElems;
    const int64_t qin0 = b * a.q_in.sb + nn * a.q_in.sn + e, qout0 = b * a.q_out.sb + nn * a.q_out.sn + e;
    const int64_t kin0 = b * a.k_in.sb + nn * a.k_in.sn + e, kout0 = b * a.k_out.sb + nn * a.k_out.sn + e;
    float2 cs[kPairsPerChunk];
    for (int h0 = 0; h0 < H; h0 += kRopeGroup) {
      uint4 v[kRopeGroup];
#pragma unroll
      for (int g = 0; g < kRopeGroup; ++g) {
        const int h = h0 + g;
        if (h < H) {
          const T* src = h < hq ? qi + qin0 + h * a.q_in.sh : ki + kin0 + (h - hq) * a.k_in.sh;
          v[g] = __ldcs(reinterpret_cast<const uint4*>(src));
        }
      }
      if (h0 == 0) {                            // angles while the first loads are in flight
        const int64_t m = a.positions ? a.positions[nn] : nn;
#pragma unroll
        for (int q = 0; q < kPairsPerChunk; ++q) rope_cos_sin(m, th[q], cs[q].x, cs[q].y);
      }
#pragma unroll
      for (int g = 0; g < kRopeGroup; ++g) {
        const int h = h0 + g;
        if (h < H) {
          rope_chunk_regs<T>(v[g], cs);
          T* dst = h < hq ? qo + qout0 + h * a.q_out.sh : ko + kout0 + (h - hq) * a.k_out.sh;
          *reinterpret_cast<uint4*>(dst) = v[g];
        }
      }
    }
  }
}

}  // namespace rcx

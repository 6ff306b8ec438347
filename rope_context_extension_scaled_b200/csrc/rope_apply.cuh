// rope_apply: rotate Q and K by R(m) -- memory-bound elementwise kernel.
//
// "Context Extension" concept page, Technical principles: q_m = R(m) W_q x_m,
// k_n = R(n) W_k x_n with R(m) turning each pair (2i, 2i+1) by m * theta_i.
//
// Layout: [B, N, H, d] views, unit stride on d.  A CTA takes T tokens per
// iteration (T * chunks-per-token ~ 2048 16-byte chunks).  Phase 1 computes the
// d/2 (cos, sin) pairs of each of the T tokens once into shared memory
// (float64 angle reduction, see rope_cos_sin) together with each token's
// row offsets; phase 2 rotates the chunks (8 bf16 or 4 fp32 values) of all Q
// and K heads of those tokens.  Which (token, head, chunk) a thread handles is
// the same every iteration, so it is decoded once into registers and no
// integer division runs in the data loop.  Algorithmic traffic: one read and
// one write of every element.
#pragma once
#include "common.cuh"

namespace rcx {

struct RopeArgs {
  View4 q_in, q_out, k_in, k_out;   // ptr == nullptr: operand skipped
  const int64_t* positions;         // nullptr: m = n
  int64_t n_tok;                    // B * N
  int64_t N;
  int pairs;                        // d / 2
  int tok_per_iter;                 // T
  Freqs f;
};

constexpr int kRopeThreads = 256;
constexpr int kRopeMaxTok = 64;
constexpr int kRopeSlots = 8;       // chunks per thread per iteration (T * chunks/token <= 2048)

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
__global__ void __launch_bounds__(kRopeThreads) rope_apply_kernel(const RopeArgs a) {
  constexpr int kElems = 16 / sizeof(T);       // elements per chunk
  constexpr int kPairsPerChunk = kElems / 2;
  __shared__ float2 cs[kRopeMaxTok * 64];      // T * pairs <= 4096 (host-checked)
  __shared__ int64_t off[4][kRopeMaxTok];      // per token: q_in, q_out, k_in, k_out row offsets
  const int pairs = a.pairs;
  const int TPI = a.tok_per_iter;
  const int cph = (2 * pairs) / kElems;        // chunks per head
  const int hq = a.q_in.ptr ? (int)a.q_in.H : 0;
  const int hk = a.k_in.ptr ? (int)a.k_in.H : 0;
  const int cpt = (hq + hk) * cph;             // chunks per token
  const int work = TPI * cpt;                  // chunks per iteration (<= kRopeSlots * blockDim)

  // This thread's (token, head, chunk) slots, decoded once.
  // slot_w packs (is-Q << 31) | (head << 16) | chunk.
  int slot_t[kRopeSlots];
  uint32_t slot_w[kRopeSlots];
#pragma unroll
  for (int k = 0; k < kRopeSlots; ++k) {
    const int e = threadIdx.x + k * kRopeThreads;
    slot_t[k] = e < work ? e / cpt : -1;
    const int hc = e < work ? e % cpt : 0;
    const bool isq = hc < hq * cph;
    const int r = isq ? hc : hc - hq * cph;
    slot_w[k] = ((isq ? 1u : 0u) << 31) | ((uint32_t)(r / cph) << 16) | (uint32_t)(r % cph);
  }

  for (int64_t tok0 = (int64_t)blockIdx.x * TPI; tok0 < a.n_tok; tok0 += (int64_t)gridDim.x * TPI) {
    const int ntok = (int)(a.n_tok - tok0 < TPI ? a.n_tok - tok0 : TPI);
    for (int e = threadIdx.x; e < ntok * pairs; e += blockDim.x) {
      const int t = e / pairs, i = e - t * pairs;
      const int64_t tok = tok0 + t;
      const int64_t b = tok / a.N, n = tok - b * a.N;
      if (i == 0) {
        off[0][t] = b * a.q_in.sb + n * a.q_in.sn;
        off[1][t] = b * a.q_out.sb + n * a.q_out.sn;
        off[2][t] = b * a.k_in.sb + n * a.k_in.sn;
        off[3][t] = b * a.k_out.sb + n * a.k_out.sn;
      }
      const int64_t m = a.positions ? a.positions[n] : n;
      float c, s;
      rope_cos_sin(m, a.f.theta[i], c, s);
      cs[t * pairs + i] = make_float2(c, s);
    }
    __syncthreads();
    uint4 u[kRopeSlots];
#pragma unroll
    for (int k = 0; k < kRopeSlots; ++k) {
      const int t = slot_t[k];
      if (t >= 0 && t < ntok) {
        const bool isq = slot_w[k] >> 31;
        const int h = (slot_w[k] >> 16) & 0x7fff, c = slot_w[k] & 0xffff;
        const View4& vi = isq ? a.q_in : a.k_in;
        const T* src = reinterpret_cast<const T*>(vi.ptr) + off[isq ? 0 : 2][t] + h * vi.sh + c * kElems;
        u[k] = *reinterpret_cast<const uint4*>(src);
      }
    }
#pragma unroll
    for (int k = 0; k < kRopeSlots; ++k) {
      const int t = slot_t[k];
      if (t >= 0 && t < ntok) {
        const bool isq = slot_w[k] >> 31;
        const int h = (slot_w[k] >> 16) & 0x7fff, c = slot_w[k] & 0xffff;
        const View4& vo = isq ? a.q_out : a.k_out;
        rope_chunk_regs<T>(u[k], &cs[t * pairs + c * kPairsPerChunk]);
        T* dst = reinterpret_cast<T*>(vo.ptr) + off[isq ? 1 : 3][t] + h * vo.sh + c * kElems;
        *reinterpret_cast<uint4*>(dst) = u[k];
      }
    }
    __syncthreads();
  }
}

}  // namespace rcx

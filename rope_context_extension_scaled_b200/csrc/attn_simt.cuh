// SIMT fp32 blockwise attention: the fp32 path (and a readable statement, on
// the GPU, of the mask, ring order and online softmax the tensor-core kernel
// also follows).
//
// "Context Extension" concept page, FlashAttention section: Q, K, V in tiles of
// B_r x B_c held on chip, local QK^T, online softmax with a running max,
// accumulated output, no n x n matrix in HBM.  KV blocks of kv_block keys are
// visited in Ring-Attention order: a query tile in shard r = i / kv_block sees
// block r first, then r - 1, ... ("Context window extension: 4K to 1M" 5.3).
//
// CTA: 64 query rows of one (batch, head); TPR = d/32 threads per row, thread
// part p holds elements p, p + TPR, p + 2 TPR, ... (conflict-free shared reads).
// K and V tiles of 64 keys are staged in shared memory as fp32, K rotated on
// the way in when RCX_ROTATE_K is set (Q likewise, once).
#pragma once
#include "attn_common.cuh"

namespace rcx {

constexpr int kSimtBR = 64;
constexpr int kSimtBC = 64;

template <typename T>
__device__ __forceinline__ void simt_load_tile(float* dst, const View4& src, int64_t b, int64_t h,
                                               int64_t r0, int nrows, int64_t g0, bool rotate,
                                               const AttnArgs& a) {
  // dst[r][0..D) for rows r < 64 (zero beyond nrows); pairs rotated at the
  // position of global token g0 + r when asked.
  const int D = 2 * a.pairs;
  const T* base = reinterpret_cast<const T*>(src.ptr);
  for (int e = threadIdx.x; e < kSimtBR * a.pairs; e += blockDim.x) {
    const int r = e / a.pairs, i = e % a.pairs;
    float x = 0.f, y = 0.f;
    if (r < nrows) {
      const T* p = base + b * src.sb + (r0 + r) * src.sn + h * src.sh + 2 * i;
      x = to_f<T>(p[0]);
      y = to_f<T>(p[1]);
      if (rotate) {
        const int64_t g = g0 + r;
        const int64_t m = a.positions ? a.positions[g] : g;
        float c, s;
        rope_cos_sin(m, a.f.theta[i], c, s);
        const float xr = x * c - y * s, yr = x * s + y * c;
        x = xr; y = yr;
      }
    }
    dst[r * D + 2 * i] = x;
    dst[r * D + 2 * i + 1] = y;
  }
}

template <typename T, typename Tout, int TPR>
__global__ void __launch_bounds__(kSimtBR * TPR) attn_simt_kernel(const AttnArgs a) {
  constexpr int D = 32 * TPR;
  extern __shared__ float smem[];
  float* Ks = smem;
  float* Vs = smem + kSimtBC * D;

  const int64_t qt = blockIdx.x;
  const int64_t h = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int64_t hk = h / a.G;
  const int tid = threadIdx.x;
  const int row = tid / TPR, part = tid % TPR;
  const int64_t Nq = a.q.N, Nk = a.k.N;
  const int64_t r0 = qt * kSimtBR;
  const int nrows = (int)(Nq - r0 < kSimtBR ? Nq - r0 : kSimtBR);
  const int64_t gi0 = a.q_start + r0;                    // global index of row 0
  const int64_t gi = gi0 + row;                          // this thread's row
  const bool row_ok = row < nrows;

  // Q tile: rotate once while staging, keep this thread's strided slice.
  simt_load_tile<T>(Ks, a.q, b, h, r0, nrows, gi0, a.rope_flags & RCX_ROTATE_Q, a);
  __syncthreads();
  float q[32], acc[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    q[e] = Ks[row * D + e * TPR + part];
    acc[e] = 0.f;
  }
  __syncthreads();

  float m = -INFINITY, l = 0.f;
  const int64_t i_lo = gi0, i_hi = gi0 + nrows - 1;
  const int64_t kv = a.kv_block;
  const int64_t key_end = a.k_start + Nk;                 // one past the last global key
  const int64_t shard = i_lo / kv;
  const int64_t blk_first = a.k_start / kv;
  // Ring order: block shard, shard-1, ..., then wrap (blocks above the shard
  // hold only later keys and fail the causal test).
  const int64_t nblk = (key_end + kv - 1) / kv;
  const int64_t blk_start = min(shard, nblk - 1);          // highest block this call holds
  for (int64_t t = 0; t < nblk; ++t) {
    int64_t blk = blk_start - t;
    if (blk < 0) blk += nblk;
    if (blk < blk_first) continue;
    const int64_t kb0 = max(blk * kv, a.k_start);
    const int64_t kb1 = min((blk + 1) * kv, key_end);
    for (int64_t j0 = kb0; j0 < kb1; j0 += kSimtBC) {
      const int64_t j1 = min(j0 + kSimtBC, kb1);            // exclusive
      if (!tile_any_visible(i_lo, i_hi, j0, j1 - 1, a.window, a.n_sink)) continue;
      const bool full = tile_all_visible(i_lo, i_hi, j0, j1 - 1, a.window, a.n_sink);
      const int nk = (int)(j1 - j0);
      simt_load_tile<T>(Ks, a.k, b, hk, j0 - a.k_start, nk, j0, a.rope_flags & RCX_ROTATE_K, a);
      simt_load_tile<T>(Vs, a.v, b, hk, j0 - a.k_start, nk, j0, false, a);
      __syncthreads();
      float sv[kSimtBC];
      float mt = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < kSimtBC; ++jj) {
        float dsum = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) dsum = fmaf(q[e], Ks[jj * D + e * TPR + part], dsum);
        if (TPR > 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, 1);
        if (TPR > 2) dsum += __shfl_xor_sync(0xffffffffu, dsum, 2);
        float s = dsum * a.scale_log2;
        const bool vis = jj < nk && (full || mask_visible(gi, j0 + jj, a.window, a.n_sink));
        s = vis ? s : -INFINITY;
        sv[jj] = s;
        mt = fmaxf(mt, s);
      }
      const float m_new = fmaxf(m, mt);
      if (m_new != -INFINITY) {
        const float alpha = exp2f(m - m_new);             // m = -inf gives 0
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] *= alpha;
#pragma unroll
        for (int jj = 0; jj < kSimtBC; ++jj) {
          const float p = exp2f(sv[jj] - m_new);
          l += p;
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = fmaf(p, Vs[jj * D + e * TPR + part], acc[e]);
        }
        m = m_new;
      }
      __syncthreads();
    }
  }

  // Epilogue: O = ca * O_prev + cb * acc with cb = 1 / l alone, or the LSE
  // merge with a previous partial result (ring accumulator) when one is given.
  const float lse_b = l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
  float cb = l > 0.f ? 1.f / l : 0.f, ca = 0.f, lse_out = lse_b;
  const float* accp = nullptr;
  if (a.acc.ptr != nullptr && row_ok) {
    accp = reinterpret_cast<const float*>(a.acc.ptr) + b * a.acc.sb + (r0 + row) * a.acc.sn + h * a.acc.sh;
    const float lse_a = a.acc_lse[b * a.acc_lse_sb + h * a.acc_lse_sh + r0 + row];
    const float mm = fmaxf(lse_a, lse_b);
    if (mm == -INFINITY) {
      cb = 0.f;
      lse_out = -INFINITY;
    } else {
      const float wa = expf(lse_a - mm), wb = expf(lse_b - mm), den = wa + wb;
      ca = wa / den;
      cb *= wb / den;
      lse_out = mm + logf(den);
    }
  }
  __syncwarp();   // every part of the row has read the previous LSE before it is overwritten
  if (row_ok) {
    Tout* op = reinterpret_cast<Tout*>(a.o.ptr) + b * a.o.sb + (r0 + row) * a.o.sn + h * a.o.sh;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float x = acc[e] * cb;
      if (accp) x = fmaf(ca, accp[e * TPR + part], x);
      op[e * TPR + part] = from_f<Tout>(x);
    }
    if (a.lse && part == 0) a.lse[b * a.lse_sb + h * a.lse_sh + r0 + row] = lse_out;
  }
}

}  // namespace rcx

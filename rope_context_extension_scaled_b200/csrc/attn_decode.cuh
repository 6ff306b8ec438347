// Decode attention over a long KV cache, split over key ranges, bf16, d = 128.
//
// "Context Extension" concept page, KV-cache section: each new token computes
// its Q, K, V, appends K and V to the cache and attends with its Q to the
// whole cache.  One query row per (batch, head); the keys are global tokens
// 0 .. Nk-1 (already rotated, as stored in the cache), the query is token
// q_index, with the causal / window / sink mask of the prefill kernels.
//
// Memory-bound: every cached key and value is read once.  A CTA takes one KV
// head of one batch entry (all G query heads that share it) and one range of
// keys; its 8 warps split the range.  In a warp, lane l owns dimensions
// 4l .. 4l+3 and holds those dimensions of all G query rows in registers, so a
// key row is one coalesced 256-byte read.  The G partial dot products of a
// key are summed over the warp with a transpose-reduce (each step halves the
// set of heads a lane carries), after which lane l holds the score of head
// (l >> (5 - log2 G)).  Keys are taken 16 at a time: batch max, one rescale of
// the running state, then P V with the per-head p broadcast by shuffles.
// The 8 warps merge their states in shared memory and the CTA writes an fp32
// partial (O, LSE); a second kernel merges the partials of all key ranges
// with the LSE-weighted rule of the ring merge.
#pragma once
#include "attn_common.cuh"

namespace rcx {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecBatch = 16;                 // keys per warp step
constexpr int kDecMaxG = 8;

struct DecodeArgs {
  View4 q, k, v, o;             // q, o: [B, 1, Hq, 128]; k, v: [B, Nk, Hkv, 128]
  float* lse;                   // [B, Hq] (stride lse_sb, lse_sh) or null
  int64_t lse_sb, lse_sh;
  float* part_o;                // [splits, B, Hq, 128] fp32
  float* part_lse;              // [splits, B, Hq]
  int splits;
  int64_t keys_per_split;
  int64_t q_index;              // global token index of the query
  int64_t window, n_sink;
  float scale_log2;
  const int64_t* positions;     // nullptr: identity
  int rope_q;
  int G;
  Freqs f;
};

__device__ __forceinline__ float dec_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int G>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(const DecodeArgs a) {
  constexpr int LG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;   // log2 G
  const int split = blockIdx.x;
  const int hk = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int my_head = lane >> (5 - LG);                          // head whose score this lane ends with

  // ---- Q rows of the group in registers (rotated at the query's position)
  float qv[G][4];
  const int64_t qpos = a.positions ? a.positions[a.q_index] : a.q_index;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16* qp =
        reinterpret_cast<const __nv_bfloat16*>(a.q.ptr) + b * a.q.sb + (int64_t)(hk * G + g) * a.q.sh + 4 * lane;
    const uint2 u = *reinterpret_cast<const uint2*>(qp);
    const float2 x0 = bf2_to_f2(u.x), x1 = bf2_to_f2(u.y);
    qv[g][0] = x0.x; qv[g][1] = x0.y; qv[g][2] = x1.x; qv[g][3] = x1.y;
    if (a.rope_q) {
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        float c, s;
        rope_cos_sin(qpos, a.f.theta[2 * lane + pp], c, s);
        const float x = qv[g][2 * pp], y = qv[g][2 * pp + 1];
        qv[g][2 * pp] = x * c - y * s;
        qv[g][2 * pp + 1] = x * s + y * c;
      }
    }
  }

  // ---- this warp's key range
  const int64_t Nk = a.k.N;
  const int64_t s_lo = (int64_t)split * a.keys_per_split;
  const int64_t s_hi = min(Nk, s_lo + a.keys_per_split);
  const int64_t per_warp = (s_hi - s_lo + kDecWarps - 1) / kDecWarps;
  const int64_t k_lo = s_lo + warp * per_warp;
  const int64_t k_hi = min(s_hi, k_lo + per_warp);
  const int64_t qi = a.q_index;

  float m = -INFINITY, l = 0.f;          // state of head my_head (replicated over its lanes)
  float acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[g][e] = 0.f;

  const __nv_bfloat16* kbase = reinterpret_cast<const __nv_bfloat16*>(a.k.ptr) + b * a.k.sb + hk * a.k.sh + 4 * lane;
  const __nv_bfloat16* vbase = reinterpret_cast<const __nv_bfloat16*>(a.v.ptr) + b * a.v.sb + hk * a.v.sh + 4 * lane;

  for (int64_t j0 = k_lo; j0 < k_hi; j0 += kDecBatch) {
    // skip batches with no visible key (window / causal)
    const int64_t j1 = min(k_hi, j0 + kDecBatch) - 1;
    if (!tile_any_visible(qi, qi, j0, j1, a.window, a.n_sink)) continue;
    uint2 kr[kDecBatch], vr[kDecBatch];
#pragma unroll
    for (int t = 0; t < kDecBatch; ++t) {
      const int64_t j = j0 + t;
      kr[t] = j <= j1 ? *reinterpret_cast<const uint2*>(kbase + j * a.k.sn) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < kDecBatch; ++t) {
      const int64_t j = j0 + t;
      vr[t] = j <= j1 ? *reinterpret_cast<const uint2*>(vbase + j * a.v.sn) : make_uint2(0u, 0u);
    }
    float sc[kDecBatch];
#pragma unroll
    for (int t = 0; t < kDecBatch; ++t) {
      const float2 k0 = bf2_to_f2(kr[t].x), k1 = bf2_to_f2(kr[t].y);
      float part[G];
#pragma unroll
      for (int g = 0; g < G; ++g)
        part[g] = fmaf(qv[g][3], k1.y, fmaf(qv[g][2], k1.x, fmaf(qv[g][1], k0.y, qv[g][0] * k0.x)));
      // transpose-reduce: after step o, a lane keeps half of its heads
#pragma unroll
      for (int st = 0, n = G; st < LG; ++st, n >>= 1) {
        const int off = 16 >> st;
        const bool hi = lane & off;
#pragma unroll
        for (int g = 0; g < n / 2; ++g) {
          const float send = hi ? part[g] : part[g + n / 2];
          const float keep = hi ? part[g + n / 2] : part[g];
          part[g] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      float sres = part[0];
#pragma unroll
      for (int off = 16 >> LG; off >= 1; off >>= 1) sres += __shfl_xor_sync(0xffffffffu, sres, off);
      const int64_t j = j0 + t;
      const bool vis = j <= j1 && mask_visible(qi, j, a.window, a.n_sink);
      sc[t] = vis ? sres * a.scale_log2 : -INFINITY;
    }
    float bm = sc[0];
#pragma unroll
    for (int t = 1; t < kDecBatch; ++t) bm = fmaxf(bm, sc[t]);
    const float m_new = fmaxf(m, bm);
    const float mref = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = dec_exp2(m - mref);          // 0 when m = -inf
    float p[kDecBatch];
    float ps = 0.f;
#pragma unroll
    for (int t = 0; t < kDecBatch; ++t) {
      p[t] = dec_exp2(sc[t] - mref);
      ps += p[t];
    }
    l = l * alpha + ps;
    m = m_new;
    // rescale and accumulate every head this lane carries in acc
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float ag = __shfl_sync(0xffffffffu, alpha, g << (5 - LG));
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[g][e] *= ag;
    }
#pragma unroll
    for (int t = 0; t < kDecBatch; ++t) {
      const float2 v0 = bf2_to_f2(vr[t].x), v1 = bf2_to_f2(vr[t].y);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pg = __shfl_sync(0xffffffffu, p[t], g << (5 - LG));
        acc[g][0] = fmaf(pg, v0.x, acc[g][0]);
        acc[g][1] = fmaf(pg, v0.y, acc[g][1]);
        acc[g][2] = fmaf(pg, v1.x, acc[g][2]);
        acc[g][3] = fmaf(pg, v1.y, acc[g][3]);
      }
    }
  }

  // ---- merge the warps' states in shared memory
  __shared__ float sm_m[kDecWarps][kDecMaxG], sm_l[kDecWarps][kDecMaxG];
  __shared__ float sm_acc[kDecWarps][kDecMaxG][128];
  if ((lane & ((32 >> LG) - 1)) == 0) {
    sm_m[warp][my_head] = m;
    sm_l[warp][my_head] = l;
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e) sm_acc[warp][g][4 * lane + e] = acc[g][e];
  __syncthreads();
  for (int e = threadIdx.x; e < G * 128; e += blockDim.x) {
    const int g = e / 128, dd = e % 128;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) mm = fmaxf(mm, sm_m[w][g]);
    const float mr = mm == -INFINITY ? 0.f : mm;
    float lt = 0.f, ot = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float wgt = dec_exp2(sm_m[w][g] - mr);
      lt += wgt * sm_l[w][g];
      ot += wgt * sm_acc[w][g][dd];
    }
    const int64_t hq = (int64_t)hk * G + g;
    const int64_t pidx = ((int64_t)split * a.q.B + b) * a.q.H + hq;
    a.part_o[pidx * 128 + dd] = lt > 0.f ? ot / lt : 0.f;
    if (dd == 0) a.part_lse[pidx] = lt > 0.f ? (mr + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// Tensor-core variant (mma.sync m16n8k16, bf16 in, fp32 accumulate), computed
// transposed so that the G <= 8 query heads are the 8 columns of each MMA and
// no operand row is padding: per warp and 16-key tile,
//   S^T [16 keys x 8 heads]  = K [16 keys x 128] . Q^T        (8 MMAs over d)
//   O^T [128 x 8 heads]     += V^T [128 x 16 keys] . P^T      (8 MMAs over d)
// K and V tiles go to shared memory with cp.async (three stages per warp, two
// tiles in flight while one is computed) and come back as MMA operands with
// ldmatrix (K) and ldmatrix.trans (V^T).  Each lane's S^T fragment holds keys
// g, g + 8 of heads 2c, 2c + 1 (g = lane / 4, c = lane % 4): the online softmax
// reduces each head's max and sum over the 8 lanes of a column, and
// movmatrix.trans turns the bf16 P^T fragment into the B operand of the P V
// product.  The 4 warps merge their states in shared memory as above.

constexpr int kDmWarps = 4;
constexpr int kDmStages = 3;
constexpr int kDmRow = 272;                                // 256-byte row + 16 pad (ldmatrix banks)
constexpr int kDmTile = 16 * kDmRow;                       // one 16-key K or V tile
constexpr int kDmStage = 2 * kDmTile;                      // K and V
constexpr int kDmSmem = kDmWarps * kDmStages * kDmStage;   // 104,448 B: two CTAs per SM
static_assert(kDmSmem >= kDmWarps * kDecMaxG * 128 * 4, "merge area aliases the stage buffers");

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <int G>
__global__ void __launch_bounds__(kDmWarps * 32) attn_decode_mma_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t dm_smem[];
  __shared__ float sm_m[kDmWarps][kDecMaxG], sm_l[kDmWarps][kDecMaxG];
  const int split = blockIdx.x;
  const int hk = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, c = lane & 3;

  // ---- Q^T operand: head g, dims 16 kc + {2c, 2c + 1} (b0) and + 8 (b1)
  uint32_t qb[8][2];
  if (g < G) {
    const __nv_bfloat16* qp =
        reinterpret_cast<const __nv_bfloat16*>(a.q.ptr) + b * a.q.sb + (int64_t)(hk * G + g) * a.q.sh;
    const int64_t qpos = a.positions ? a.positions[a.q_index] : a.q_index;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int d0 = 16 * kc + 2 * c + 8 * hf;
        float2 x = bf2_to_f2(*reinterpret_cast<const uint32_t*>(qp + d0));
        if (a.rope_q) {
          float cs, sn;
          rope_cos_sin(qpos, a.f.theta[d0 >> 1], cs, sn);
          x = make_float2(x.x * cs - x.y * sn, x.x * sn + x.y * cs);
        }
        qb[kc][hf] = f2_to_bf2(x.x, x.y);
      }
  } else {
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) qb[kc][0] = qb[kc][1] = 0u;
  }

  // ---- this warp's key range, in 16-key tiles from k_lo
  const int64_t Nk = a.k.N;
  const int64_t s_lo = (int64_t)split * a.keys_per_split;
  const int64_t s_hi = min(Nk, s_lo + a.keys_per_split);
  const int64_t per_warp = ((s_hi - s_lo + kDmWarps - 1) / kDmWarps + 15) / 16 * 16;
  const int64_t k_lo = s_lo + warp * per_warp;
  const int64_t k_hi = min(s_hi, k_lo + per_warp);
  const int64_t qi = a.q_index;
  auto next_visible = [&](int64_t t) {
    while (t < k_hi && !tile_any_visible(qi, qi, t, min(t + 15, k_hi - 1), a.window, a.n_sink)) {
      if (t > qi) return k_hi;
      t += 16;
    }
    return t < k_hi ? t : k_hi;
  };

  const __nv_bfloat16* kbase = reinterpret_cast<const __nv_bfloat16*>(a.k.ptr) + b * a.k.sb + hk * a.k.sh;
  const __nv_bfloat16* vbase = reinterpret_cast<const __nv_bfloat16*>(a.v.ptr) + b * a.v.sb + hk * a.v.sh;
  const uint32_t wbuf = static_cast<uint32_t>(__cvta_generic_to_shared(dm_smem)) + warp * kDmStages * kDmStage;
  // K and V rows t .. t + 15 -> stage st (rows past the range are zero-filled)
  auto issue = [&](int64_t t, int st) {
    if (t < k_hi) {
      const uint32_t ks = wbuf + st * kDmStage;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        const int key = e >> 4, col = e & 15;
        const int64_t j = t + key;
        const bool ok = j < k_hi;
        const int64_t jj = ok ? j : t;
        const int bytes = ok ? 16 : 0;
        const uint32_t off = key * kDmRow + col * 16;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(ks + off),
                     "l"(kbase + jj * a.k.sn + col * 8), "r"(bytes)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(ks + kDmTile + off),
                     "l"(vbase + jj * a.v.sn + col * 8), "r"(bytes)
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // heads 2c, 2c + 1 (l: this lane's share)
  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;

  // ldmatrix lane addresses (row offsets inside a tile)
  const int mi = lane >> 3, r8 = lane & 7;
  const uint32_t k_lane = (r8 + (mi & 1) * 8) * kDmRow + (mi >> 1) * 16;    // K: keys x d
  const uint32_t v_lane = (r8 + (mi >> 1) * 8) * kDmRow + (mi & 1) * 16;    // V^T from V: keys x d

  int64_t t0 = next_visible(k_lo);
  int64_t t1 = t0 < k_hi ? next_visible(t0 + 16) : k_hi;
  issue(t0, 0);
  issue(t1, 1);
  int st = 0;
  while (t0 < k_hi) {
    const int64_t t2 = t1 < k_hi ? next_visible(t1 + 16) : k_hi;
    issue(t2, st == 0 ? 2 : st - 1);
    asm volatile("cp.async.wait_group 2;" ::: "memory");
    __syncwarp();
    const uint32_t ks = wbuf + st * kDmStage, vs = ks + kDmTile;
    // S^T = K Q^T
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      uint32_t ka[4];
      ldsm_x4(ka, ks + k_lane + kc * 32);
      mma_bf16_16816(sacc, ka, qb[kc][0], qb[kc][1]);
    }
    // online softmax per head over keys t0 + g, t0 + g + 8
    const int64_t ja = t0 + g, jb = t0 + g + 8;
    const bool va = ja < k_hi && mask_visible(qi, ja, a.window, a.n_sink);
    const bool vb = jb < k_hi && mask_visible(qi, jb, a.window, a.n_sink);
    float sv[4];
    sv[0] = va ? sacc[0] * a.scale_log2 : -INFINITY;
    sv[1] = va ? sacc[1] * a.scale_log2 : -INFINITY;
    sv[2] = vb ? sacc[2] * a.scale_log2 : -INFINITY;
    sv[3] = vb ? sacc[3] * a.scale_log2 : -INFINITY;
    float p[4], alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = fmaxf(sv[h], sv[h + 2]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m[h], mx);
      const float mref = m_new == -INFINITY ? 0.f : m_new;
      alpha[h] = dec_exp2(m[h] - mref);
      p[h] = dec_exp2(sv[h] - mref);
      p[h + 2] = dec_exp2(sv[h + 2] - mref);
      l[h] = l[h] * alpha[h] + (p[h] + p[h + 2]);
      m[h] = m_new;
    }
    const uint32_t pb0 = movmatrix_t(f2_to_bf2(p[0], p[1]));   // keys 2c, 2c + 1 of head g
    const uint32_t pb1 = movmatrix_t(f2_to_bf2(p[2], p[3]));   // keys 2c + 8, 2c + 9
    // O^T = alpha O^T + V^T P^T
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      o[mt][0] *= alpha[0];
      o[mt][1] *= alpha[1];
      o[mt][2] *= alpha[0];
      o[mt][3] *= alpha[1];
      uint32_t va4[4];
      ldsm_x4_t(va4, vs + v_lane + mt * 32);
      mma_bf16_16816(o[mt], va4, pb0, pb1);
    }
    __syncwarp();   // stage st is refilled two iterations on
    st = st == kDmStages - 1 ? 0 : st + 1;
    t0 = t1;
    t1 = t2;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");

  // ---- merge the warps' states in shared memory (aliases the stage buffers)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 4);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 8);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 16);
  }
  __syncthreads();
  float* sm_o = reinterpret_cast<float*>(dm_smem);   // [warps][kDecMaxG][128]
  if (g == 0) {
    sm_m[warp][2 * c] = m[0];
    sm_m[warp][2 * c + 1] = m[1];
    sm_l[warp][2 * c] = l[0];
    sm_l[warp][2 * c + 1] = l[1];
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    float* w0 = sm_o + (warp * kDecMaxG + 2 * c) * 128 + 16 * mt + g;
    w0[0] = o[mt][0];
    w0[128] = o[mt][1];
    w0[8] = o[mt][2];
    w0[128 + 8] = o[mt][3];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * 128; e += blockDim.x) {
    const int hh = e / 128, dd = e % 128;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDmWarps; ++w) mm = fmaxf(mm, sm_m[w][hh]);
    const float mr = mm == -INFINITY ? 0.f : mm;
    float lt = 0.f, ot = 0.f;
#pragma unroll
    for (int w = 0; w < kDmWarps; ++w) {
      const float wgt = dec_exp2(sm_m[w][hh] - mr);
      lt += wgt * sm_l[w][hh];
      ot += wgt * sm_o[(w * kDecMaxG + hh) * 128 + dd];
    }
    const int64_t hq = (int64_t)hk * G + hh;
    const int64_t pidx = ((int64_t)split * a.q.B + b) * a.q.H + hq;
    a.part_o[pidx * 128 + dd] = lt > 0.f ? ot / lt : 0.f;
    if (dd == 0) a.part_lse[pidx] = lt > 0.f ? (mr + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
  }
}

// Merge the key-range partials of each (batch, query head) row.
template <typename Tout>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeArgs a) {
  // One CTA of 8 warps per (batch, query head) row: warp w merges key ranges
  // w, w + 8, ... (lane c holds dims 4c .. 4c + 3), so the reads of all
  // partials are spread over the CTA, and the 8 warp results merge in shared
  // memory by the same LSE rule.
  __shared__ float sm_m[8], sm_l[8];
  __shared__ float4 sm_o[8][32];
  const int64_t rows = a.q.B * a.q.H;
  const int warp = threadIdx.x / 32, c = threadIdx.x % 32;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    float mm = -INFINITY;
    for (int s = warp; s < a.splits; s += 8) mm = fmaxf(mm, a.part_lse[(int64_t)s * rows + row]);
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (mm != -INFINITY) {
#pragma unroll 4
      for (int s = warp; s < a.splits; s += 8) {
        const float ls = a.part_lse[(int64_t)s * rows + row];
        const float w = ls == -INFINITY ? 0.f : expf(ls - mm);
        const float4 x = *reinterpret_cast<const float4*>(a.part_o + ((int64_t)s * rows + row) * 128 + 4 * c);
        r.x += w * x.x; r.y += w * x.y; r.z += w * x.z; r.w += w * x.w;
        wsum += w;
      }
    }
    if (c == 0) {
      sm_m[warp] = mm;
      sm_l[warp] = wsum;
    }
    sm_o[warp][c] = r;
    __syncthreads();
    if (warp == 0) {
      float mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < 8; ++w) mt = fmaxf(mt, sm_m[w]);
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      float lse = -INFINITY;
      if (mt != -INFINITY) {
        float lt = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const float f = sm_m[w] == -INFINITY ? 0.f : expf(sm_m[w] - mt);
          const float4 x = sm_o[w][c];
          o.x += f * x.x; o.y += f * x.y; o.z += f * x.z; o.w += f * x.w;
          lt += f * sm_l[w];
        }
        const float inv = 1.f / lt;
        o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
        lse = mt + logf(lt);
      }
      const int64_t b = row / a.q.H, h = row % a.q.H;
      Tout* op = reinterpret_cast<Tout*>(a.o.ptr) + b * a.o.sb + h * a.o.sh + 4 * c;
      if constexpr (sizeof(Tout) == 2) {
        *reinterpret_cast<uint2*>(op) = make_uint2(f2_to_bf2(o.x, o.y), f2_to_bf2(o.z, o.w));
      } else {
        *reinterpret_cast<float4*>(op) = o;
      }
      if (c == 0 && a.lse) a.lse[b * a.lse_sb + h * a.lse_sh] = lse;
    }
    __syncthreads();
  }
}

}  // namespace rcx

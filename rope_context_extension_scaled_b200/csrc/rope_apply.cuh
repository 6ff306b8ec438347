// rope_apply: rotate Q and K by R(m) -- memory-bound elementwise kernel.
//
// "Context Extension" concept page, Technical principles: q_m = R(m) W_q x_m,
// k_n = R(n) W_k x_n with R(m) turning each pair (2i, 2i+1) by m * theta_i.
//
// Layout: [B, N, H, d] views, unit stride on d.  A CTA takes T tokens per
// iteration (T * chunks-per-token ~ 2048 16-byte chunks).  Each iteration
// first issues the loads of its chunks (8 bf16 or 4 fp32 values; all Q and K
// heads of the T tokens), then, while they are in flight, computes the d/2
// (cos, sin) pairs of each token once into shared memory (float64 angle
// reduction, see rope_cos_sin; two buffers, so one barrier per iteration),
// then rotates and stores.  Which (token, head, chunk) a thread handles is the
// same every iteration, so it is decoded once into registers.  Algorithmic
// traffic: one read and one write of every element.
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
constexpr int kRopeMaxAngles = 2048;  // T * pairs per buffer
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

// kSame: the output views have the input views' strides (in place, or out of
// place with one layout), so one set of slot offsets serves loads and stores.
template <typename T, bool kSame>
__global__ void __launch_bounds__(kRopeThreads, 2) rope_apply_kernel(const RopeArgs a) {
  constexpr int kElems = 16 / sizeof(T);       // elements per chunk
  constexpr int kPairsPerChunk = kElems / 2;
  __shared__ float2 cs[2][kRopeMaxAngles];     // T * pairs <= kRopeMaxAngles (host-checked)
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

  // Element offsets of this thread's slots relative to the first token of an
  // iteration: constant while the iteration's tokens stay in one batch entry.
  int64_t rel_in[kRopeSlots], rel_out[kSame ? 1 : kRopeSlots];
#pragma unroll
  for (int k = 0; k < kRopeSlots; ++k) {
    const bool isq = slot_w[k] >> 31;
    const int h = (slot_w[k] >> 16) & 0x7fff, c = slot_w[k] & 0xffff;
    const View4& vi = isq ? a.q_in : a.k_in;
    const View4& vo = isq ? a.q_out : a.k_out;
    const int t = slot_t[k] < 0 ? 0 : slot_t[k];
    rel_in[k] = t * vi.sn + h * vi.sh + c * kElems;
    if (!kSame) rel_out[kSame ? 0 : k] = t * vo.sn + h * vo.sh + c * kElems;
  }

  int buf = 0;
  for (int64_t tok0 = (int64_t)blockIdx.x * TPI; tok0 < a.n_tok; tok0 += (int64_t)gridDim.x * TPI, buf ^= 1) {
    const int ntok = (int)(a.n_tok - tok0 < TPI ? a.n_tok - tok0 : TPI);
    const int64_t b0 = tok0 / a.N, n0 = tok0 - b0 * a.N;
    const bool one_batch = n0 + ntok <= a.N;      // no batch boundary inside this iteration
    // 1. loads of this iteration's chunks
    uint4 u[kRopeSlots];
#pragma unroll
    for (int k = 0; k < kRopeSlots; ++k) {
      const int t = slot_t[k];
      if (t >= 0 && t < ntok) {
        const bool isq = slot_w[k] >> 31;
        const View4& vi = isq ? a.q_in : a.k_in;
        int64_t off;
        if (one_batch) {
          off = b0 * vi.sb + n0 * vi.sn + rel_in[k];
        } else {
          int64_t bo = b0, no = n0 + t;
          while (no >= a.N) { no -= a.N; ++bo; }
          off = bo * vi.sb + no * vi.sn + (rel_in[k] - t * vi.sn);
        }
        u[k] = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(vi.ptr) + off);
      }
    }
    // 2. angles of this iteration's tokens (overlaps the loads)
    for (int e = threadIdx.x; e < ntok * pairs; e += blockDim.x) {
      const int t = e / pairs, i = e - t * pairs;
      int64_t n = n0 + t;
      while (n >= a.N) n -= a.N;
      const int64_t m = a.positions ? a.positions[n] : n;
      float c, s;
      rope_cos_sin(m, a.f.theta[i], c, s);
      cs[buf][t * pairs + i] = make_float2(c, s);
    }
    __syncthreads();
    // 3. rotate and store
#pragma unroll
    for (int k = 0; k < kRopeSlots; ++k) {
      const int t = slot_t[k];
      if (t >= 0 && t < ntok) {
        const bool isq = slot_w[k] >> 31;
        const int c = slot_w[k] & 0xffff;
        const View4& vo = isq ? a.q_out : a.k_out;
        int64_t off;
        const int64_t rel = kSame ? rel_in[k] : rel_out[kSame ? 0 : k];
        if (one_batch) {
          off = b0 * vo.sb + n0 * vo.sn + rel;
        } else {
          int64_t bo = b0, no = n0 + t;
          while (no >= a.N) { no -= a.N; ++bo; }
          off = bo * vo.sb + no * vo.sn + (rel - t * vo.sn);
        }
        rope_chunk_regs<T>(u[k], &cs[buf][t * pairs + c * kPairsPerChunk]);
        *reinterpret_cast<uint4*>(reinterpret_cast<T*>(vo.ptr) + off) = u[k];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Bulk-copy path for dense layouts ([B, N, H, d] with no gaps, in and out).
// A token's H x d values are one contiguous row, so a chunk of T tokens is one
// contiguous span: cp.async.bulk brings it into shared memory (four stages per
// CTA, three loading while one is rotated; two CTAs per SM).  Two warps build
// the next chunk's T x d/2 (cos, sin) table (with consecutive positions: one
// precise angle per pair and the angle-addition identity for the rest) while
// six warps rotate the current chunk on its way out with coalesced 16-byte
// stores.  Every wait on a copy is bounded (about
// one second) and
// records RCX_ERR_DEVICE_TIMEOUT if it runs out.

constexpr int kRopeBulkStages = 4;
constexpr int kRopeBulkBytes = 18432;      // bytes of one stage (T * token bytes)

struct RopeBulkArgs {
  const void* in;
  void* out;
  const int64_t* positions;    // nullptr: m = n
  int64_t n_tok;               // B * N
  int64_t N;
  int64_t token_bytes;         // H * d * element size
  int tok_per_chunk;           // T
  int pairs;                   // d / 2
  int d;
  Freqs f;
};

__device__ __forceinline__ uint32_t rb_smem(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool rb_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok = 0;
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (it == 0) t0 = t;
    else if (t - t0 > 1000000000ull) {
      record_device_error(RCX_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads, 2) rope_bulk_kernel(const RopeBulkArgs a) {
  // Warps 0-5 rotate chunk i while warps 6-7 build the angle table of chunk
  // i + 1 into the other table buffer; one barrier per chunk.
  constexpr int kElems = 16 / sizeof(T);
  constexpr int kPairsPerChunk = kElems / 2;
  constexpr int kRotThreads = kRopeThreads - 64;
  extern __shared__ __align__(128) uint8_t rb_raw[];
  uint8_t* stage_buf = rb_raw;                                                        // [stages][kRopeBulkBytes]
  float2* cs = reinterpret_cast<float2*>(rb_raw + kRopeBulkStages * kRopeBulkBytes);  // [2][kRopeMaxAngles / 2]
  uint64_t* full = reinterpret_cast<uint64_t*>(cs + kRopeMaxAngles);                  // [stages]
  __shared__ int abort_flag;
  constexpr int kTab = kRopeMaxAngles / 2;

  const int64_t n_chunks = (a.n_tok + a.tok_per_chunk - 1) / a.tok_per_chunk;
  const int64_t first = blockIdx.x, step = gridDim.x;
  const bool rot = threadIdx.x < kRotThreads;
  auto chunk_tokens = [&](int64_t c) {
    const int64_t left = a.n_tok - c * a.tok_per_chunk;
    return (int)(left < a.tok_per_chunk ? left : a.tok_per_chunk);
  };
  auto issue_load = [&](int64_t c, int st) {
    const int64_t t0 = c * a.tok_per_chunk;
    const uint32_t bytes = (uint32_t)(chunk_tokens(c) * a.token_bytes);
    const uint32_t bar = rb_smem(&full[st]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            rb_smem(stage_buf + st * kRopeBulkBytes)),
        "l"(static_cast<const uint8_t*>(a.in) + t0 * a.token_bytes), "r"(bytes), "r"(bar)
        : "memory");
  };
  // Angle table of chunk c into cs[buf]: one precise angle per pair and the
  // angle-addition identity for consecutive positions, else direct angles.
  auto build_table = [&](int64_t c, int buf) {
    const int lt = threadIdx.x - kRotThreads;          // 0 .. 63
    const int ntok = chunk_tokens(c);
    const int64_t t0 = c * a.tok_per_chunk;
    const int64_t n0 = t0 - (t0 / a.N) * a.N;
    float2* tab = cs + buf * kTab;
    if (!a.positions && n0 + ntok <= a.N) {
      for (int p = lt; p < a.pairs; p += 64) {
        float cc, sn, c1, s1;
        rope_cos_sin(n0, a.f.theta[p], cc, sn);
        rope_cos_sin(1, a.f.theta[p], c1, s1);
        tab[p] = make_float2(cc, sn);
        for (int t = 1; t < ntok; ++t) {
          const float c2 = cc * c1 - sn * s1, s2 = sn * c1 + cc * s1;
          cc = c2;
          sn = s2;
          tab[t * a.pairs + p] = make_float2(cc, sn);
        }
      }
    } else {
      for (int e = lt; e < ntok * a.pairs; e += 64) {
        const int t = e / a.pairs, p = e - t * a.pairs;
        int64_t n = n0 + t;
        while (n >= a.N) n -= a.N;
        const int64_t m = a.positions ? a.positions[n] : n;
        float cc, sn;
        rope_cos_sin(m, a.f.theta[p], cc, sn);
        tab[t * a.pairs + p] = make_float2(cc, sn);
      }
    }
  };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < kRopeBulkStages; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(rb_smem(&full[st])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int st = 0; st < kRopeBulkStages; ++st)
      if (first + st * step < n_chunks) issue_load(first + st * step, st);
  }
  if (!rot && first < n_chunks) build_table(first, 0);
  __syncthreads();

  int i = 0;
  for (int64_t c = first; c < n_chunks; c += step, ++i) {
    const int st = i % kRopeBulkStages;
    const int buf = i & 1;
    if (rot) {
      if (!rb_wait(rb_smem(&full[st]), (i / kRopeBulkStages) & 1)) abort_flag = 1;
      if (!abort_flag) {
        const int ntok = chunk_tokens(c);
        const int64_t t0 = c * a.tok_per_chunk;
        const uint8_t* src = stage_buf + st * kRopeBulkBytes;
        uint8_t* dst = static_cast<uint8_t*>(a.out) + t0 * a.token_bytes;
        const float2* tab = cs + buf * kTab;
        const int row_chunks = (int)(a.token_bytes / 16);
        const int d_chunks = a.d / kElems;
        for (int e = threadIdx.x; e < ntok * row_chunks; e += kRotThreads) {
          const int t = e / row_chunks, rc = e - t * row_chunks;
          const int dc = rc % d_chunks;                  // 16-byte chunk within the head
          uint4 u = *reinterpret_cast<const uint4*>(src + (size_t)e * 16);
          rope_chunk_regs<T>(u, &tab[t * a.pairs + dc * kPairsPerChunk]);
          *reinterpret_cast<uint4*>(dst + (size_t)e * 16) = u;
        }
      }
    } else if (c + step < n_chunks) {
      build_table(c + step, buf ^ 1);
    }
    __syncthreads();
    if (abort_flag) break;
    if (threadIdx.x == 0) {
      const int64_t nc = c + (int64_t)kRopeBulkStages * step;
      if (nc < n_chunks) issue_load(nc, st);
    }
  }
  if (threadIdx.x == 0 && abort_flag) {
    // let copies that may still be landing finish before the CTA exits
    for (int st = 0; st < kRopeBulkStages; ++st) {
      uint32_t ok;
      uint64_t t0, t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
      do {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(rb_smem(&full[st])), "r"(0u)
            : "memory");
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      } while (!ok && t - t0 < 100000000ull);
    }
  }
}

}  // namespace rcx

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
// Path for dense layouts ([B, N, H, d] with no gaps, in and out): a token's
// H x d values are one contiguous row, so a chunk of T consecutive tokens is
// one contiguous span of T * token_bytes bytes.  A CTA takes chunks in turn;
// each thread owns the same kRopePieces 16-byte pieces of every chunk (piece
// e = thread + 256 k), so which token and which pairs a piece holds is decoded
// once.  The next chunk's pieces are loaded into registers before the current
// one is rotated and stored, so every thread keeps 2 x kRopePieces 16-byte
// loads in flight; one barrier per chunk publishes the chunk's angles.
//
// Each chunk's (token, pair) cos/sin table is built while the previous chunk
// is rotated (double buffer), so rotating a piece costs table loads and four
// rotations.  With consecutive positions (positions == NULL; position = token
// index within its batch entry) the entry for token t of a chunk starting at
// n0 comes from the angle-addition identity applied once to two exact values,
// the base angle n0 theta (computed by each thread for the pair it owns) and
// the step angle t theta (t < T, a table built once per CTA).  Both come from
// rope_cos_sin, so the applied angle is within a few 1e-7 rad of m theta and
// there is no recurrence whose rounding grows with t.  With explicit
// positions, or in a chunk that crosses into the next batch entry, every
// entry is computed directly.

constexpr int kRopePieces = 4;                         // 16-byte pieces per thread per chunk
constexpr int kRopeBulkBytes = kRopeThreads * kRopePieces * 16;   // 16 KB chunk
constexpr int kRopeBulkTab = kRopeMaxAngles / 2;       // float2 entries of one angle table (>= T * pairs)
constexpr size_t kRopeBulkSmem = 3 * kRopeBulkTab * sizeof(float2);   // step table + two chunk tables

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
  int row_chunks;              // 16-byte pieces per token (token_bytes / 16)
  int d_chunks;                // 16-byte pieces per head (d * element size / 16)
  Freqs f;
};

// cos/sin product (a then b): the angle-addition identity.
__device__ __forceinline__ float2 cs_add(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads, 4) rope_bulk_kernel(const RopeBulkArgs a) {
  constexpr int kElems = 16 / sizeof(T);
  constexpr int kPairsPerChunk = kElems / 2;
  extern __shared__ __align__(16) float2 rb_tabs[];     // [3][kRopeBulkTab]
  const int tid = threadIdx.x;
  const int pairs = a.pairs;
  const bool dense_pos = a.positions == nullptr;
  // tabs[0] = step table [T][pairs] (consecutive positions); tabs[1 + buf] =
  // (cos, sin) of the chunk's entries [t][pairs], double-buffered
  float2* step_tab = rb_tabs;
  auto chunk_tab = [&](int buf) { return rb_tabs + (1 + buf) * kRopeBulkTab; };

  const int64_t n_chunks = (a.n_tok + a.tok_per_chunk - 1) / a.tok_per_chunk;
  const int64_t step = gridDim.x;
  auto chunk_tokens = [&](int64_t c) {
    const int64_t left = a.n_tok - c * a.tok_per_chunk;
    return (int)(left < a.tok_per_chunk ? left : a.tok_per_chunk);
  };
  // Table of chunk c into buffer `buf`, entry e = t * pairs + p.  When 256 is
  // a multiple of pairs, a thread's entries share one pair p, so each thread
  // computes the base angle of its own pair (the redundant sincos keeps every
  // thread's share of the work equal ahead of the next barrier).
  const bool fixed_pair = (kRopeThreads % pairs) == 0;
  auto prepare = [&](int64_t c, int buf) {
    const int ntok = chunk_tokens(c);
    const int64_t t0 = c * a.tok_per_chunk;
    const int64_t n0 = t0 - (t0 / a.N) * a.N;
    const bool consecutive = dense_pos && n0 + ntok <= a.N;
    float2* tab = chunk_tab(buf);
    const int total = ntok * pairs;
    if (consecutive && fixed_pair) {
      if (tid < total) {
        float bc, bs;
        rope_cos_sin(n0, a.f.theta[tid % pairs], bc, bs);
        const float2 base = make_float2(bc, bs);
        for (int e = tid; e < total; e += kRopeThreads) tab[e] = cs_add(base, step_tab[e]);
      }
      return;
    }
    for (int e = tid; e < total; e += kRopeThreads) {
      const int t = e / pairs, p = e - t * pairs;
      float cc, sn;
      if (consecutive) {
        rope_cos_sin(n0, a.f.theta[p], cc, sn);
        tab[e] = cs_add(make_float2(cc, sn), step_tab[e]);
      } else {
        int64_t n = n0 + t;
        while (n >= a.N) n -= a.N;
        rope_cos_sin(a.positions ? a.positions[n] : n, a.f.theta[p], cc, sn);
        tab[e] = make_float2(cc, sn);
      }
    }
  };

  // This thread's pieces: table offset (token * pairs + first pair) of piece
  // e = tid + 256 k.
  int pofs[kRopePieces];
#pragma unroll
  for (int k = 0; k < kRopePieces; ++k) {
    const int e = tid + k * kRopeThreads;
    const int t = e / a.row_chunks;
    pofs[k] = t * pairs + ((e - t * a.row_chunks) % a.d_chunks) * kPairsPerChunk;
  }
  auto load = [&](int64_t c, uint4* u) {
    const int total = chunk_tokens(c) * a.row_chunks;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.in) +
                                                      c * a.tok_per_chunk * a.token_bytes);
#pragma unroll
    for (int k = 0; k < kRopePieces; ++k) {
      const int e = tid + k * kRopeThreads;
      if (e < total) u[k] = src[e];
    }
  };

  if (dense_pos)
    for (int e = tid; e < a.tok_per_chunk * pairs; e += kRopeThreads) {
      const int t = e / pairs, p = e - t * pairs;
      float cc, sn;
      rope_cos_sin(t, a.f.theta[p], cc, sn);
      step_tab[e] = make_float2(cc, sn);
    }
  __syncthreads();
  int64_t c = blockIdx.x;
  if (c < n_chunks) prepare(c, 0);
  uint4 u[kRopePieces], un[kRopePieces];
  if (c < n_chunks) load(c, u);
  for (int i = 0; c < n_chunks; c += step, ++i) {
    const int buf = i & 1;
    __syncthreads();                                  // the table of chunk c is in buffer buf
    const bool more = c + step < n_chunks;
    if (more) load(c + step, un);                     // next chunk's loads in flight during this one
    const int total = chunk_tokens(c) * a.row_chunks;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.out) + c * a.tok_per_chunk * a.token_bytes);
    const float2* tab = chunk_tab(buf);
#pragma unroll
    for (int k = 0; k < kRopePieces; ++k) {
      const int e = tid + k * kRopeThreads;
      if (e < total) {
        float2 cs[kPairsPerChunk];
#pragma unroll
        for (int q = 0; q < kPairsPerChunk; ++q) cs[q] = tab[pofs[k] + q];
        rope_chunk_regs<T>(u[k], cs);
        dst[e] = u[k];
      }
    }
    if (more) {
      prepare(c + step, buf ^ 1);
#pragma unroll
      for (int k = 0; k < kRopePieces; ++k) u[k] = un[k];
    }
  }
}

}  // namespace rcx

// Int8 KV cache: per-row quantisation and decode attention over the codes.
//
// "Context window extension: 4K to 1M" section 6.1 keeps the KV cache in INT8
// instead of 16-bit floats, halving its memory; the "Context Extension"
// concept page lists the same compression in its KV-cache table.  Format
// (the plainest symmetric reading; the pages fix none): one fp32 scale per
// row of d = 128 values (one token of one KV head), scale = amax / 127 and
// code = rint(x * (127 / amax)) in [-127, 127], all decided in IEEE fp32.
// Scales are stored head-major, [B, H, N], so that the scales of a tile of
// consecutive keys of one head are one contiguous row.
//
// Decode over the codes follows attn_decode_mma_kernel (three cp.async stages
// per warp, transposed mma.sync with the G <= 8 query heads as the MMA
// columns), with 32-key tiles so that a tile moves as many bytes as the bf16
// kernel's 16-key tile and the per-tile softmax work is shared by 32 keys, and
// the dequantisation in the tile load:
//  * S^T = Kq Q^T runs on int8 MMAs (m16n8k32, int32 accumulate) with the
//    codes as they are stored: the rotated query of each head is split as
//    q = s_q (128 hi + lo) + e, hi in [-127, 127], lo in [-64, 64],
//    |e| <= s_q / 2 with s_q = amax / (127 * 128), and two MMAs per 32 dims
//    give codes . hi and codes . lo exactly; 128 hi-part + lo-part (|.| < 2^29)
//    times s_q and the key's scale is the logit.  The query error is 15 bits
//    of its largest element, finer than an fp16 operand;
//  * the P V product runs in fp16 (m16n8k16, fp32 accumulate), because an int8
//    code becomes an exact fp16 in three integer/half instructions: the byte
//    with its sign bit flipped (u = code + 128) is placed under the exponent
//    pattern of 1024, which reads as 1024 + u, and 1152 is subtracted (the
//    offset cannot stay in the product: it would grow with the number of keys
//    summed into O);
//  * V codes go into O^T += Vq^T P'^T unscaled, with each key's V scale folded
//    into P: P' = p * s_v / s_max, where s_max is the largest V scale the warp
//    has met so far (so P' stays in [0, 1], clear of fp16 subnormals).  When
//    s_max grows, O is rescaled together with the online-softmax correction,
//    and O * s_max is the warp's result.
// K row reads use the same d permutation trick as the bf16 kernel's first
// form: lane c of a row group takes dims [32c, 32c + 32) of the key in order,
// and Q is laid out with the same permutation, so every dot product is
// unchanged.  The V^T operand comes from ldmatrix.trans of the code tile read
// as 16-bit elements (two dims of one key), which hands each lane dims 2g and
// 2g + 1 of two consecutive keys in one register: A row g of m-tile mt is dim
// 16 mt + 2g and row g + 8 is dim 16 mt + 2g + 1, so each register becomes two
// A registers by two byte selections, and the merge writes the rows back in
// natural order.
#pragma once
#include <cuda_fp16.h>
#include "attn_decode.cuh"

namespace rcx {

// ---------------------------------------------------------------- quantise

// Unsigned division by a run-time constant d, exact for n < 2^31 (Granlund
// and Montgomery, "Division by invariant integers using multiplication",
// 1994): with l = ceil(log2 d), p = 31 + l and m = ceil(2^p / d) (< 2^32),
// floor(n / d) = (n * m) >> p, because m = (2^p + e) / d with 0 <= e < d adds
// n e / (d 2^p) < 2^(31 - p) <= 1 / d to n / d.
struct FastDiv {
  uint32_t m, p;
};

inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  FastDiv f;
  f.p = 31 + l;
  f.m = (uint32_t)(((uint64_t(1) << f.p) + d - 1) / d);
  return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, FastDiv f) {
  return (uint32_t)(((uint64_t)n * f.m) >> f.p);
}

struct QuantArgs {
  View4 x;          // bf16 [B, N, H, 128]
  View4 c;          // int8 [B, N, H, 128]
  float* scale;     // [B, H, N] contiguous (head-major)
  int64_t rows;     // B * N * H
  FastDiv div_h, div_n;    // by H and by N, exact for rows < 2^31
  int fast;         // rows < 2^31: 32-bit row decoding by div_h / div_n
};

// One warp per row; lane l holds dims 4l .. 4l + 3.  A warp takes kQRows rows
// per pass (grid-strided) and issues all their loads before any arithmetic.
constexpr int kQRows = 4;

static __global__ void __launch_bounds__(256) kv_quantize_int8_kernel(const QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x / 32);
  const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  for (int64_t r0 = w0; r0 < a.rows; r0 += kQRows * nwarps) {
    uint2 u[kQRows];
    int64_t off_c[kQRows], sidx[kQRows];
#pragma unroll
    for (int i = 0; i < kQRows; ++i) {
      const int64_t r = r0 + i * nwarps;
      const int64_t rr = r < a.rows ? r : r0;
      int64_t h, n, b;
      if (a.rows < (int64_t(1) << 31)) {          // 32-bit index arithmetic (the usual case)
        const uint32_t r32 = (uint32_t)rr, H32 = (uint32_t)a.x.H, N32 = (uint32_t)a.x.N;
        const uint32_t t32 = r32 / H32;
        h = r32 - t32 * H32;
        n = t32 % N32;
        b = t32 / N32;
      } else {
        h = rr % a.x.H;
        n = (rr / a.x.H) % a.x.N;
        b = rr / (a.x.H * a.x.N);
      }
      const __nv_bfloat16* xp = reinterpret_cast<const __nv_bfloat16*>(a.x.ptr) + b * a.x.sb + n * a.x.sn +
                                h * a.x.sh + 4 * lane;
      u[i] = *reinterpret_cast<const uint2*>(xp);
      off_c[i] = b * a.c.sb + n * a.c.sn + h * a.c.sh + 4 * lane;
      sidx[i] = (b * a.x.H + h) * a.x.N + n;
    }
#pragma unroll
    for (int i = 0; i < kQRows; ++i) {
      const int64_t r = r0 + i * nwarps;
      if (r >= a.rows) break;                      // warp-uniform
      const float2 x01 = bf2_to_f2(u[i].x), x23 = bf2_to_f2(u[i].y);
      const float v[4] = {x01.x, x01.y, x23.x, x23.y};
      float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
      const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int q = __float2int_rn(__fmul_rn(v[e], inv));
        q = q > 127 ? 127 : (q < -127 ? -127 : q);
        packed |= (uint32_t)(q & 0xff) << (8 * e);
      }
      *reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(a.c.ptr) + off_c[i]) = packed;
      if (lane == 0) a.scale[sidx[i]] = am > 0.f ? __fdiv_rn(am, 127.f) : 0.f;
    }
  }
}

// Eight lanes per row, for rows whose bf16 values and codes are both 16-byte
// aligned: lane l of an eight-lane group holds dims 16l .. 16l + 15 (two
// 16-byte loads, so a row is one coalesced 256-byte read), the row max takes
// three shuffles within the group, and the lane stores its 16 codes as one
// 16-byte word.  A warp covers four consecutive rows (in [B, N, H] order) per
// pass and keeps kQPasses passes of loads in flight.  The per-row work (max,
// the two IEEE divisions, the row decoding by multiplicative division) is
// shared by 16 values per lane, which keeps the kernel below the SM's issue
// rate at HBM speed.  Rounding: y = fl(x * inv) satisfies |y| <= 127
// (inv = fl(127 / amax) exceeds 127 / amax by at most half an ulp, so
// |y| < 127.5 and rint(y) is within [-127, 127], where the clamp never acts),
// and fl(y + 1.5 * 2^23) holds rint(y), ties to even, in its low bits (the sum
// lies in [2^23, 2^24), where the fp32 spacing is 1), whose low byte is the
// two's-complement code.  So the codes and scales equal those of
// kv_quantize_int8_kernel.
constexpr int kQPasses = 2;

__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float inv) {
  const float kRound = 12582912.f;                      // 1.5 * 2^23
  const uint32_t qa = __float_as_uint(__fadd_rn(__fmul_rn(a, inv), kRound));
  const uint32_t qb = __float_as_uint(__fadd_rn(__fmul_rn(b, inv), kRound));
  const uint32_t qc = __float_as_uint(__fadd_rn(__fmul_rn(c, inv), kRound));
  const uint32_t qd = __float_as_uint(__fadd_rn(__fmul_rn(d, inv), kRound));
  return __byte_perm(__byte_perm(qa, qb, 0x0040), __byte_perm(qc, qd, 0x0040), 0x5410);
}

static __global__ void __launch_bounds__(256) kv_quantize_int8_r8_kernel(const QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int sub = lane >> 3, el = lane & 7;
  const int64_t quads = (a.rows + 3) / 4;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x / 32);
  const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int64_t N = a.x.N, H = a.x.H;
  for (int64_t p0 = w0; p0 < quads; p0 += kQPasses * nwarps) {
    uint4 u[kQPasses][2];
    int64_t off_c[kQPasses], sidx[kQPasses];
    bool live[kQPasses];
#pragma unroll
    for (int i = 0; i < kQPasses; ++i) {
      const int64_t p = p0 + i * nwarps;
      const int64_t r = 4 * (p < quads ? p : p0) + sub;   // row (b * N + n) * H + h
      live[i] = p < quads && r < a.rows;                   // ragged last quad: repeats a row, stores nothing
      const int64_t rr = r < a.rows ? r : a.rows - 1;
      int64_t b, n, h;
      if (a.fast) {
        const uint32_t r32 = (uint32_t)rr;
        const uint32_t t = fast_div(r32, a.div_h);
        h = r32 - t * (uint32_t)H;
        const uint32_t bb = fast_div(t, a.div_n);
        n = t - bb * (uint32_t)N;
        b = bb;
      } else {
        h = rr % H;
        n = (rr / H) % N;
        b = rr / (H * N);
      }
      const int64_t off_x = b * a.x.sb + n * a.x.sn + h * a.x.sh;
      off_c[i] = b * a.c.sb + n * a.c.sn + h * a.c.sh;
      sidx[i] = (b * H + h) * N + n;
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.x.ptr) + off_x) + 2 * el;
      u[i][0] = __ldcs(src);
      u[i][1] = __ldcs(src + 1);
    }
#pragma unroll
    for (int i = 0; i < kQPasses; ++i) {
      const int64_t p = p0 + i * nwarps;
      if (p >= quads) break;                         // warp-uniform
      float v[16];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t w[4] = {u[i][hf].x, u[i][hf].y, u[i][hf].z, u[i][hf].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = bf2_to_f2(w[e]);
          v[8 * hf + 2 * e] = f.x;
          v[8 * hf + 2 * e + 1] = f.y;
        }
      }
      float am = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) am = fmaxf(am, fabsf(v[e]));
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
      const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
      uint4 q;
      q.x = quant4(v[0], v[1], v[2], v[3], inv);
      q.y = quant4(v[4], v[5], v[6], v[7], inv);
      q.z = quant4(v[8], v[9], v[10], v[11], inv);
      q.w = quant4(v[12], v[13], v[14], v[15], inv);
      if (live[i]) {
        *reinterpret_cast<uint4*>(reinterpret_cast<int8_t*>(a.c.ptr) + off_c[i] + 16 * el) = q;
        if (el == 0) a.scale[sidx[i]] = am > 0.f ? __fdiv_rn(am, 127.f) : 0.f;
      }
    }
  }
}

// ---------------------------------------------------------------- decode

constexpr int kDqWarps = 4;
constexpr int kDqStages = 3;
constexpr int kDqKeys = 32;                                  // keys per tile (two 16-key MMA halves)
constexpr int kDqRow = 144;                                  // 128-byte code row + 16 pad (banks)
constexpr int kDqTile = kDqKeys * kDqRow;                    // one 32-key K or V tile
constexpr int kDqStage = 2 * kDqTile + 2 * 4 * kDqKeys;      // K, V, 32 K scales, 32 V scales
constexpr int kDqSmem = kDqWarps * kDqStages * kDqStage;     // 113,664 B: two CTAs (8 warps) per SM
constexpr int kDqCtasPerSm = 2;
static_assert(kDqSmem >= kDqWarps * kDecMaxG * 128 * 4, "merge area aliases the stage buffers");

__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// S^T tile from int8 codes (A, 16 x 32) and int8 query parts (B, 32 x 8), int32 accumulate
__device__ __forceinline__ void mma_s8_16832(int* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two int8 codes (bytes 0 and 2 of u ^ 0x80808080 selected by sel) -> exact fp16 pair.
__device__ __forceinline__ uint32_t codes_to_h2(uint32_t u_flipped, uint32_t sel) {
  const uint32_t h = __byte_perm(u_flipped, 0x64646464u, sel);      // halves 0x64uu = 1024 + u
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h), __half2half2(__ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&r);                    // 0x6480 = 1152
}

template <int G>
__global__ void __launch_bounds__(kDqWarps * 32) attn_decode_i8_kernel(const DecodeArgs a,
                                                                        const float* __restrict__ k_scale,
                                                                        const float* __restrict__ v_scale) {
  extern __shared__ __align__(128) uint8_t dq_smem[];
  __shared__ float sm_m[kDqWarps][kDecMaxG], sm_l[kDqWarps][kDecMaxG];
  const int split = blockIdx.x;
  const int hk = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, c = lane & 3;

  // ---- Q^T operand (int8 pair): head g, dims [32c, 32c + 32) of the rotated q,
  // split as q = s_q (128 hi + lo) + e with hi in [-127, 127], lo in [-64, 64]
  // and |e| <= s_q / 2, s_q = amax / (127 * 128) per head (15 bits, finer
  // than the fp16 operand's 11).  Word w holds dims 32c + 4w .. 32c + 4w + 3.
  uint32_t qhi[8], qlo[8];
  float sqc[2];                                     // s_q of heads 2c, 2c + 1 (this lane's S columns)
  {
    float qf[32];
    if (g < G) {
      const __nv_bfloat16* qp =
          reinterpret_cast<const __nv_bfloat16*>(a.q.ptr) + b * a.q.sb + (int64_t)(hk * G + g) * a.q.sh + 32 * c;
      const int64_t qpos = a.positions ? a.positions[a.q_index] : a.q_index;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float2 x = bf2_to_f2(*reinterpret_cast<const uint32_t*>(qp + 2 * i));
        if (a.rope_q) {
          float cs, sn;
          rope_cos_sin(qpos, a.f.theta[16 * c + i], cs, sn);
          x = make_float2(x.x * cs - x.y * sn, x.x * sn + x.y * cs);
        }
        qf[2 * i] = x.x;
        qf[2 * i + 1] = x.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) qf[i] = 0.f;
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(qf[i]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));     // lanes 4g .. 4g + 3 hold head g
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    const float inv = am > 0.f ? 16256.f / am : 0.f;
    const float sq = am > 0.f ? am / 16256.f : 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t ph = 0u, pl = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float y = qf[4 * w + e] * inv;
        const float hi = rintf(y * (1.f / 128.f));
        const int lo = __float2int_rn(y - 128.f * hi);
        ph |= ((uint32_t)(int)hi & 0xffu) << (8 * e);
        pl |= ((uint32_t)lo & 0xffu) << (8 * e);
      }
      qhi[w] = ph;
      qlo[w] = pl;
    }
    sqc[0] = __shfl_sync(0xffffffffu, sq, 8 * c);
    sqc[1] = __shfl_sync(0xffffffffu, sq, 8 * c + 4);
  }

  // ---- this warp's key range, in kDqKeys-key tiles from k_lo
  const int64_t Nk = a.k.N, Hkv = a.k.H;
  const int64_t s_lo = (int64_t)split * a.keys_per_split;
  const int64_t s_hi = min(Nk, s_lo + a.keys_per_split);
  const int64_t per_warp = ((s_hi - s_lo + kDqWarps - 1) / kDqWarps + kDqKeys - 1) / kDqKeys * kDqKeys;
  const int64_t k_lo = s_lo + warp * per_warp;
  const int64_t k_hi = min(s_hi, k_lo + per_warp);
  const int64_t qi = a.q_index;
  auto next_visible = [&](int64_t t) {
    while (t < k_hi && !tile_any_visible(qi, qi, t, min(t + kDqKeys - 1, k_hi - 1), a.window, a.n_sink)) {
      if (t > qi) return k_hi;
      t += kDqKeys;
    }
    return t < k_hi ? t : k_hi;
  };

  const int8_t* kbase = reinterpret_cast<const int8_t*>(a.k.ptr) + b * a.k.sb + hk * a.k.sh;
  const int8_t* vbase = reinterpret_cast<const int8_t*>(a.v.ptr) + b * a.v.sb + hk * a.v.sh;
  const float* ksc = k_scale + (b * Hkv + hk) * Nk;          // key j: ksc[j] (head-major scales)
  const float* vsc = v_scale + (b * Hkv + hk) * Nk;
  uint8_t* wptr = dq_smem + warp * kDqStages * kDqStage;
  const uint32_t wbuf = static_cast<uint32_t>(__cvta_generic_to_shared(wptr));
  // ldmatrix row address of this lane inside a 16-key half of a V tile: matrix
  // lane / 8 is keys 0-7 or 8-15 (bit 0) and bytes [0, 16) or [16, 32) of a
  // 32-byte slice (bit 1)
  const uint32_t v_lane = ((lane & 7) + 8 * ((lane >> 3) & 1)) * kDqRow + 16 * (lane >> 4);
  // codes and scales of keys t .. t + 31 -> stage st (keys past the range are
  // zero-filled).  Lane l copies 16-byte piece l % 8 of keys l / 8 + 4i
  // (i < 8) of both tiles; its global and shared offsets are fixed per lane,
  // so a tile costs one 64-bit product per operand and constant steps.
  const int lk = lane >> 3;
  const int8_t* k_lane = kbase + lk * a.k.sn + (lane & 7) * 16;
  const int8_t* v_lane_g = vbase + lk * a.v.sn + (lane & 7) * 16;
  const int64_t k_step = 4 * a.k.sn, v_step = 4 * a.v.sn;
  const uint32_t s_lane = lk * kDqRow + (lane & 7) * 16;
  auto issue = [&](int64_t t, int st) {
    if (t < k_hi) {
      const uint32_t ks = wbuf + st * kDqStage + s_lane;
      const int8_t* kp = k_lane + t * a.k.sn;
      const int8_t* vp = v_lane_g + t * a.v.sn;
      const int64_t rem = k_hi - t;                 // keys of the tile in range (warp-uniform)
      if (rem >= kDqKeys) {
#pragma unroll
        for (int i = 0; i < kDqKeys / 4; ++i) {
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ks + 4 * i * kDqRow), "l"(kp + i * k_step)
                       : "memory");
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ks + kDqTile + 4 * i * kDqRow),
                       "l"(vp + i * v_step)
                       : "memory");
        }
      } else {
#pragma unroll
        for (int i = 0; i < kDqKeys / 4; ++i) {
          const bool ok = lk + 4 * i < rem;
          const int bytes = ok ? 16 : 0;             // zero-fill; the source stays inside the tile's first key
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(ks + 4 * i * kDqRow),
                       "l"(ok ? kp + i * k_step : kp - lk * a.k.sn), "r"(bytes)
                       : "memory");
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(ks + kDqTile + 4 * i * kDqRow),
                       "l"(ok ? vp + i * v_step : vp - lk * a.v.sn), "r"(bytes)
                       : "memory");
        }
      }
      {
        const bool ok = lane < rem;
        const int64_t jj = ok ? t + lane : t;              // one coalesced 128-byte row per operand
        const uint32_t dst = wbuf + st * kDqStage + 2 * kDqTile + lane * 4;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(ksc + jj), "r"(ok ? 4 : 0)
                     : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst + 4 * kDqKeys), "l"(vsc + jj),
                     "r"(ok ? 4 : 0)
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // heads 2c, 2c + 1 (l: this lane's share)
  float smax = 0.f;                                         // largest V scale met so far
  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;

  int64_t t0 = next_visible(k_lo);
  int64_t t1 = t0 < k_hi ? next_visible(t0 + kDqKeys) : k_hi;
  issue(t0, 0);
  issue(t1, 1);
  int st = 0;
  while (t0 < k_hi) {
    const int64_t t2 = t1 < k_hi ? next_visible(t1 + kDqKeys) : k_hi;
    issue(t2, st == 0 ? 2 : st - 1);
    asm volatile("cp.async.wait_group 2;" ::: "memory");
    __syncwarp();
    const uint8_t* ks = wptr + st * kDqStage;
    const float* sk = reinterpret_cast<const float*>(ks + 2 * kDqTile);
    const float* sv_ = sk + kDqKeys;
    // S^T = Kq Q^T for the two 16-key halves u (keys 16u + g, 16u + g + 8 in
    // this lane's rows), dims [32c, 32c + 32) per lane: two independent chains
    float sacc[2][4];                         // codes . (128 hi + lo) of the lane's (key, head) pairs
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint32_t kw[2][8];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint8_t* row = ks + (16 * u + g + 8 * r) * kDqRow + 32 * c;
        const uint4 u0 = *reinterpret_cast<const uint4*>(row);
        const uint4 u1 = *reinterpret_cast<const uint4*>(row + 16);
        kw[r][0] = u0.x; kw[r][1] = u0.y; kw[r][2] = u0.z; kw[r][3] = u0.w;
        kw[r][4] = u1.x; kw[r][5] = u1.y; kw[r][6] = u1.z; kw[r][7] = u1.w;
      }
      // the codes are the A operand as they are: chunk kc is dims 32c + 8kc + [0, 8)
      int shi[4] = {0, 0, 0, 0}, slo[4] = {0, 0, 0, 0};
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        const uint32_t af[4] = {kw[0][2 * kc], kw[1][2 * kc], kw[0][2 * kc + 1], kw[1][2 * kc + 1]};
        mma_s8_16832(shi, af, qhi[2 * kc], qhi[2 * kc + 1]);
        mma_s8_16832(slo, af, qlo[2 * kc], qlo[2 * kc + 1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[u][e] = (float)(128 * shi[e] + slo[e]);   // exact: |S| < 2^29
    }
    // key scales of this lane's keys (u, r): 16u + g + 8r
    float skr[2][2], svr[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        skr[u][r] = sk[16 * u + g + 8 * r];
        svr[u][r] = sv_[16 * u + g + 8 * r];
      }
    // largest V scale of the tile: scales are >= 0, so their bit patterns order
    // like the values and one integer max-reduction over the warp finds it
    const float lmax = fmaxf(fmaxf(svr[0][0], svr[0][1]), fmaxf(svr[1][0], svr[1][1]));
    const float tmax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(lmax)));
    const float smax_new = fmaxf(smax, tmax);
    const float ratio = smax_new > 0.f ? smax / smax_new : 1.f;
    const float inv_smax = smax_new > 0.f ? 1.f / smax_new : 0.f;
    smax = smax_new;
    // per-key mask only on tiles that are ragged or cut by the mask (warp-uniform)
    bool vis[2][2] = {{true, true}, {true, true}};
    if (t0 + kDqKeys > k_hi || !tile_all_visible(qi, qi, t0, t0 + kDqKeys - 1, a.window, a.n_sink)) {
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int64_t j = t0 + 16 * u + g + 8 * r;
          vis[u][r] = j < k_hi && mask_visible(qi, j, a.window, a.n_sink);
        }
    }
    // logits in log2 units: fragment element e of half u is (key 16u + g + 8(e >> 1), head 2c + (e & 1))
    float sv[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = e >> 1;
        sv[u][e] = vis[u][r] ? sacc[u][e] * (sqc[e & 1] * skr[u][r] * a.scale_log2) : -INFINITY;
      }
    float p[2][4], beta[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = fmaxf(fmaxf(sv[0][h], sv[0][h + 2]), fmaxf(sv[1][h], sv[1][h + 2]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m[h], mx);
      const float mref = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = dec_exp2(m[h] - mref);
      float sum = 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        p[u][h] = dec_exp2(sv[u][h] - mref);
        p[u][h + 2] = dec_exp2(sv[u][h + 2] - mref);
        sum += p[u][h] + p[u][h + 2];
      }
      l[h] = l[h] * alpha + sum;
      m[h] = m_new;
      beta[h] = alpha * ratio;
    }
    // O rescale only when some column's factor moved (the max or s_max grew)
    if (__any_sync(0xffffffffu, beta[0] != 1.f || beta[1] != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= beta[0];
        o[mt][1] *= beta[1];
        o[mt][2] *= beta[0];
        o[mt][3] *= beta[1];
      }
    }
    // O^T += Vq^T P'^T per half u, P' = p * s_v / s_max transposed into the B
    // operand.  ldmatrix.trans of the V codes (16-bit elements = two dims of
    // one key) gives lane (g, c) dims 2g, 2g + 1 of keys 2c, 2c + 1 in one
    // register, so two byte selections make A rows "dim 16 mt + 2g" (row g)
    // and "dim 16 mt + 2g + 1" (row g + 8).
    const uint32_t vs_lane = wbuf + st * kDqStage + kDqTile + v_lane;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float wa = svr[u][0] * inv_smax, wb = svr[u][1] * inv_smax;
      const uint32_t pb0 = movmatrix_t(f2_to_h2(p[u][0] * wa, p[u][1] * wa));   // keys 2c, 2c + 1 of head g
      const uint32_t pb1 = movmatrix_t(f2_to_h2(p[u][2] * wb, p[u][3] * wb));   // keys 2c + 8, 2c + 9
#pragma unroll
      for (int mp = 0; mp < 4; ++mp) {
        uint32_t rr[4];
        ldsm_x4_t(rr, vs_lane + 16 * u * kDqRow + 32 * mp);   // rr0/rr1: keys 0-7 / 8-15, dims 32mp + [0, 16); rr2/rr3: + 16
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t x0 = rr[2 * h] ^ 0x80808080u, x1 = rr[2 * h + 1] ^ 0x80808080u;
          const uint32_t af[4] = {codes_to_h2(x0, 0x4240), codes_to_h2(x0, 0x4341), codes_to_h2(x1, 0x4240),
                                  codes_to_h2(x1, 0x4341)};
          mma_f16_16816(o[2 * mp + h], af, pb0, pb1);
        }
      }
    }
    __syncwarp();   // stage st is refilled two iterations on
    st = st == kDqStages - 1 ? 0 : st + 1;
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
  float* sm_o = reinterpret_cast<float*>(dq_smem);   // [warps][kDecMaxG][128]
  if (g == 0) {
    sm_m[warp][2 * c] = m[0];
    sm_m[warp][2 * c + 1] = m[1];
    sm_l[warp][2 * c] = l[0];
    sm_l[warp][2 * c + 1] = l[1];
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    // C rows: g -> dim 16mt + 2g, g + 8 -> dim 16mt + 2g + 1; columns: heads 2c, 2c + 1
    float* w0 = sm_o + (warp * kDecMaxG + 2 * c) * 128 + 16 * mt + 2 * g;
    w0[0] = o[mt][0] * smax;
    w0[128] = o[mt][1] * smax;
    w0[1] = o[mt][2] * smax;
    w0[128 + 1] = o[mt][3] * smax;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * 128; e += blockDim.x) {
    const int hh = e / 128, dd = e % 128;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDqWarps; ++w) mm = fmaxf(mm, sm_m[w][hh]);
    const float mr = mm == -INFINITY ? 0.f : mm;
    float lt = 0.f, ot = 0.f;
#pragma unroll
    for (int w = 0; w < kDqWarps; ++w) {
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

}  // namespace rcx

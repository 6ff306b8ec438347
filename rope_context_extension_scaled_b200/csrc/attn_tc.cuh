// Tensor-core (tcgen05 / TMEM / TMA) blockwise causal attention, bf16, d = 128.
//
// What it computes is the FlashAttention recipe of the "Context Extension"
// concept page (FlashAttention section): Q, K, V cut into B_r x B_c tiles kept
// on chip, S = QK^T per tile, an online softmax with a running max, O
// accumulated tile by tile, no n x n matrix in HBM -- with the RoPE rotation of
// Q folded into the Q tile load ("Technical principles" of the same page), a
// causal / sliding-window / sink mask ("Context window extension: 4K to 1M"
// 4.1, 4.2), GQA, the YaRN temperature in the logit scale (same page 2.4) and
// KV blocks visited in Ring-Attention order (same page 5.3).
//
// B200 design: a persistent kernel, one CTA per SM (grid = SM count, or the
// number of work items if smaller), each CTA walking work items blockIdx.x,
// blockIdx.x + gridDim.x, ... in a static heaviest-first, KV-head-major order.
// A work item is two Q tiles (slots) of 128 rows that share every K/V tile:
// two query heads of one GQA group over the same rows, or (odd group size)
// rows r and r + 128 of one head.  320 threads:
//   warps 0-3  softmax for Q tile 0 (one thread per row; TMEM lanes 0-127)
//   warps 4-7  softmax for Q tile 1
//   warp  8    producer: per item the two Q tiles, then the item's K and V
//              tiles through a two-stage ring of 128B-swizzled shared-memory
//              buffers (lane 0 issues the TMA copies); the whole warp
//              computes the base rotation angles of the item's Q tiles
//   warp  9    MMA issuer (the converged warp waits, one elected lane issues
//              tcgen05.mma and tcgen05.commit) and TMEM owner
// TMEM (512 columns x 128 lanes, fp32): S0 | S1 | O0 | O1, 128 columns each.
// The softmax writes P as packed bf16 over the first 64 columns of its S, 16
// columns at a time as it is produced, and O += P V reads P straight from
// TMEM (the .kind::f16 form with A in TMEM).  Issue order per KV tile
// PV0(j), S0(j+1), PV1(j), S1(j+1) ping-pongs the softmax warpgroups against
// the tensor core.
// Across items: the next item's Q tiles are loaded as soon as the last S MMA
// of the current item has read the Q buffers, and its first S MMAs follow the
// current item's last PV while the softmax warps write the current item's
// output, so the tensor core does not wait for a CTA launch between items.
// Q is rotated in shared memory before its first MMA; with consecutive
// positions the angle of row r = 16 a + b of a tile starting at token m0 is
// base(m0) x step(16 a) x step(b) (angle-addition identity over three exact
// cos/sin values: per-item bases from the producer, step tables built once
// per CTA), otherwise each angle is computed directly.
// Rescaling of O is lazy: the reference max only moves when the row max grows
// by more than 2^8, so most tiles skip the TMEM round trip of O.
// The epilogue either writes O / l and the LSE, or merges them into a previous
// partial result over other keys (fp32 O and LSE, e.g. a ring accumulator) by
// the LSE rule before writing.
// Every mbarrier wait is bounded (about one second); on expiry the kernel
// records RCX_ERR_DEVICE_TIMEOUT, raises a CTA-wide abort flag, lets its own
// TMA copies and MMAs drain, frees TMEM and returns.
#pragma once
#include <cudaTypedefs.h>
#include <atomic>
#include "attn_common.cuh"

namespace rcx {

constexpr int kTcBM = 128;          // query rows per Q tile
constexpr int kTcBN = 128;          // keys per KV tile
constexpr int kTcD = 128;           // head dim
constexpr int kTcStages = 2;        // K/V pipeline depth
constexpr int kTcThreads = 320;
constexpr int kWarpProd = 8;        // producer warp
constexpr int kWarpMma = 9;         // MMA-issuing warp
constexpr uint32_t kTileBytes = kTcBM * kTcD * 2;   // 32 KB bf16 tile
constexpr uint32_t kHalfTileBytes = kTileBytes / 2; // one 64-column swizzled block
constexpr float kLazyRescale = 8.0f;                // log2 units
constexpr uint64_t kWaitLimitNs = 1000000000ull;    // one second

struct TcParams {
  AttnArgs a;
  int pair_heads;        // 1: slots are heads h, h+1 over the same rows; 0: rows r, r+128 of one head
  int n_rb;              // row blocks per (batch, head-or-pair)
  int n_hg;              // heads (or head pairs) per batch
  int n_items;           // n_rb * n_hg * batch
  int64_t inject_spins;  // test hook: wait this long on a barrier nobody signals
};

// Shared-memory layout (offsets from a 1024-byte aligned base).
constexpr uint32_t kSmQ = 0;                                  // 2 Q tiles
constexpr uint32_t kSmK = kSmQ + 2 * kTileBytes;              // stages of K
constexpr uint32_t kSmV = kSmK + kTcStages * kTileBytes;      // stages of V
constexpr uint32_t kSmBar = kSmV + kTcStages * kTileBytes;    // barriers, TMEM slot, abort flag
constexpr uint32_t kSmRot = kSmBar + 512;                     // rotation tables
constexpr int kRotHi = 8, kRotLo = 16;                        // row r = 16 a + b of a Q tile
constexpr uint32_t kSmRotBytes = (kRotHi + kRotLo + 2) * 64 * 8;   // step tables + two base rows (float2)
constexpr uint32_t kSmTotal = kSmRot + kSmRotBytes + 1024;    // + alignment slack

// ------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false when the CTA is aborting or the limit passed
// (the latter records the timeout and raises the abort flag).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       uint64_t limit_ns = kWaitLimitNs, bool honour_abort = true) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(bar, parity)) return true;
    if ((it & 31) == 0) {
      if (honour_abort && *abort_flag) return false;
      if (global_timer() - t0 > limit_ns) {
        if (honour_abort) {
          *abort_flag = 1;
          record_device_error(RCX_ERR_DEVICE_TIMEOUT);
        }
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                              int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T (SS) and D[tmem] (+)= A[tmem] * B[smem]
// (TS), shapes from the instruction descriptor, with each shared-memory
// descriptor passed as its two 32-bit words.  The low word holds start
// address >> 4 in bits 0-13 and LBO >> 4 in bits 16-29; shared memory is
// below 256 KB, so adding (byte offset >> 4) to the low word steps the start
// address without carrying into LBO.  The issuing thread then spends a few
// instructions per MMA: it shares its SM sub-partition with two softmax warps,
// and MMA issue is on the kernel's critical path.
__device__ __forceinline__ void umma_ss_w(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Converged-warp forms: the whole warp executes these and one elected lane
// issues (elect.sync inside the instruction sequence), so the warp stays
// converged and its descriptor arithmetic stays warp-uniform.
__device__ __forceinline__ void umma_ss_e(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_ts_e(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 db;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit_e(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

#define RCX_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                  "=r"(r[i + 6]), "=r"(r[i + 7])
#define RCX_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), \
                  "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive TMEM columns of this warp's 32 lanes -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : RCX_R8(0), RCX_R8(8), RCX_R8(16), RCX_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      RCX_W8(0), RCX_W8(8), RCX_W8(16), RCX_W8(24)
      : "memory");
}

// 16 registers per thread -> 16 consecutive TMEM columns of this warp's lanes.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// max of three floats in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float2 cs_mul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 layout
// (start >> 4 at bit 0, leading byte offset >> 4 at 16, stride byte offset
// >> 4 at 32, descriptor version 1 at bit 46, swizzle mode 2 at bit 61).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator,
// M = 128, N = 128; b_mn_major selects an MN-major B (V, d contiguous).
__host__ __device__ constexpr uint32_t idesc_bf16(bool b_mn_major) {
  return (1u << 4)                        // D format f32
         | (1u << 7)                      // A format bf16
         | (1u << 10)                     // B format bf16
         | ((b_mn_major ? 1u : 0u) << 16) // B major
         | ((uint32_t)(kTcBN >> 3) << 17) // N / 8
         | ((uint32_t)(kTcBM >> 4) << 24);// M / 16
}

// ------------------------------------------------------------ tile walk

// KV tiles (128 keys, local index t covers keys k_start + 128 t ...) that a
// work item may see, in Ring-Attention block order: the block holding the
// item's query rows first, then the blocks below it, then (wrapping) the
// blocks above.  Visible tiles are the window/causal range [main_lo,
// main_hi] and the sink tiles [0, sink_hi].  32-bit arithmetic: the host keeps
// global token indices below 2^31.
struct TileWalk {
  int main_lo, main_hi, sink_hi, top;
  int k0, kvb;
  int blk, blk_min, blk_max, blk_start;
  int cur, phase;
};

__device__ __forceinline__ int tw_block_of(const TileWalk& w, int t) { return (w.k0 + t * kTcBN) / w.kvb; }

__device__ __forceinline__ int tw_first_tile(const TileWalk& w, int blk) {
  const int x = blk * w.kvb - w.k0;
  return x <= 0 ? 0 : (x + kTcBN - 1) / kTcBN;
}

__device__ __forceinline__ void tw_init(TileWalk& w, int i_lo, int i_hi, const AttnArgs& a) {
  const int Nk = (int)a.k.N, ks = (int)a.k_start;
  const int key_end = ks + Nk;
  w.k0 = ks;
  w.kvb = (int)a.kv_block;
  w.main_lo = 0x3fffffff;
  w.main_hi = -1;
  w.sink_hi = -1;
  w.phase = 2;
  w.cur = -1;
  const int a1 = min(i_hi, key_end - 1) - ks;                 // last causal key (local)
  if (a1 < 0) return;
  const int win = (int)a.window;
  const int a0 = win > 0 ? max(i_lo - win + 1 - ks, 0) : 0;
  if (a0 <= a1) {
    w.main_lo = a0 / kTcBN;
    w.main_hi = a1 / kTcBN;
  }
  if (win > 0 && a.n_sink > ks) {
    const int s_last = min(min((int)a.n_sink - ks, Nk) - 1, a1);   // last sink key (local)
    if (s_last >= 0) w.sink_hi = min(s_last / kTcBN, w.main_lo - 1);
  }
  w.top = w.main_hi >= w.main_lo ? w.main_hi : w.sink_hi;
  if (w.top < 0) return;
  w.blk_min = tw_block_of(w, 0);
  w.blk_max = tw_block_of(w, w.top);
  w.blk_start = min(max(i_lo / w.kvb, w.blk_min), w.blk_max);
  w.blk = w.blk_start;
  w.phase = 0;
}

__device__ __forceinline__ bool tw_next(TileWalk& w, int& tile) {
  while (w.phase < 2) {
    const int first = tw_first_tile(w, w.blk);
    const int last = min(tw_first_tile(w, w.blk + 1) - 1, w.top);
    int c = max(w.cur, first);
    if (c > w.sink_hi && c < w.main_lo) c = w.main_lo;
    if (c <= last) {
      tile = c;
      w.cur = c + 1;
      return true;
    }
    w.cur = -1;
    if (w.phase == 0) {
      if (w.blk > w.blk_min) {
        --w.blk;
      } else {
        w.phase = 1;
        w.blk = w.blk_max;
        if (w.blk <= w.blk_start) w.phase = 2;
      }
    } else {
      if (w.blk - 1 > w.blk_start) --w.blk;
      else w.phase = 2;
    }
  }
  return false;
}

// ------------------------------------------------------------ work items

// One work item: (batch, KV head, row block, head group within the KV head),
// KV head slowest so that the CTAs resident at any time stream the same K/V
// block (which then stays in L2), heaviest row blocks first.
struct Item {
  int bb;
  int head[2];
  int row0[2];
  int kvh;
  int gi_lo, gi_hi;   // global token range of the item's real rows
};

__device__ __forceinline__ Item decode_item(int item, const TcParams& P) {
  const AttnArgs& a = P.a;
  Item it;
  const int hg_per_kv = P.n_hg / (int)a.k.H;
  const int per_kv = P.n_rb * hg_per_kv;
  const int per_b = per_kv * (int)a.k.H;
  it.bb = item / per_b;
  const int kv_i = (item % per_b) / per_kv;
  const int rem = (item % per_b) % per_kv;
  const int rb = P.n_rb - 1 - rem / hg_per_kv;
  const int hg = kv_i * hg_per_kv + rem % hg_per_kv;
  if (P.pair_heads) {
    it.head[0] = 2 * hg;
    it.head[1] = 2 * hg + 1;
    it.row0[0] = it.row0[1] = rb * kTcBM;
  } else {
    it.head[0] = it.head[1] = hg;
    it.row0[0] = rb * 2 * kTcBM;
    it.row0[1] = it.row0[0] + kTcBM;
  }
  it.kvh = it.head[0] / a.G;
  it.gi_lo = (int)a.q_start + it.row0[0];
  it.gi_hi = (int)a.q_start + min(max(it.row0[0], it.row0[1]) + kTcBM, (int)a.q.N) - 1;
  return it;
}

__device__ __forceinline__ int count_tiles(const Item& it, const AttnArgs& a) {
  TileWalk w;
  tw_init(w, it.gi_lo, it.gi_hi, a);
  int n = 0, tile;
  while (tw_next(w, tile)) ++n;
  return n;
}

// ------------------------------------------------------------------ kernel

template <typename Tout>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ TcParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const AttnArgs& a = P.a;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmBar);
  const uint32_t bar0 = smem_addr(bars);
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  enum {
    B_QFULL = 0,      // [2] Q tiles landed
    B_QREADY = 2,     // [2] Q tiles rotated (128 arrivals)
    B_QEMPTY = 4,     // the item's last S MMA has read the Q buffers
    B_BASE = 5,       // base angles of the item's Q tiles written (32 arrivals)
    B_KFULL = 6,      // [stages]
    B_KEMPTY = 6 + kTcStages,
    B_VFULL = 6 + 2 * kTcStages,
    B_VEMPTY = 6 + 3 * kTcStages,
    B_SFULL = 6 + 4 * kTcStages,  // [2]
    B_PREADY = B_SFULL + 2,       // [2] (128 arrivals)
    B_OFINAL = B_PREADY + 2,      // [2]
    B_DRAIN = B_OFINAL + 2,
    B_NEVER = B_DRAIN + 1,
    B_COUNT = B_NEVER + 1
  };
  static_assert(8 * B_COUNT + 16 <= 512, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmBar + 8 * B_COUNT + 8);
  float2* rot_hi = reinterpret_cast<float2*>(smem + kSmRot);   // [8][64]: cos/sin of 16 a theta_p
  float2* rot_lo = rot_hi + kRotHi * 64;                       // [16][64]: cos/sin of b theta_p
  float2* rot_base = rot_lo + kRotLo * 64;                     // [2][64]: per slot, cos/sin of m0 theta_p

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int key_end = (int)(a.k_start + a.k.N);
  const bool table_rot = (a.rope_flags & RCX_ROTATE_Q) && a.positions == nullptr && a.pairs == 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == B_QREADY || i == B_QREADY + 1 || i == B_PREADY || i == B_PREADY + 1) cnt = kTcBM;
      if (i == B_BASE) cnt = 32;
      mbar_init(BAR(i), cnt);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  if (table_rot)
    for (int e = threadIdx.x; e < (kRotHi + kRotLo) * 64; e += kTcThreads) {
      const int row = e / 64, p = e % 64;
      const int64_t m = row < kRotHi ? 16 * row : row - kRotHi;
      float c, sn;
      rope_cos_sin(m, a.f.theta[p], c, sn);
      rot_hi[e] = make_float2(c, sn);
    }
  if (warp == kWarpMma) tmem_alloc(smem_addr(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS[2] = {tmem + 0, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 384};
  // A wait of a whole warp: every lane polls, so the warp stays converged
  // (one lane polling while the others wait in a shuffle made the diverged
  // warp slow to see the barrier complete: 2x slower issue, measured).
  auto warp_wait = [&](int b, uint32_t par) {
    return __all_sync(0xffffffffu, mbar_wait(BAR(b), par, abort_flag));
  };

  if (warp == kWarpProd) {
    // ================================================================ producer
    int jg = 0, it = 0, q_issued = -1;
    int issued_k[kTcStages], issued_v[kTcStages];   // last load index per stage
    for (int s = 0; s < kTcStages; ++s) issued_k[s] = issued_v[s] = -1;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < P.n_items; item += gridDim.x, ++it) {
      const Item itm = decode_item(item, P);
      if (it > 0 && !(ok = warp_wait(B_QEMPTY, (it - 1) & 1))) break;
      if (lane == 0) {
        for (int s = 0; s < 2; ++s) {
          mbar_expect_tx(BAR(B_QFULL + s), kTileBytes);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_tile(sbase + kSmQ + s * kTileBytes + kb * kHalfTileBytes, &tm_q, BAR(B_QFULL + s), kb * 64,
                          itm.head[s], itm.row0[s], itm.bb);
        }
      }
      q_issued = it;
      // base angles of the two Q tiles (first token q_start + row0[s]) while the copies fly
      if (table_rot)
        for (int e = lane; e < 128; e += 32) {
          const int s = e / 64, p = e % 64;
          float c, sn;
          rope_cos_sin(a.q_start + itm.row0[s], a.f.theta[p], c, sn);
          rot_base[e] = make_float2(c, sn);
        }
      mbar_arrive(BAR(B_BASE));
      TileWalk w;
      tw_init(w, itm.gi_lo, itm.gi_hi, a);
      int tile;
      while (tw_next(w, tile)) {
        const int st = jg % kTcStages;
        const uint32_t par = ((jg / kTcStages) & 1) ^ 1;
        if (!(ok = warp_wait(B_KEMPTY + st, par))) break;
        if (lane == 0) {
          mbar_expect_tx(BAR(B_KFULL + st), kTileBytes);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_tile(sbase + kSmK + st * kTileBytes + kb * kHalfTileBytes, &tm_k, BAR(B_KFULL + st), kb * 64,
                          itm.kvh, tile * kTcBN, itm.bb);
        }
        issued_k[st] = jg;
        if (!(ok = warp_wait(B_VEMPTY + st, par))) break;
        if (lane == 0) {
          mbar_expect_tx(BAR(B_VFULL + st), kTileBytes);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_tile(sbase + kSmV + st * kTileBytes + kb * kHalfTileBytes, &tm_v, BAR(B_VFULL + st), kb * 64,
                          itm.kvh, tile * kTcBN, itm.bb);
        }
        issued_v[st] = jg;
        ++jg;
      }
    }
    if (*abort_flag && lane == 0) {
      // drain: wait (bounded, ignoring the abort flag) for copies in flight
      if (q_issued >= 0)
        for (int s = 0; s < 2; ++s) mbar_wait(BAR(B_QFULL + s), q_issued & 1, abort_flag, 100000000ull, false);
      for (int st = 0; st < kTcStages; ++st) {
        if (issued_k[st] >= 0)
          mbar_wait(BAR(B_KFULL + st), (issued_k[st] / kTcStages) & 1, abort_flag, 100000000ull, false);
        if (issued_v[st] >= 0)
          mbar_wait(BAR(B_VFULL + st), (issued_v[st] / kTcStages) & 1, abort_flag, 100000000ull, false);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ================================================================ MMA issuer
    constexpr uint32_t id_qk = idesc_bf16(false);
    constexpr uint32_t id_pv = idesc_bf16(true);
    // descriptor words, built once: Q (K-major, per slot), K and V (per stage)
    const uint32_t d_hi = (uint32_t)(sw128_desc(sbase, 16, 1024) >> 32);
    const uint32_t q_lo = (uint32_t)sw128_desc(sbase + kSmQ, 16, 1024);
    const uint32_t k_lo = (uint32_t)sw128_desc(sbase + kSmK, 16, 1024);
    const uint32_t v_lo = (uint32_t)sw128_desc(sbase + kSmV, kHalfTileBytes, 1024);
    auto issue_s = [&](int s, int st) {
      const uint32_t a0 = q_lo + s * (kTileBytes >> 4), b0 = k_lo + st * (kTileBytes >> 4);
#pragma unroll
      for (int kk = 0; kk < kTcD / 16; ++kk) {
        const uint32_t off = ((kk / 4) * kHalfTileBytes + (kk % 4) * 32) >> 4;
        umma_ss_e(tS[s], a0 + off, b0 + off, d_hi, id_qk, kk > 0);
      }
    };
    auto issue_pv = [&](int s, int st, bool first_tile) {
      const uint32_t b0 = v_lo + st * (kTileBytes >> 4);
#pragma unroll
      for (int kk = 0; kk < kTcBN / 16; ++kk)
        umma_ts_e(tO[s], tS[s] + kk * 8, b0 + kk * (2048 >> 4), d_hi, id_pv, (!first_tile || kk > 0) ? 1u : 0u);
    };
    bool ok = true;
    if (P.inject_spins > 0) {
      // test hook: a wait that nothing ends
      bool got = false;
      if (lane == 0) {
        for (int64_t i = 0; i < P.inject_spins && !got; ++i) got = mbar_test(BAR(B_NEVER), 0);
        if (!got) {
          *abort_flag = 1;
          record_device_error(RCX_ERR_DEVICE_TIMEOUT);
        }
      }
      ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
    }
    int jg = 0, it = 0;
    for (int item = blockIdx.x; ok && item < P.n_items; item += gridDim.x, ++it) {
      const Item itm = decode_item(item, P);
      const int n = count_tiles(itm, a);
      if (!(ok = warp_wait(B_QREADY + 0, it & 1) && warp_wait(B_QREADY + 1, it & 1))) break;
      if (n == 0) {                        // nothing visible: the Q buffers are free at once
        umma_commit_e(BAR(B_QEMPTY));
        continue;
      }
      {
        const int st0 = jg % kTcStages;
        if (!(ok = warp_wait(B_KFULL + st0, (jg / kTcStages) & 1))) break;
        tc_fence_after();
        issue_s(0, st0);
        umma_commit_e(BAR(B_SFULL + 0));
        issue_s(1, st0);
        umma_commit_e(BAR(B_SFULL + 1));
        umma_commit_e(BAR(B_KEMPTY + st0));
        if (n == 1) umma_commit_e(BAR(B_QEMPTY));
      }
      for (int j = 0; ok && j < n; ++j) {
        const int g = jg + j;
        const int st = g % kTcStages;
        const uint32_t par = (g / kTcStages) & 1;
        const bool last = j == n - 1;
        const int st1 = (g + 1) % kTcStages;
        const uint32_t par1 = ((g + 1) / kTcStages) & 1;
        if (!(ok = warp_wait(B_VFULL + st, par))) break;
        if (!(ok = warp_wait(B_PREADY + 0, g & 1))) break;
        tc_fence_after();
        issue_pv(0, st, j == 0);
        if (last) umma_commit_e(BAR(B_OFINAL + 0));
        if (!last) {
          if (!(ok = warp_wait(B_KFULL + st1, par1))) break;
          tc_fence_after();
          issue_s(0, st1);
          umma_commit_e(BAR(B_SFULL + 0));
        }
        if (!(ok = warp_wait(B_PREADY + 1, g & 1))) break;
        tc_fence_after();
        issue_pv(1, st, j == 0);
        umma_commit_e(BAR(B_VEMPTY + st));
        if (last) umma_commit_e(BAR(B_OFINAL + 1));
        if (!last) {
          issue_s(1, st1);
          umma_commit_e(BAR(B_SFULL + 1));
          umma_commit_e(BAR(B_KEMPTY + st1));
          if (j + 1 == n - 1) umma_commit_e(BAR(B_QEMPTY));   // the item's last S MMAs are issued
        }
      }
      jg += n;
    }
    // all MMAs issued complete before TMEM is released
    umma_commit_e(BAR(B_DRAIN));
    if (lane == 0) mbar_wait(BAR(B_DRAIN), 0, abort_flag, 100000000ull, false);
    __syncwarp();
  } else {
    // ================================================================ softmax + epilogue
    const int s = warp / 4;                 // Q tile (slot) of this warpgroup
    const int q4 = warp % 4;                // TMEM lane quarter
    const int r = q4 * 32 + lane;           // row within the tile
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bool ok = true;
    int jg = 0, it = 0, on = 0;
    for (int item = blockIdx.x; ok && item < P.n_items; item += gridDim.x, ++it) {
      const Item itm = decode_item(item, P);
      const int n = count_tiles(itm, a);
      const int row = itm.row0[s] + r;                // local q row
      const int gi = (int)a.q_start + row;            // global token index
      const bool row_ok = row < (int)a.q.N;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(B_QFULL + s), it & 1, abort_flag) &&
                                             mbar_wait(BAR(B_BASE), it & 1, abort_flag))))
        break;
      // Rotate this row of the Q tile in shared memory (fused RoPE on Q).
      if ((a.rope_flags & RCX_ROTATE_Q) && row_ok) {
        uint8_t* qrow = smem + kSmQ + s * kTileBytes + r * 128;
        const float2* hi = rot_hi + (r >> 4) * 64;
        const float2* lo = rot_lo + (r & 15) * 64;
        const float2* bs = rot_base + s * 64;
        const int64_t m = a.positions ? a.positions[gi] : gi;
#pragma unroll 1
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* p = reinterpret_cast<uint4*>(qrow + kb * kHalfTileBytes + ((c ^ (r & 7)) * 16));
            uint4 u = *p;
            uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int pp = kb * 32 + c * 4 + e;
              float2 cs;
              if (table_rot) {
                cs = cs_mul(cs_mul(bs[pp], hi[pp]), lo[pp]);
              } else {
                rope_cos_sin(m, a.f.theta[pp], cs.x, cs.y);
              }
              const float2 x = bf2_to_f2(wv[e]);
              wv[e] = f2_to_bf2(x.x * cs.x - x.y * cs.y, x.x * cs.y + x.y * cs.x);
            }
            *p = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(BAR(B_QREADY + s));

      TileWalk w;
      tw_init(w, itm.gi_lo, itm.gi_hi, a);
      const int ti_lo = (int)a.q_start + itm.row0[s], ti_hi = ti_lo + kTcBM - 1;
      float m_used = -INFINITY, l = 0.f;
      int tile, j = 0;
      while (ok && tw_next(w, tile)) {
        const int g = jg + j;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(B_SFULL + s), g & 1, abort_flag)))) break;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(tS[s] + lane_off + 0, sr);
        tmem_ld32(tS[s] + lane_off + 32, sr + 32);
        tmem_ld32(tS[s] + lane_off + 64, sr + 64);
        tmem_ld32(tS[s] + lane_off + 96, sr + 96);
        tmem_wait_ld();
        const int j0 = (int)a.k_start + tile * kTcBN;
        const bool full = (j0 + kTcBN <= key_end) &&
                          tile_all_visible(ti_lo, ti_hi, j0, j0 + kTcBN - 1, a.window, a.n_sink);
        float mx = -INFINITY;
        if (full) {
          // row max in eight independent chains of three-input max
          float m8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) m8[u] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 128; c += 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              m8[u] = fmax3(m8[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
          }
          mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        } else {
          // The mask of this row over columns c of the tile, in 32-bit form:
          // c <= lim (causal and inside the keys) and (c > win_lo or c <= snk).
          auto clip = [](int x) { return x < -1 ? -1 : (x > kTcBN ? kTcBN : x); };
          const int lim = clip(min(gi, key_end - 1) - j0);
          const int win_lo = a.window > 0 ? clip(gi - (int)a.window - j0) : -1;
          const int snk = a.window > 0 ? clip((int)a.n_sink - 1 - j0) : -1;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool vis = c <= lim && (c > win_lo || c <= snk);
            if (!vis) sr[c] = __float_as_uint(-INFINITY);
            mx = fmaxf(mx, __uint_as_float(sr[c]));
          }
        }
        const float m_new = fmaxf(m_used, mx * a.scale_log2);
        const bool need = m_new > m_used + kLazyRescale;
        float alpha = 1.f;
        if (need) {
          alpha = fast_exp2(m_used - m_new);   // 0 when m_used = -inf
          m_used = m_new;
          l *= alpha;
        }
        const float mref = (m_used == -INFINITY) ? 0.f : m_used;
        // P to TMEM in four 16-column chunks as it is produced
        float sm2[2] = {0.f, 0.f};
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t pc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int col = blk * 32 + 2 * c;
            const float p0 = fast_exp2(fmaf(__uint_as_float(sr[col]), a.scale_log2, -mref));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sr[col + 1]), a.scale_log2, -mref));
            sm2[c & 1] += p0 + p1;
            pc[c] = f2_to_bf2(p0, p1);
          }
          tmem_st16(tS[s] + lane_off + blk * 16, pc);
        }
        l += sm2[0] + sm2[1];
        if (__any_sync(0xffffffffu, need && j > 0)) {
#pragma unroll 1
          for (int cb = 0; cb < 4; ++cb) {
            uint32_t o[32];
            tmem_ld32(tO[s] + lane_off + cb * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO[s] + lane_off + cb * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(B_PREADY + s));
        ++j;
      }
      if (!ok) break;

      // ---- epilogue: O / l (or its LSE merge with a previous partial) -> global, LSE
      if (n > 0) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(B_OFINAL + s), on & 1, abort_flag)))) break;
        tc_fence_after();
      }
      // O = ca * O_prev + cb * O_unnormalised: cb = 1 / l alone, or the LSE
      // merge with a previous partial over other keys (weights w = exp(lse -
      // max) of both partials).
      const float lse_b = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      float cb = l > 0.f ? 1.f / l : 0.f, ca = 0.f, lse_out = lse_b;
      const float* accp = nullptr;
      if (a.acc.ptr != nullptr && row_ok) {
        accp = reinterpret_cast<const float*>(a.acc.ptr) + itm.bb * a.acc.sb + row * a.acc.sn +
               itm.head[s] * a.acc.sh;
        const float lse_a = a.acc_lse[itm.bb * a.acc_lse_sb + itm.head[s] * a.acc_lse_sh + row];
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
      Tout* op = reinterpret_cast<Tout*>(a.o.ptr) + itm.bb * a.o.sb + row * a.o.sn + itm.head[s] * a.o.sh;
#pragma unroll 1
      for (int cbk = 0; cbk < 4; ++cbk) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld32(tO[s] + lane_off + cbk * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (row_ok) {
          float f[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(o[c]) * cb;
          if (accp) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 pv = *reinterpret_cast<const float4*>(accp + cbk * 32 + c);
              f[c] = fmaf(ca, pv.x, f[c]);
              f[c + 1] = fmaf(ca, pv.y, f[c + 1]);
              f[c + 2] = fmaf(ca, pv.z, f[c + 2]);
              f[c + 3] = fmaf(ca, pv.w, f[c + 3]);
            }
          }
          if constexpr (sizeof(Tout) == 2) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = f2_to_bf2(f[c + 0], f[c + 1]);
              v.y = f2_to_bf2(f[c + 2], f[c + 3]);
              v.z = f2_to_bf2(f[c + 4], f[c + 5]);
              v.w = f2_to_bf2(f[c + 6], f[c + 7]);
              *reinterpret_cast<uint4*>(op + cbk * 32 + c) = v;
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(op + cbk * 32 + c) = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
          }
        }
      }
      if (row_ok && a.lse) a.lse[itm.bb * a.lse_sb + itm.head[s] * a.lse_sh + row] = lse_out;
      jg += n;
      on += n > 0 ? 1 : 0;
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

}  // namespace rcx

// librcx.so: the C ABI declared in include/rcx.h.
//
// One translation unit: host-side argument checks, launch configuration, the
// Ring-Attention schedule and the host float64 frequency schedules; the
// kernels live in the *.cuh files included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <functional>
#include <mutex>
#include <vector>

#include "launch.h"
#include "common.cuh"
#include "rope_apply.cuh"
#include "merge.cuh"
#include "attn_common.cuh"
#include "attn_simt.cuh"
#include "attn_decode.cuh"
#include "kv_int8.cuh"
#include "rope_freqs.inc"

using namespace rcx;

namespace {

struct Stats {
  std::mutex mu;
  bool timing = false;
  int64_t launches[RCX_KERNEL_KINDS] = {0, 0, 0, 0, 0};
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> spans[RCX_KERNEL_KINDS];
  std::vector<cudaEvent_t> pool;

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};

Stats& stats() {
  static Stats* s = new Stats();   // kept until exit
  return *s;
}

}  // namespace

// ------------------------------------------------------------ launch accounting

namespace rcx {

LaunchScope::LaunchScope(int kind, cudaStream_t stream) : kind_(kind), stream_(stream) {
  Stats& st = stats();
  std::lock_guard<std::mutex> g(st.mu);
  ++st.launches[kind];
  if (st.timing) {
    start_ = st.take();
    stop_ = st.take();
    cudaEventRecord(start_, stream_);
  }
}

LaunchScope::~LaunchScope() {
  if (!start_) return;
  cudaEventRecord(stop_, stream_);
  Stats& st = stats();
  std::lock_guard<std::mutex> g(st.mu);
  st.spans[kind_].push_back({start_, stop_});
}

int sm_count() {
  // initialised once, thread-safely (every device this library targets is a B200)
  static const int n = [] {
    int dev = 0, c = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
      c = 148;
    return c;
  }();
  return n;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    std::fprintf(stderr, "librcx: launch failed: %s\n", cudaGetErrorString(e));
    return RCX_ERR_CUDA;
  }
  return RCX_OK;
}

}  // namespace rcx

namespace {

constexpr int kAbiVersion = 100;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int elem_size(int dtype) { return dtype == RCX_BF16 ? 2 : dtype == RCX_I8 ? 1 : 4; }

int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

bool shape_ok(const rcx_tensor& t) {
  for (int i = 0; i < 4; ++i)
    if (t.shape[i] < 0) return false;
  return t.dtype == RCX_F32 || t.dtype == RCX_BF16;
}

// [B, N, H, d] activation view: unit stride on d, non-negative strides.
int check_act(const rcx_tensor& t) {
  if (!shape_ok(t)) return RCX_ERR_INVALID_ARG;
  const bool empty = t.shape[0] == 0 || t.shape[1] == 0 || t.shape[2] == 0 || t.shape[3] == 0;
  if (!t.ptr && !empty) return RCX_ERR_INVALID_ARG;
  if (!t.ptr && t.shape[0] == 0 && t.shape[3] == 0) return RCX_ERR_INVALID_ARG;   // an all-zero (null) view
  if (t.stride[3] != 1 || t.stride[0] < 0 || t.stride[1] < 0 || t.stride[2] < 0) return RCX_ERR_INVALID_ARG;
  return RCX_OK;
}

// 16-byte vector access along d: base and token/head/batch strides aligned.
bool vec16_ok(const rcx_tensor& t) {
  const int es = elem_size(t.dtype);
  const int per = 16 / es;
  if (reinterpret_cast<uintptr_t>(t.ptr) % 16) return false;
  if (t.shape[3] % per) return false;
  for (int i = 0; i < 3; ++i)
    if (t.stride[i] % per) return false;
  return true;
}

// [B, H, N, 1] fp32 LSE view with unit stride on N.
int check_lse(const rcx_tensor& t, int64_t B, int64_t H, int64_t N) {
  if (!t.ptr && B * H * N != 0) return RCX_ERR_INVALID_ARG;
  if (t.dtype != RCX_F32) return RCX_ERR_INVALID_ARG;
  if (t.shape[0] != B || t.shape[1] != H || t.shape[2] != N) return RCX_ERR_INVALID_ARG;
  if (t.stride[2] != 1 || t.stride[0] < 0 || t.stride[1] < 0) return RCX_ERR_INVALID_ARG;
  return RCX_OK;
}


rcx_tensor null_tensor() {
  rcx_tensor t;
  std::memset(&t, 0, sizeof(t));
  return t;
}

// Sub-view of tokens [n0, n0 + n) of a [B, N, H, d] tensor.
rcx_tensor token_slice(const rcx_tensor& t, int64_t n0, int64_t n) {
  rcx_tensor s = t;
  s.ptr = static_cast<char*>(t.ptr) + n0 * t.stride[1] * elem_size(t.dtype);
  s.shape[1] = n;
  return s;
}

// Sub-view of tokens [n0, n0 + n) of a [B, H, N, 1] LSE tensor.
rcx_tensor lse_slice(const rcx_tensor& t, int64_t n0, int64_t n) {
  rcx_tensor s = t;
  s.ptr = static_cast<char*>(t.ptr) + n0 * 4;
  s.shape[2] = n;
  return s;
}

rcx_tensor make_tensor(void* p, int dtype, int64_t B, int64_t N, int64_t H, int64_t D) {
  rcx_tensor t;
  t.ptr = p;
  t.dtype = dtype;
  t.shape[0] = B; t.shape[1] = N; t.shape[2] = H; t.shape[3] = D;
  t.stride[3] = 1; t.stride[2] = D; t.stride[1] = H * D; t.stride[0] = N * H * D;
  return t;
}

rcx_tensor make_lse(void* p, int64_t B, int64_t H, int64_t N) {
  rcx_tensor t;
  t.ptr = p;
  t.dtype = RCX_F32;
  t.shape[0] = B; t.shape[1] = H; t.shape[2] = N; t.shape[3] = 1;
  t.stride[3] = 1; t.stride[2] = 1; t.stride[1] = N; t.stride[0] = H * N;
  return t;
}

// ------------------------------------------------------------------ rope_apply

int rope_apply_impl(const rcx_tensor& q, const rcx_tensor& k, const rcx_tensor& q_out,
                    const rcx_tensor& k_out, const int64_t* positions, int64_t n_positions,
                    const double* inv_freq, cudaStream_t stream) {
  if (!inv_freq) return RCX_ERR_INVALID_ARG;
  const bool has_q = q.ptr != nullptr, has_k = k.ptr != nullptr;
  if (!has_q && !has_k) return RCX_OK;
  const rcx_tensor& ref = has_q ? q : k;
  const int dtype = ref.dtype;
  const int64_t B = ref.shape[0], N = ref.shape[1], D = ref.shape[3];
  if (D < 2 || D > 2 * kMaxPairs || (D & 1)) return RCX_ERR_INVALID_ARG;
  const rcx_tensor* ins[2] = {&q, &k};
  const rcx_tensor* outs[2] = {&q_out, &k_out};
  for (int i = 0; i < 2; ++i) {
    if (!ins[i]->ptr) continue;
    int st = check_act(*ins[i]);
    if (st) return st;
    st = check_act(*outs[i]);
    if (st) return st;
    if (ins[i]->dtype != dtype || outs[i]->dtype != dtype) return RCX_ERR_INVALID_ARG;
    if (ins[i]->shape[0] != B || ins[i]->shape[1] != N || ins[i]->shape[3] != D) return RCX_ERR_INVALID_ARG;
    for (int j = 0; j < 4; ++j)
      if (outs[i]->shape[j] != ins[i]->shape[j]) return RCX_ERR_INVALID_ARG;
    if (!vec16_ok(*ins[i]) || !vec16_ok(*outs[i])) return RCX_ERR_ALIGNMENT;
  }
  if (positions && n_positions < N) return RCX_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return RCX_OK;
  RopeArgs a;
  std::memset(&a, 0, sizeof(a));
  if (has_q) { a.q_in = make_view(q); a.q_out = make_view(q_out); }
  if (has_k) { a.k_in = make_view(k); a.k_out = make_view(k_out); }
  a.positions = positions;
  a.n_tok = B * N;
  a.N = N;
  a.d_chunks = (int)(D * elem_size(dtype) / 16);    // vec16_ok: D * element size is a multiple of 16
  for (int i = 0; i < (int)(D / 2); ++i) a.f.theta[i] = inv_freq[i];
  const int tpb = kRopeThreads / a.d_chunks;          // d_chunks <= 2 * kMaxPairs * 4 / 16 = 64
  const int64_t passes = (a.n_tok + tpb - 1) / tpb;
  const int grid = (int)std::min<int64_t>(passes, (int64_t)sm_count() * kRopeCtasPerSm);
  return rope_apply_launch(a, dtype, grid, tpb * a.d_chunks, stream);
}

// ---------------------------------------------------------------------- merge

int merge_impl(const rcx_tensor& oa, const rcx_tensor& la, const rcx_tensor& ob, const rcx_tensor& lb,
               const rcx_tensor& oo_in, const rcx_tensor& lo_in, cudaStream_t stream) {
  const bool in_place = oo_in.ptr == nullptr;
  const rcx_tensor& oo = in_place ? oa : oo_in;
  const rcx_tensor& lo = in_place ? la : lo_in;
  int st;
  if ((st = check_act(oa)) || (st = check_act(ob)) || (st = check_act(oo))) return st;
  if (oa.dtype != RCX_F32 || ob.dtype != RCX_F32) return RCX_ERR_INVALID_ARG;
  const int64_t B = oa.shape[0], N = oa.shape[1], H = oa.shape[2], D = oa.shape[3];
  for (int j = 0; j < 4; ++j)
    if (ob.shape[j] != oa.shape[j] || oo.shape[j] != oa.shape[j]) return RCX_ERR_INVALID_ARG;
  if ((st = check_lse(la, B, H, N)) || (st = check_lse(lb, B, H, N)) || (st = check_lse(lo, B, H, N)))
    return st;
  if (D < 4 || D > 128 || (D & (D - 1))) return RCX_ERR_UNSUPPORTED;   // d/4 must divide 32
  if (!vec16_ok(oa) || !vec16_ok(ob)) return RCX_ERR_ALIGNMENT;
  if (oo.dtype == RCX_BF16 ? (reinterpret_cast<uintptr_t>(oo.ptr) % 8 || oo.stride[0] % 4 ||
                              oo.stride[1] % 4 || oo.stride[2] % 4)
                           : !vec16_ok(oo))
    return RCX_ERR_ALIGNMENT;
  if (B == 0 || N == 0 || H == 0) return RCX_OK;
  MergeArgs a;
  a.oa = make_view(oa); a.ob = make_view(ob); a.oo = make_view(oo);
  a.la = static_cast<float*>(la.ptr); a.lb = static_cast<const float*>(lb.ptr);
  a.lo = static_cast<float*>(lo.ptr);
  a.la_sb = la.stride[0]; a.la_sh = la.stride[1];
  a.lb_sb = lb.stride[0]; a.lb_sh = lb.stride[1];
  a.lo_sb = lo.stride[0]; a.lo_sh = lo.stride[1];
  a.rows = B * N * H;
  a.d4 = (int)(D / 4);
  const int64_t warps = B * N;     // one warp per token at a time
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, (int64_t)sm_count() * 8));
  return merge_launch(a, oo.dtype, grid, stream);
}

// ------------------------------------------------------------------ attention

// acc / acc_lse: optional previous partial result over other keys (fp32
// normalised O and its LSE), merged into this call's result in the epilogue;
// o / lse may alias them.  Null pointers: no previous partial.
int attn_impl(const rcx_tensor& q, const rcx_tensor& k, const rcx_tensor& v, const rcx_tensor& o,
              const rcx_tensor& lse, int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
              int64_t q_start, int64_t k_start, const int64_t* positions, int64_t n_positions,
              const double* inv_freq, int rope_flags, cudaStream_t stream, const rcx_tensor* acc = nullptr,
              const rcx_tensor* acc_lse = nullptr) {
  int st;
  if ((st = check_act(q)) || (st = check_act(k)) || (st = check_act(v)) || (st = check_act(o))) return st;
  const int64_t B = q.shape[0], Nq = q.shape[1], Hq = q.shape[2], D = q.shape[3];
  const int64_t Nk = k.shape[1], Hkv = k.shape[2];
  if (k.shape[0] != B || v.shape[0] != B || o.shape[0] != B) return RCX_ERR_INVALID_ARG;
  if (k.shape[3] != D || v.shape[3] != D || o.shape[3] != D) return RCX_ERR_INVALID_ARG;
  if (v.shape[1] != Nk || v.shape[2] != Hkv || o.shape[1] != Nq || o.shape[2] != Hq) return RCX_ERR_INVALID_ARG;
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv) return RCX_ERR_INVALID_ARG;
  if (q.dtype != k.dtype || q.dtype != v.dtype) return RCX_ERR_INVALID_ARG;
  if (lse.ptr && (st = check_lse(lse, B, Hq, Nq))) return st;
  if (kv_block < 0 || window < 0 || n_sink < 0 || q_start < 0 || k_start < 0) return RCX_ERR_INVALID_ARG;
  if (!(temperature > 0.0) || !std::isfinite(temperature)) return RCX_ERR_INVALID_ARG;
  if (rope_flags & ~(RCX_ROTATE_Q | RCX_ROTATE_K)) return RCX_ERR_INVALID_ARG;
  if (rope_flags && !inv_freq) return RCX_ERR_INVALID_ARG;
  if (rope_flags && positions && n_positions < std::max(q_start + Nq, k_start + Nk)) return RCX_ERR_INVALID_ARG;
  if (D < 2 || (D & 1)) return RCX_ERR_INVALID_ARG;
  const bool merging = acc != nullptr && acc->ptr != nullptr;
  if (merging) {
    if ((st = check_act(*acc))) return st;
    if (acc->dtype != RCX_F32) return RCX_ERR_INVALID_ARG;
    for (int j = 0; j < 4; ++j)
      if (acc->shape[j] != o.shape[j]) return RCX_ERR_INVALID_ARG;
    if (!acc_lse || (st = check_lse(*acc_lse, B, Hq, Nq))) return st ? st : RCX_ERR_INVALID_ARG;
    if (!vec16_ok(*acc)) return RCX_ERR_ALIGNMENT;
  }
  if (B == 0 || Nq == 0) return RCX_OK;

  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = make_view(q); a.k = make_view(k); a.v = make_view(v); a.o = make_view(o);
  a.lse = static_cast<float*>(lse.ptr);
  a.lse_sb = lse.ptr ? lse.stride[0] : 0;
  a.lse_sh = lse.ptr ? lse.stride[1] : 0;
  a.q_start = q_start; a.k_start = k_start;
  a.kv_block = kv_block > 0 ? kv_block : (k_start + Nk > 0 ? k_start + Nk : 1);
  a.window = window; a.n_sink = n_sink;
  a.scale_log2 = (float)(1.4426950408889634074 / (std::sqrt((double)D) * temperature));
  a.positions = positions;
  a.rope_flags = rope_flags;
  a.pairs = (int)(D / 2);
  a.G = (int)(Hq / Hkv);
  if (merging) {
    a.acc = make_view(*acc);
    a.acc_lse = static_cast<const float*>(acc_lse->ptr);
    a.acc_lse_sb = acc_lse->stride[0];
    a.acc_lse_sh = acc_lse->stride[1];
  }
  if (rope_flags) {
    if (a.pairs > kMaxPairs) return RCX_ERR_INVALID_ARG;
    for (int i = 0; i < a.pairs; ++i) a.f.theta[i] = inv_freq[i];
  }

  if (q.dtype == RCX_BF16 && D == 128) {
    if (rope_flags & RCX_ROTATE_K) return RCX_ERR_UNSUPPORTED;
    return attn_tc_launch(a, q, k, v, o, stream);
  }
  if (D != 32 && D != 64 && D != 128) return RCX_ERR_UNSUPPORTED;
  if (q.dtype == RCX_F32)
    return o.dtype == RCX_F32 ? attn_simt_launch_f32_f32(a, stream) : attn_simt_launch_f32_bf16(a, stream);
  return o.dtype == RCX_F32 ? attn_simt_launch_bf16_f32(a, stream) : attn_simt_launch_bf16_bf16(a, stream);
}

// --------------------------------------------------------------------- decode

struct DecodePlan {
  int splits;
  int64_t keys_per_split, off_lse, total;
};

DecodePlan decode_plan(const rcx_tensor& q, const rcx_tensor& k, int ctas_per_sm = 2) {
  DecodePlan p;
  const int64_t B = q.shape[0], Hq = q.shape[2], Nk = k.shape[1], Hkv = std::max<int64_t>(k.shape[2], 1);
  // at most one wave: splits x Hkv x B <= ctas_per_sm x SMs
  const int64_t want = std::max<int64_t>(1, (ctas_per_sm * (int64_t)sm_count()) / std::max<int64_t>(1, Hkv * B));
  const int64_t cap = std::max<int64_t>(1, (Nk + 127) / 128);
  p.splits = (int)std::min<int64_t>(std::min<int64_t>(want, cap), 4096);
  p.keys_per_split = std::max<int64_t>(1, (Nk + p.splits - 1) / p.splits);
  p.off_lse = align256((int64_t)p.splits * B * Hq * 128 * 4);
  p.total = align256(p.off_lse + (int64_t)p.splits * B * Hq * 4);
  return p;
}

int decode_impl(const rcx_tensor& q, const rcx_tensor& k, const rcx_tensor& v, const rcx_tensor& o,
                const rcx_tensor& lse, int64_t window, int64_t n_sink, double temperature, int64_t q_index,
                const int64_t* positions, int64_t n_positions, const double* inv_freq, int rope_flags,
                void* workspace, int64_t workspace_bytes, cudaStream_t stream) {
  int st;
  if ((st = check_act(q)) || (st = check_act(k)) || (st = check_act(v)) || (st = check_act(o))) return st;
  const int64_t B = q.shape[0], Hq = q.shape[2], D = q.shape[3], Nk = k.shape[1], Hkv = k.shape[2];
  if (q.shape[1] != 1 || o.shape[1] != 1) return RCX_ERR_INVALID_ARG;
  if (q.dtype != RCX_BF16 || k.dtype != RCX_BF16 || v.dtype != RCX_BF16) return RCX_ERR_UNSUPPORTED;
  if (D != 128 || k.shape[3] != 128 || v.shape[3] != 128 || o.shape[3] != 128) return RCX_ERR_UNSUPPORTED;
  if (k.shape[0] != B || v.shape[0] != B || o.shape[0] != B || v.shape[1] != Nk || v.shape[2] != Hkv ||
      o.shape[2] != Hq)
    return RCX_ERR_INVALID_ARG;
  if (Hkv <= 0 || Hq % Hkv) return RCX_ERR_INVALID_ARG;
  const int64_t G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return RCX_ERR_UNSUPPORTED;
  if (lse.ptr && (st = check_lse(lse, B, Hq, 1))) return st;
  if (window < 0 || n_sink < 0 || q_index < 0) return RCX_ERR_INVALID_ARG;
  if (!(temperature > 0.0) || !std::isfinite(temperature)) return RCX_ERR_INVALID_ARG;
  if (rope_flags & ~RCX_ROTATE_Q) return rope_flags & RCX_ROTATE_K ? RCX_ERR_UNSUPPORTED : RCX_ERR_INVALID_ARG;
  if (rope_flags && !inv_freq) return RCX_ERR_INVALID_ARG;
  if (positions && n_positions <= std::max(q_index, Nk - 1)) return RCX_ERR_INVALID_ARG;
  // 8-byte row accesses for q, k, v; 16 (fp32) or 8 (bf16) for o
  auto al = [](const rcx_tensor& t, int bytes) {
    const int per = bytes / elem_size(t.dtype);
    return reinterpret_cast<uintptr_t>(t.ptr) % bytes == 0 && t.stride[0] % per == 0 && t.stride[1] % per == 0 &&
           t.stride[2] % per == 0;
  };
  if (!al(q, 8) || !al(k, 8) || !al(v, 8) || !al(o, o.dtype == RCX_BF16 ? 8 : 16)) return RCX_ERR_ALIGNMENT;
  if (B == 0 || Hq == 0) return RCX_OK;
  if (B > 65535 || Hkv > 65535) return RCX_ERR_UNSUPPORTED;
  const DecodePlan p = decode_plan(q, k);
  if (!workspace || workspace_bytes < p.total) return RCX_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return RCX_ERR_ALIGNMENT;
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = make_view(q); a.k = make_view(k); a.v = make_view(v); a.o = make_view(o);
  a.lse = static_cast<float*>(lse.ptr);
  a.lse_sb = lse.ptr ? lse.stride[0] : 0;
  a.lse_sh = lse.ptr ? lse.stride[1] : 0;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.off_lse);
  a.splits = p.splits;
  a.keys_per_split = p.keys_per_split;
  a.q_index = q_index;
  a.window = window; a.n_sink = n_sink;
  a.scale_log2 = (float)(1.4426950408889634074 / (std::sqrt((double)D) * temperature));
  a.positions = positions;
  a.rope_q = rope_flags & RCX_ROTATE_Q;
  a.G = (int)G;
  if (a.rope_q)
    for (int i = 0; i < 64; ++i) a.f.theta[i] = inv_freq[i];
  {
    dim3 grid((unsigned)p.splits, (unsigned)Hkv, (unsigned)B);
    if ((st = decode_launch(a, (int)G, al(k, 16) && al(v, 16), grid, stream))) return st;
  }
  const int grid2 = (int)std::max<int64_t>(1, std::min<int64_t>(B * Hq, (int64_t)sm_count() * 8));   // a CTA per row
  return decode_combine_launch(a, o.dtype, grid2, stream);
}

// ------------------------------------------------------------ int8 KV cache

// [B, N, H, d] int8 view: unit stride on d, non-negative strides.
int check_i8(const rcx_tensor& t) {
  for (int i = 0; i < 4; ++i)
    if (t.shape[i] < 0) return RCX_ERR_INVALID_ARG;
  if (t.dtype != RCX_I8) return RCX_ERR_INVALID_ARG;
  const bool empty = t.shape[0] == 0 || t.shape[1] == 0 || t.shape[2] == 0 || t.shape[3] == 0;
  if (!t.ptr && !empty) return RCX_ERR_INVALID_ARG;
  if (t.stride[3] != 1 || t.stride[0] < 0 || t.stride[1] < 0 || t.stride[2] < 0) return RCX_ERR_INVALID_ARG;
  return RCX_OK;
}

bool aligned_rows(const rcx_tensor& t, int bytes) {
  const int per = bytes / elem_size(t.dtype);
  return reinterpret_cast<uintptr_t>(t.ptr) % bytes == 0 && t.stride[0] % per == 0 && t.stride[1] % per == 0 &&
         t.stride[2] % per == 0;
}

int quantize_i8_impl(const rcx_tensor& x, const rcx_tensor& c, float* scale, cudaStream_t stream) {
  int st;
  if ((st = check_act(x)) || (st = check_i8(c))) return st;
  if (x.dtype != RCX_BF16) return RCX_ERR_UNSUPPORTED;
  if (x.shape[3] != 128) return RCX_ERR_UNSUPPORTED;
  for (int i = 0; i < 4; ++i)
    if (c.shape[i] != x.shape[i]) return RCX_ERR_INVALID_ARG;
  const int64_t rows = x.shape[0] * x.shape[1] * x.shape[2];
  if (rows == 0) return RCX_OK;
  if (!scale) return RCX_ERR_INVALID_ARG;
  if (!aligned_rows(x, 8) || !aligned_rows(c, 4) || reinterpret_cast<uintptr_t>(scale) % 4) return RCX_ERR_ALIGNMENT;
  QuantArgs a;
  std::memset(&a, 0, sizeof(a));
  a.x = make_view(x);
  a.c = make_view(c);
  a.scale = scale;
  a.rows = rows;
  a.fast = rows < (int64_t(1) << 31);
  if (a.fast) {
    a.div_h = make_fastdiv((uint32_t)x.shape[2]);
    a.div_n = make_fastdiv((uint32_t)x.shape[1]);
  }
  const bool rows16 = aligned_rows(x, 16) && aligned_rows(c, 16);
  const int64_t per_cta = rows16 ? 32 : 8;      // rows a CTA covers per pass (four or one per warp)
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((rows + per_cta - 1) / per_cta,
                                                              (int64_t)sm_count() * 8));
  return quantize_i8_launch(a, rows16, grid, stream);
}

int decode_i8_impl(const rcx_tensor& q, const rcx_tensor& k, const float* k_scale, const rcx_tensor& v,
                   const float* v_scale, const rcx_tensor& o, const rcx_tensor& lse, int64_t window, int64_t n_sink,
                   double temperature, int64_t q_index, const int64_t* positions, int64_t n_positions,
                   const double* inv_freq, int rope_flags, void* workspace, int64_t workspace_bytes,
                   cudaStream_t stream) {
  int st;
  if ((st = check_act(q)) || (st = check_i8(k)) || (st = check_i8(v)) || (st = check_act(o))) return st;
  const int64_t B = q.shape[0], Hq = q.shape[2], D = q.shape[3], Nk = k.shape[1], Hkv = k.shape[2];
  if (q.shape[1] != 1 || o.shape[1] != 1) return RCX_ERR_INVALID_ARG;
  if (q.dtype != RCX_BF16) return RCX_ERR_UNSUPPORTED;
  if (D != 128 || k.shape[3] != 128 || v.shape[3] != 128 || o.shape[3] != 128) return RCX_ERR_UNSUPPORTED;
  if (k.shape[0] != B || v.shape[0] != B || o.shape[0] != B || v.shape[1] != Nk || v.shape[2] != Hkv ||
      o.shape[2] != Hq)
    return RCX_ERR_INVALID_ARG;
  if (Hkv <= 0 || Hq % Hkv) return RCX_ERR_INVALID_ARG;
  const int64_t G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return RCX_ERR_UNSUPPORTED;
  if (lse.ptr && (st = check_lse(lse, B, Hq, 1))) return st;
  if (window < 0 || n_sink < 0 || q_index < 0) return RCX_ERR_INVALID_ARG;
  if (!(temperature > 0.0) || !std::isfinite(temperature)) return RCX_ERR_INVALID_ARG;
  if (rope_flags & ~RCX_ROTATE_Q) return rope_flags & RCX_ROTATE_K ? RCX_ERR_UNSUPPORTED : RCX_ERR_INVALID_ARG;
  if (rope_flags && !inv_freq) return RCX_ERR_INVALID_ARG;
  if (positions && n_positions <= std::max(q_index, Nk - 1)) return RCX_ERR_INVALID_ARG;
  if (Nk > 0 && B > 0 && (!k_scale || !v_scale)) return RCX_ERR_INVALID_ARG;
  // 16-byte code rows (cp.async), 8-byte q rows, 4-byte scales
  if (!aligned_rows(q, 8) || !aligned_rows(k, 16) || !aligned_rows(v, 16) ||
      !aligned_rows(o, o.dtype == RCX_BF16 ? 8 : 16))
    return RCX_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(k_scale) % 4 || reinterpret_cast<uintptr_t>(v_scale) % 4) return RCX_ERR_ALIGNMENT;
  if (B == 0 || Hq == 0) return RCX_OK;
  if (B > 65535 || Hkv > 65535) return RCX_ERR_UNSUPPORTED;
  const DecodePlan p = decode_plan(q, k, kDqCtasPerSm);
  if (!workspace || workspace_bytes < p.total) return RCX_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return RCX_ERR_ALIGNMENT;
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = make_view(q); a.k = make_view(k); a.v = make_view(v); a.o = make_view(o);
  a.lse = static_cast<float*>(lse.ptr);
  a.lse_sb = lse.ptr ? lse.stride[0] : 0;
  a.lse_sh = lse.ptr ? lse.stride[1] : 0;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.off_lse);
  a.splits = p.splits;
  a.keys_per_split = p.keys_per_split;
  a.q_index = q_index;
  a.window = window; a.n_sink = n_sink;
  a.scale_log2 = (float)(1.4426950408889634074 / (std::sqrt((double)D) * temperature));
  a.positions = positions;
  a.rope_q = rope_flags & RCX_ROTATE_Q;
  a.G = (int)G;
  if (a.rope_q)
    for (int i = 0; i < 64; ++i) a.f.theta[i] = inv_freq[i];
  {
    dim3 grid((unsigned)p.splits, (unsigned)Hkv, (unsigned)B);
    if ((st = decode_i8_launch(a, (int)G, k_scale, v_scale, grid, stream))) return st;
  }
  const int grid2 = (int)std::max<int64_t>(1, std::min<int64_t>(B * Hq, (int64_t)sm_count() * 8));   // a CTA per row
  return decode_combine_launch(a, o.dtype, grid2, stream);
}

// -------------------------------------------------------------- device status

// Reads and clears the status words of every kernel family with bounded
// waits (synchronising `s`); the tensor-core attention's word wins if both are set.
int device_status_all(cudaStream_t s, int* out) {
  int a = 0, b = 0, st;
  if ((st = status_exchange_attn_tc(s, &a))) return st;
  if ((st = status_exchange_rope(s, &b))) return st;
  *out = a != 0 ? a : b;
  return RCX_OK;
}

// ----------------------------------------------------------------------- ring

struct RingPlan {
  int64_t B, N, Hq, Hkv, D, kv, P;
  bool rotate_k_separately;
  int64_t off_acc, off_lacc, off_krot, total;
};

RingPlan ring_plan(const rcx_tensor& q, const rcx_tensor& k, int64_t kv_block, int rope_flags) {
  RingPlan p;
  p.B = q.shape[0]; p.N = q.shape[1]; p.Hq = q.shape[2]; p.D = q.shape[3]; p.Hkv = k.shape[2];
  p.kv = kv_block > 0 ? std::min(kv_block, std::max<int64_t>(p.N, 1)) : std::max<int64_t>(p.N, 1);
  p.P = (p.N + p.kv - 1) / p.kv;
  p.rotate_k_separately = (rope_flags & RCX_ROTATE_K) && q.dtype == RCX_BF16 && p.D == 128;
  int64_t off = 0;
  p.off_acc = off;   off = align256(off + p.B * p.N * p.Hq * p.D * 4);
  p.off_lacc = off;  off = align256(off + p.B * p.Hq * p.N * 4);
  p.off_krot = off;
  if (p.rotate_k_separately) off = align256(off + p.B * p.N * p.Hkv * p.D * 2);
  p.total = off;
  return p;
}

// Points where a caller that streams the inputs in and the outputs out (the
// host-buffer entry point) joins the ring schedule on its stream: before the
// first kernel that reads K, before the launch of query shard r against key
// block b, and after the launch that writes shard r's final output.
struct RingHooks {
  std::function<int()> before_k;
  std::function<int(int64_t r, int64_t b)> before_launch;
  std::function<int(int64_t r)> after_final;
};

int ring_impl(const rcx_tensor& q, const rcx_tensor& k, const rcx_tensor& v, const rcx_tensor& o,
              const rcx_tensor& lse, int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
              const int64_t* positions, int64_t n_positions, const double* inv_freq, int rope_flags,
              void* workspace, int64_t workspace_bytes, cudaStream_t stream, const RingHooks* hooks = nullptr) {
  int st;
  if ((st = check_act(q)) || (st = check_act(k)) || (st = check_act(v)) || (st = check_act(o))) return st;
  if (k.shape[1] != q.shape[1]) return RCX_ERR_INVALID_ARG;     // self-attention over one sequence
  if (kv_block < 0) return RCX_ERR_INVALID_ARG;
  RingPlan p = ring_plan(q, k, kv_block, rope_flags);
  if (p.B == 0 || p.N == 0) return RCX_OK;
  if (!workspace || workspace_bytes < p.total) return RCX_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return RCX_ERR_ALIGNMENT;
  char* ws = static_cast<char*>(workspace);
  rcx_tensor acc = make_tensor(ws + p.off_acc, RCX_F32, p.B, p.N, p.Hq, p.D);
  rcx_tensor lacc = make_lse(ws + p.off_lacc, p.B, p.Hq, p.N);

  rcx_tensor kk = k;
  int flags = rope_flags;
  if (hooks && (st = hooks->before_k())) return st;
  if (p.rotate_k_separately) {
    // K is shared by G query heads and by every query tile: rotate it once.
    rcx_tensor krot = make_tensor(ws + p.off_krot, RCX_BF16, p.B, p.N, p.Hkv, p.D);
    if ((st = rope_apply_impl(null_tensor(), k, null_tensor(), krot, positions, n_positions, inv_freq, stream)))
      return st;
    kk = krot;
    flags &= ~RCX_ROTATE_K;
  }

  // Per shard: which ring steps carry visible keys (first and last).
  std::vector<int64_t> first(p.P, -1), last(p.P, -1), count(p.P, 0);
  for (int64_t t = 0; t < p.P; ++t)
    for (int64_t r = 0; r < p.P; ++r) {
      const int64_t b = ((r - t) % p.P + p.P) % p.P;
      const int64_t i0 = r * p.kv, i1 = std::min((r + 1) * p.kv, p.N) - 1;
      const int64_t j0 = b * p.kv, j1 = std::min((b + 1) * p.kv, p.N) - 1;
      if (!tile_any_visible(i0, i1, j0, j1, window, n_sink)) continue;
      if (first[r] < 0) first[r] = t;
      last[r] = t;
      ++count[r];
    }

  for (int64_t t = 0; t < p.P; ++t) {
    for (int64_t r = 0; r < p.P; ++r) {
      const int64_t b = ((r - t) % p.P + p.P) % p.P;
      const int64_t i0 = r * p.kv, ni = std::min((r + 1) * p.kv, p.N) - i0;
      const int64_t j0 = b * p.kv, nj = std::min((b + 1) * p.kv, p.N) - j0;
      if (!tile_any_visible(i0, i0 + ni - 1, j0, j0 + nj - 1, window, n_sink)) continue;
      rcx_tensor qs = token_slice(q, i0, ni);
      rcx_tensor ks = token_slice(kk, j0, nj);
      rcx_tensor vs = token_slice(v, j0, nj);
      rcx_tensor os_final = token_slice(o, i0, ni);
      rcx_tensor ls_final = lse.ptr ? lse_slice(lse, i0, ni) : null_tensor();
      if (hooks && (st = hooks->before_launch(r, b))) return st;
      if (count[r] == 1) {          // one visible block: write the result directly
        st = attn_impl(qs, ks, vs, os_final, ls_final, 0, window, n_sink, temperature, i0, j0, positions,
                       n_positions, inv_freq, flags, stream);
        if (st) return st;
        if (hooks && (st = hooks->after_final(r))) return st;
        continue;
      }
      rcx_tensor as = token_slice(acc, i0, ni);
      rcx_tensor las = lse_slice(lacc, i0, ni);
      if (t == first[r]) {          // first visible block: the fp32 accumulator
        st = attn_impl(qs, ks, vs, as, las, 0, window, n_sink, temperature, i0, j0, positions, n_positions,
                       inv_freq, flags, stream);
      } else if (t == last[r]) {    // last: merged with the accumulator into the final output
        rcx_tensor lo = lse.ptr ? ls_final : las;
        st = attn_impl(qs, ks, vs, os_final, lo, 0, window, n_sink, temperature, i0, j0, positions, n_positions,
                       inv_freq, flags, stream, &as, &las);
      } else {                      // merged into the accumulator in place
        st = attn_impl(qs, ks, vs, as, las, 0, window, n_sink, temperature, i0, j0, positions, n_positions,
                       inv_freq, flags, stream, &as, &las);
      }
      if (st) return st;
      if (hooks && t == last[r] && (st = hooks->after_final(r))) return st;
    }
  }
  return RCX_OK;
}

}  // namespace

namespace {

// Staging memory of rcx_ring_attn_fwd_host: one pool per device that keeps
// what it has mapped (release threshold: all), so that a repeated call reuses
// the ~73 GB of a 1M-token call instead of mapping it again; handed back by
// rcx_release_staging.
constexpr int kMaxDevices = 64;
std::mutex g_staging_mu;
cudaMemPool_t g_staging[kMaxDevices] = {};

cudaError_t staging_pool(int dev, bool fresh, cudaMemPool_t* out) {
  std::lock_guard<std::mutex> lock(g_staging_mu);
  if (fresh) g_staging[dev] = nullptr;          // a handle that stopped working (context re-created)
  if (!g_staging[dev]) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = UINT64_MAX;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    g_staging[dev] = pool;
  }
  *out = g_staging[dev];
  return cudaSuccess;
}

cudaError_t staging_alloc(void** p, size_t bytes, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaMallocAsync(p, bytes, s);
  for (int attempt = 0; attempt < 2; ++attempt) {
    cudaMemPool_t pool = nullptr;
    if ((e = staging_pool(dev, attempt > 0, &pool)) != cudaSuccess) return e;
    if ((e = cudaMallocFromPoolAsync(p, bytes, pool, s)) == cudaSuccess) return e;
    if (e == cudaErrorMemoryAllocation) return e;
    cudaGetLastError();                         // clear, and retry once with a new pool
  }
  return e;
}

// Copy streams and events of rcx_ring_attn_fwd_host; released by the
// destructor (after the call has synchronised them).
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  std::vector<cudaEvent_t> events;
  bool ok = true;
  cudaEvent_t event() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      ok = false;
      return nullptr;
    }
    events.push_back(e);
    return e;
  }
  ~HostPipe() {
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
  }
};

}  // namespace

// =============================================================== C entry points

extern "C" {

int rcx_abi_version(void) { return kAbiVersion; }

const char* rcx_status_string(int status) {
  switch (status) {
    case RCX_OK: return "ok";
    case RCX_ERR_INVALID_ARG: return "invalid argument";
    case RCX_ERR_UNSUPPORTED: return "unsupported configuration";
    case RCX_ERR_ALIGNMENT: return "misaligned pointer or stride";
    case RCX_ERR_CUDA: return "CUDA error";
    case RCX_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int rcx_rope_freqs(int scheme, double base, int d, int64_t L_train, int64_t L_target, double alpha,
                   double beta, double* inv_freq_out, double* temperature_out) {
  return rope_freqs_host(scheme, base, d, L_train, L_target, alpha, beta, inv_freq_out, temperature_out);
}

int rcx_rope_freqs_per_pair(double base, int d, const double* factors, double* inv_freq_out) {
  return rope_freqs_per_pair_host(base, d, factors, inv_freq_out);
}

int rcx_rope_apply(rcx_tensor q, rcx_tensor k, rcx_tensor q_out, rcx_tensor k_out, const int64_t* positions,
                   int64_t n_positions, const double* inv_freq, void* stream) {
  return rope_apply_impl(q, k, q_out, k_out, positions, n_positions, inv_freq, as_stream(stream));
}

int rcx_attn_blockwise_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                           int64_t kv_block, int64_t window, int64_t n_sink, double temperature, int64_t q_start,
                           int64_t k_start, const int64_t* positions, int64_t n_positions,
                           const double* inv_freq, int rope_flags, void* stream) {
  return attn_impl(q, k, v, o, lse, kv_block, window, n_sink, temperature, q_start, k_start, positions,
                   n_positions, inv_freq, rope_flags, as_stream(stream));
}

int rcx_attn_blockwise_merge_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                                 rcx_tensor acc, rcx_tensor acc_lse, int64_t kv_block, int64_t window,
                                 int64_t n_sink, double temperature, int64_t q_start, int64_t k_start,
                                 const int64_t* positions, int64_t n_positions, const double* inv_freq,
                                 int rope_flags, void* stream) {
  const bool empty = q.shape[0] == 0 || q.shape[1] == 0 || q.shape[2] == 0 || q.shape[3] == 0;
  if (!acc.ptr && !empty) return RCX_ERR_INVALID_ARG;
  return attn_impl(q, k, v, o, lse, kv_block, window, n_sink, temperature, q_start, k_start, positions,
                   n_positions, inv_freq, rope_flags, as_stream(stream), &acc, &acc_lse);
}

int64_t rcx_attn_decode_workspace_size(rcx_tensor q, rcx_tensor k) {
  if (check_act(q) || check_act(k)) return -1;
  return decode_plan(q, k).total;
}

int rcx_attn_decode_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse, int64_t window,
                        int64_t n_sink, double temperature, int64_t q_index, const int64_t* positions,
                        int64_t n_positions, const double* inv_freq, int rope_flags, void* workspace,
                        int64_t workspace_bytes, void* stream) {
  return decode_impl(q, k, v, o, lse, window, n_sink, temperature, q_index, positions, n_positions, inv_freq,
                     rope_flags, workspace, workspace_bytes, as_stream(stream));
}

int rcx_kv_quantize_int8(rcx_tensor x, rcx_tensor codes, float* scale, void* stream) {
  return quantize_i8_impl(x, codes, scale, as_stream(stream));
}

int64_t rcx_attn_decode_int8_workspace_size(rcx_tensor q, rcx_tensor k) {
  if (check_act(q) || check_i8(k)) return -1;
  return decode_plan(q, k, kDqCtasPerSm).total;
}

int rcx_attn_decode_int8_fwd(rcx_tensor q, rcx_tensor k, const float* k_scale, rcx_tensor v, const float* v_scale,
                             rcx_tensor o, rcx_tensor lse, int64_t window, int64_t n_sink, double temperature,
                             int64_t q_index, const int64_t* positions, int64_t n_positions, const double* inv_freq,
                             int rope_flags, void* workspace, int64_t workspace_bytes, void* stream) {
  return decode_i8_impl(q, k, k_scale, v, v_scale, o, lse, window, n_sink, temperature, q_index, positions,
                        n_positions, inv_freq, rope_flags, workspace, workspace_bytes, as_stream(stream));
}

int rcx_merge_partials(rcx_tensor o_a, rcx_tensor lse_a, rcx_tensor o_b, rcx_tensor lse_b, rcx_tensor o_out,
                       rcx_tensor lse_out, void* stream) {
  return merge_impl(o_a, lse_a, o_b, lse_b, o_out, lse_out, as_stream(stream));
}

int64_t rcx_ring_workspace_size(rcx_tensor q, rcx_tensor k, int64_t kv_block, int rope_flags) {
  if (check_act(q) || check_act(k) || kv_block < 0) return -1;
  return ring_plan(q, k, kv_block, rope_flags).total;
}

int rcx_ring_attn_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse, int64_t kv_block,
                      int64_t window, int64_t n_sink, double temperature, const int64_t* positions,
                      int64_t n_positions, const double* inv_freq, int rope_flags, void* workspace,
                      int64_t workspace_bytes, void* stream) {
  return ring_impl(q, k, v, o, lse, kv_block, window, n_sink, temperature, positions, n_positions, inv_freq,
                   rope_flags, workspace, workspace_bytes, as_stream(stream));
}

int rcx_ring_attn_fwd_host(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                           int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
                           const int64_t* positions, int64_t n_positions, const double* inv_freq, int rope_flags,
                           void* stream) {
  // Host buffers must be dense [B, N, H, d] / [B, H, N, 1].
  const rcx_tensor* hs[4] = {&q, &k, &v, &o};
  for (int i = 0; i < 4; ++i) {
    const rcx_tensor& t = *hs[i];
    if (!t.ptr || !shape_ok(t)) return RCX_ERR_INVALID_ARG;
    if (t.stride[3] != 1 || t.stride[2] != t.shape[3] || t.stride[1] != t.shape[2] * t.shape[3] ||
        t.stride[0] != t.shape[1] * t.stride[1])
      return RCX_ERR_INVALID_ARG;
  }
  if (k.shape[1] != q.shape[1] || v.shape[1] != q.shape[1] || o.shape[1] != q.shape[1] || kv_block < 0)
    return RCX_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  auto bytes = [](const rcx_tensor& t) {
    return t.shape[0] * t.shape[1] * t.shape[2] * t.shape[3] * (int64_t)elem_size(t.dtype);
  };
  const int64_t lse_bytes = lse.ptr ? lse.shape[0] * lse.shape[1] * lse.shape[2] * 4 : 0;
  const int64_t ws_bytes = rcx_ring_workspace_size(q, k, kv_block, rope_flags);
  if (ws_bytes < 0) return RCX_ERR_INVALID_ARG;
  const int64_t pos_bytes = positions ? n_positions * 8 : 0;
  const int64_t sizes[7] = {bytes(q), bytes(k), bytes(v), bytes(o), lse_bytes, ws_bytes, pos_bytes};
  int64_t offs[7], total = 0;
  for (int i = 0; i < 7; ++i) { offs[i] = total; total = align256(total + sizes[i]); }
  const RingPlan plan = ring_plan(q, k, kv_block, rope_flags);
  const int64_t P = std::max<int64_t>(plan.P, 1);

  // The copies run on two streams of their own and meet the schedule on `s`
  // through events: K and the positions first (the K rotation reads all of
  // K), then shard r's query rows with block r's V rows in ring order, so the
  // launches of shard r wait only for what they read; each shard's final
  // output goes back as soon as its last launch is done.
  HostPipe hp;
  char* dev = nullptr;
  int st = RCX_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && st == RCX_OK) st = RCX_ERR_CUDA;
    return st == RCX_OK;
  };
  if (!ck(cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking)) ||
      !ck(cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking)))
    return st;
  if (staging_alloc(reinterpret_cast<void**>(&dev), (size_t)std::max<int64_t>(total, 256), s) != cudaSuccess)
    return RCX_ERR_CUDA;
  rcx_tensor dq = q, dk = k, dv = v, dout = o, dl = lse;
  dq.ptr = dev + offs[0]; dk.ptr = dev + offs[1]; dv.ptr = dev + offs[2]; dout.ptr = dev + offs[3];
  if (lse.ptr) dl.ptr = dev + offs[4];
  int64_t* dpos = positions ? reinterpret_cast<int64_t*>(dev + offs[6]) : nullptr;

  // rows [r kv, min((r + 1) kv, N)) of every batch entry of a dense [B, N, H, d] tensor
  auto copy_rows = [&](void* dst, const void* src, const rcx_tensor& t, int64_t r, cudaMemcpyKind kind,
                       cudaStream_t cs) {
    const int64_t row_bytes = t.shape[2] * t.shape[3] * elem_size(t.dtype);
    const int64_t i0 = r * plan.kv, ni = std::min((r + 1) * plan.kv, t.shape[1]) - i0;
    for (int64_t b = 0; b < t.shape[0] && st == RCX_OK && ni > 0; ++b) {
      const int64_t off = (b * t.shape[1] + i0) * row_bytes;
      ck(cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off, ni * row_bytes, kind,
                         cs));
    }
  };
  cudaEvent_t ev_alloc = hp.event(), ev_k = hp.event();
  std::vector<cudaEvent_t> ev_in(P);
  for (int64_t r = 0; r < P; ++r) ev_in[r] = hp.event();
  if (!hp.ok) st = RCX_ERR_CUDA;
  if (ck(cudaEventRecord(ev_alloc, s)) && ck(cudaStreamWaitEvent(hp.in, ev_alloc, 0)) &&
      ck(cudaStreamWaitEvent(hp.out, ev_alloc, 0)) &&
      ck(cudaMemcpyAsync(dk.ptr, k.ptr, sizes[1], cudaMemcpyHostToDevice, hp.in)) &&
      (!dpos || ck(cudaMemcpyAsync(dpos, positions, pos_bytes, cudaMemcpyHostToDevice, hp.in))) &&
      ck(cudaEventRecord(ev_k, hp.in))) {
    for (int64_t r = 0; r < P && st == RCX_OK; ++r) {
      copy_rows(dq.ptr, q.ptr, q, r, cudaMemcpyHostToDevice, hp.in);
      copy_rows(dv.ptr, v.ptr, v, r, cudaMemcpyHostToDevice, hp.in);
      ck(cudaEventRecord(ev_in[r], hp.in));
    }
  }

  std::vector<char> handed(P, 0);
  int64_t waited = -1;
  RingHooks hooks;
  hooks.before_k = [&]() -> int {
    return cudaStreamWaitEvent(s, ev_k, 0) == cudaSuccess ? RCX_OK : RCX_ERR_CUDA;
  };
  hooks.before_launch = [&](int64_t r, int64_t b) -> int {
    const int64_t m = std::max(r, b);
    if (m > waited) {
      if (cudaStreamWaitEvent(s, ev_in[m], 0) != cudaSuccess) return RCX_ERR_CUDA;
      waited = m;
    }
    return RCX_OK;
  };
  hooks.after_final = [&](int64_t r) -> int {
    cudaEvent_t e = hp.event();
    if (!e || cudaEventRecord(e, s) != cudaSuccess || cudaStreamWaitEvent(hp.out, e, 0) != cudaSuccess)
      return RCX_ERR_CUDA;
    copy_rows(o.ptr, dout.ptr, o, r, cudaMemcpyDeviceToHost, hp.out);
    handed[r] = 1;
    return st;
  };
  if (st == RCX_OK)
    st = ring_impl(dq, dk, dv, dout, dl, kv_block, window, n_sink, temperature, dpos, n_positions, inv_freq,
                   rope_flags, dev + offs[5], ws_bytes, s, &hooks);
  // after the schedule: the LSE and any output not handed out yet
  if (st == RCX_OK) {
    cudaEvent_t e_end = hp.event();
    if (ck(e_end ? cudaEventRecord(e_end, s) : cudaErrorUnknown) && ck(cudaStreamWaitEvent(hp.out, e_end, 0))) {
      for (int64_t r = 0; r < P && st == RCX_OK; ++r)
        if (!handed[r]) copy_rows(o.ptr, dout.ptr, o, r, cudaMemcpyDeviceToHost, hp.out);
      if (lse.ptr) ck(cudaMemcpyAsync(lse.ptr, dl.ptr, lse_bytes, cudaMemcpyDeviceToHost, hp.out));
    }
  }
  // Both copy streams finish before the device memory is released (on every path).
  if (cudaStreamSynchronize(hp.in) != cudaSuccess && st == RCX_OK) st = RCX_ERR_CUDA;
  if (cudaStreamSynchronize(hp.out) != cudaSuccess && st == RCX_OK) st = RCX_ERR_CUDA;
  cudaFreeAsync(dev, s);
  if (cudaStreamSynchronize(s) != cudaSuccess && st == RCX_OK) st = RCX_ERR_CUDA;
  // This call is synchronous, so a bounded wait that ran out in one of its
  // kernels is reported here (and the status word cleared), not left for a
  // later rcx_device_status().
  int dev_st = RCX_OK;
  if (st == RCX_OK && device_status_all(s, &dev_st) != RCX_OK) st = RCX_ERR_CUDA;
  if (st == RCX_OK && dev_st != RCX_OK) st = dev_st;
  return st;
}

int rcx_release_staging(void) {
  std::lock_guard<std::mutex> lock(g_staging_mu);
  int st = RCX_OK;
  for (int d = 0; d < kMaxDevices; ++d)
    if (g_staging[d] && cudaMemPoolTrimTo(g_staging[d], 0) != cudaSuccess) st = RCX_ERR_CUDA;
  return st;
}

}  // extern "C"

// ------------------------------------------------- ring attention without allocation

// Scratch of rcx_ring_attn_fwd_noalloc: a module-scope device array, so the
// entry point needs no cudaMalloc.  In host code this name only stands for
// the array; its device address comes from cudaGetSymbolAddress with the
// device of the call current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RCX_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device.  Looked up on
// every call rather than cached: the lookup is a host-side query (no
// allocation, no synchronisation), and a cached address would go stale if the
// device's context were torn down and re-created (cudaDeviceReset reloads the
// module, and the array may then sit elsewhere).
int noalloc_scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    std::fprintf(stderr, "librcx: cudaGetSymbolAddress of the no-alloc scratch failed: %s\n",
                 cudaGetErrorString(e));
    return RCX_ERR_CUDA;
  }
  *out = p;
  return RCX_OK;
}

}  // namespace

extern "C" {

int rcx_ring_attn_fwd_noalloc(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                              int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
                              const int64_t* positions, int64_t n_positions, const double* inv_freq,
                              int rope_flags, void* stream) {
  if (check_act(q) || check_act(k) || kv_block < 0) return RCX_ERR_INVALID_ARG;
  const int64_t need = ring_plan(q, k, kv_block, rope_flags).total;
  if (need > (int64_t)RCX_NOALLOC_SCRATCH_BYTES) {
    std::fprintf(stderr,
                 "librcx: rcx_ring_attn_fwd_noalloc needs %lld bytes of scratch; its static buffer holds %lld\n",
                 (long long)need, (long long)RCX_NOALLOC_SCRATCH_BYTES);
    return RCX_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const int st = noalloc_scratch_address(&scratch);
  if (st) return st;
  return ring_impl(q, k, v, o, lse, kv_block, window, n_sink, temperature, positions, n_positions, inv_freq,
                   rope_flags, scratch, (int64_t)RCX_NOALLOC_SCRATCH_BYTES, as_stream(stream));
}

int rcx_device_status(void* stream, int* status_out) {
  if (!status_out) return RCX_ERR_INVALID_ARG;
  return device_status_all(as_stream(stream), status_out);
}

int rcx_stats_enable_timing(int on) {
  Stats& st = stats();
  std::lock_guard<std::mutex> g(st.mu);
  st.timing = on != 0;
  return RCX_OK;
}

int rcx_stats_reset(void) {
  Stats& st = stats();
  std::lock_guard<std::mutex> g(st.mu);
  for (int k = 0; k < RCX_KERNEL_KINDS; ++k) {
    st.launches[k] = 0;
    for (auto& p : st.spans[k]) {
      cudaEventSynchronize(p.second);
      st.pool.push_back(p.first);
      st.pool.push_back(p.second);
    }
    st.spans[k].clear();
  }
  return RCX_OK;
}

int rcx_stats_read(int kind, int64_t* launches_out, double* elapsed_ms_out) {
  if (kind < 0 || kind >= RCX_KERNEL_KINDS) return RCX_ERR_INVALID_ARG;
  Stats& st = stats();
  std::lock_guard<std::mutex> g(st.mu);
  if (launches_out) *launches_out = st.launches[kind];
  double total = 0.0;
  for (auto& p : st.spans[kind]) {
    if (cudaEventSynchronize(p.second) != cudaSuccess) return RCX_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.first, p.second) != cudaSuccess) return RCX_ERR_CUDA;
    total += ms;
  }
  if (elapsed_ms_out) *elapsed_ms_out = total;
  return RCX_OK;
}

int rcx_debug_inject_wait_timeout(int64_t spins) {
  if (spins < 0) return RCX_ERR_INVALID_ARG;
  attn_tc_set_inject(spins);
  return RCX_OK;
}

}  // extern "C"

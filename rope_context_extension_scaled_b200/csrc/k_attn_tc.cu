// Host side of the tensor-core attention kernel (attn_tc.cuh): TMA tensor
// maps, launch configuration, the bounded-wait test hook and the status word.
#include <cuda.h>
#include <algorithm>
#include <cstring>
#include "launch.h"
#include "attn_tc.cuh"

namespace rcx {

// ------------------------------------------------------------------ host side

static std::atomic<int64_t> g_tc_inject_spins{0};
void attn_tc_set_inject(int64_t spins) { g_tc_inject_spins.store(spins); }

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  // looked up once, thread-safely
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

// 4-D map over a [B, N, H, 128] bf16 view, box = 64 columns x 1 head x 128 tokens.
static int make_tile_map(CUtensorMap* map, const rcx_tensor& t) {
  auto enc = tensor_map_encoder();
  if (!enc) return RCX_ERR_CUDA;
  const int64_t B = t.shape[0], N = t.shape[1], H = t.shape[2], D = t.shape[3];
  // Unit-size dimensions get a dense stride (TMA wants 16-byte multiples).
  const int64_t sh = H > 1 ? t.stride[2] : D;
  const int64_t sn = N > 1 ? t.stride[1] : sh * H;
  const int64_t sb = B > 1 ? t.stride[0] : sn * N;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(sh * 2), (cuuint64_t)(sn * 2), (cuuint64_t)(sb * 2)};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)kTcBM, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RCX_OK : RCX_ERR_CUDA;
}

static bool tc_view_ok(const rcx_tensor& t) {
  if (t.dtype != RCX_BF16 || t.shape[3] != kTcD) return false;
  if (reinterpret_cast<uintptr_t>(t.ptr) % 16) return false;
  for (int i = 0; i < 3; ++i)
    if (t.stride[i] % 8) return false;
  if (t.shape[1] > 0x7fffffff - 2 * kTcBM || t.shape[2] > 0x7fffffff || t.shape[0] > 0x7fffffff) return false;
  return true;
}

int attn_tc_launch(const AttnArgs& a, const rcx_tensor& q, const rcx_tensor& k, const rcx_tensor& v,
                   const rcx_tensor& o, cudaStream_t stream) {
  if (!tc_view_ok(q) || !tc_view_ok(k) || !tc_view_ok(v)) return RCX_ERR_ALIGNMENT;
  const int oes = o.dtype == RCX_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(o.ptr) % 16 || o.stride[0] % (16 / oes) || o.stride[1] % (16 / oes) ||
      o.stride[2] % (16 / oes))
    return RCX_ERR_ALIGNMENT;
  if (a.k.N == 0) {
    // no keys at all: every row is empty -> handled by the kernel (zero tiles)
  }
  CUtensorMap mq, mk, mv;
  int st;
  if ((st = make_tile_map(&mq, q)) || (st = make_tile_map(&mk, k)) || (st = make_tile_map(&mv, v))) return st;
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  p.a = a;
  p.pair_heads = (a.G % 2 == 0) ? 1 : 0;
  const int64_t rows_per_item = p.pair_heads ? kTcBM : 2 * kTcBM;
  p.n_rb = (int)((a.q.N + rows_per_item - 1) / rows_per_item);
  p.n_hg = (int)(p.pair_heads ? a.q.H / 2 : a.q.H);
  p.inject_spins = g_tc_inject_spins.load();
  const int64_t items = (int64_t)p.n_rb * p.n_hg * a.q.B;
  if (items <= 0) return RCX_OK;
  if (items > 0x7fffffff) return RCX_ERR_UNSUPPORTED;
  // the kernel's tile walk and row arithmetic are 32-bit: global token
  // indices (and the window, sink and block sizes) stay below 2^31
  const int64_t lim = 0x7fffffffll - 2 * kTcBM;
  if (a.q_start + a.q.N > lim || a.k_start + a.k.N > lim || a.kv_block > lim || a.window > lim || a.n_sink > lim)
    return RCX_ERR_UNSUPPORTED;
  p.n_items = (int)items;
  // persistent: at most one CTA per SM, each walking items blockIdx.x + k * gridDim.x
  const int grid = (int)std::min<int64_t>(items, (int64_t)sm_count());
  const cudaError_t ea = o.dtype == RCX_BF16
                             ? cudaFuncSetAttribute(attn_tc_kernel<__nv_bfloat16>,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmTotal)
                             : cudaFuncSetAttribute(attn_tc_kernel<float>,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmTotal);
  if (ea != cudaSuccess) return RCX_ERR_CUDA;
  LaunchScope scope(RCX_KERNEL_ATTN_TC, stream);
  if (o.dtype == RCX_BF16)
    attn_tc_kernel<__nv_bfloat16><<<grid, kTcThreads, kSmTotal, stream>>>(mq, mk, mv, p);
  else
    attn_tc_kernel<float><<<grid, kTcThreads, kSmTotal, stream>>>(mq, mk, mv, p);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RCX_OK : RCX_ERR_CUDA;
}

int status_exchange_attn_tc(cudaStream_t stream, int* status) { return device_status_exchange(stream, status); }

}  // namespace rcx

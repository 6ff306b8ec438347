// Mask predicate, tile classification and ring-ordered KV block walk shared by
// the attention kernels.
#pragma once
#include "common.cuh"

namespace rcx {

struct AttnArgs {
  View4 q, k, v, o;
  float* lse;                 // [B, Hq, Nq] with unit stride on n; may be null
  int64_t lse_sb, lse_sh;
  int64_t q_start, k_start;   // global token index of row 0 of q / k
  int64_t kv_block;           // ring block size in keys (> 0)
  int64_t window, n_sink;     // window 0 = none
  float scale_log2;           // log2(e) / (sqrt(d) * t)
  const int64_t* positions;   // indexed by global token; null = identity
  int rope_flags;             // RCX_ROTATE_Q | RCX_ROTATE_K
  int pairs;                  // d / 2
  int G;                      // Hq / Hkv
  // Optional previous partial result over other keys (a ring accumulator):
  // acc.ptr == nullptr: none.  Otherwise fp32 [B, Nq, Hq, d] (normalised O)
  // and its natural-log LSE [B, Hq, Nq]; the kernel merges its own result
  // into it by the LSE rule before writing o and lse (which may alias acc).
  View4 acc;
  const float* acc_lse;
  int64_t acc_lse_sb, acc_lse_sh;
  Freqs f;
};

// Causal mask with sliding window of w keys and sinks ("Context window
// extension: 4K to 1M" 4.1, 4.2): j <= i and (w == 0 or j > i - w or j < n_s).
__host__ __device__ __forceinline__ bool mask_visible(int64_t i, int64_t j, int64_t w, int64_t ns) {
  return j <= i && (w == 0 || j > i - w || j < ns);
}

// Does any (i, j) with i in [i0, i1], j in [j0, j1] pass the mask?
__host__ __device__ __forceinline__ bool tile_any_visible(int64_t i0, int64_t i1, int64_t j0, int64_t j1,
                                                          int64_t w, int64_t ns) {
  if (j0 > i1) return false;                         // every key after every row
  if (w == 0) return true;
  if (j1 > i0 - w) return true;                      // some key inside some row's window
  return j0 < ns;                                    // or a sink key
}

// Does every (i, j) in the tile pass the mask (no per-element test needed)?
__host__ __device__ __forceinline__ bool tile_all_visible(int64_t i0, int64_t i1, int64_t j0, int64_t j1,
                                                          int64_t w, int64_t ns) {
  if (j1 > i0) return false;                         // diagonal tile
  if (w == 0) return true;
  if (j0 > i1 - w) return true;                      // all keys inside every row's window
  return j1 < ns;                                    // all keys are sinks
}

}  // namespace rcx

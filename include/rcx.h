/*
 * rcx.h -- C ABI of librcx.so: context-extended attention forward on B200.
 *
 * The library computes the long-context attention forward pass described by
 * the source pages: RoPE frequencies under a scaled schedule, rotation of Q
 * and K, blockwise causal attention with an online softmax over KV blocks
 * visited in Ring-Attention order, and the LSE merge of partial results.
 *
 * Conventions for every entry point:
 *   - Plain pointers and sizes only.  Tensors are passed as rcx_tensor views:
 *     a DEVICE pointer, a dtype, a 4-D shape and element strides.  Q, K, V and
 *     O use [B, N, H, d] (batch, token, head, head_dim) with stride[3] == 1.
 *     LSE tensors use [B, H, N, 1] (fp32, stride[3] ignored).
 *   - The caller owns every buffer.  No entry point allocates device memory
 *     except rcx_ring_attn_fwd_host, which stages its own device copies.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL means
 *     the legacy default stream).  Argument errors are detected on the host
 *     and returned before anything is launched.
 *   - Errors are returned as rcx_status codes; nothing throws across the ABI.
 *     A kernel whose bounded wait runs out records RCX_ERR_DEVICE_TIMEOUT in a
 *     device status word that rcx_device_status() reads.
 *   - Citations name the source page and the section that defines the step.
 */
#ifndef RCX_H
#define RCX_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RCX_OK = 0,
    RCX_ERR_INVALID_ARG = -1,    /* bad shape, stride, scheme or NULL pointer  */
    RCX_ERR_UNSUPPORTED = -2,    /* valid request this build has no path for  */
    RCX_ERR_ALIGNMENT = -3,      /* pointer or stride breaks a vector/TMA rule */
    RCX_ERR_CUDA = -4,           /* a CUDA runtime/driver call failed          */
    RCX_ERR_DEVICE_TIMEOUT = -5  /* a device-side bounded wait gave up         */
} rcx_status;

typedef enum { RCX_F32 = 0, RCX_BF16 = 1, RCX_I8 = 2 /* int8 KV-cache codes only */ } rcx_dtype;

/* RoPE frequency schedules (see rcx_rope_freqs). */
typedef enum {
    RCX_ROPE_PLAIN = 0,      /* theta_i = base^(-2i/d)                              */
    RCX_ROPE_PI = 1,         /* position interpolation m -> m/s                     */
    RCX_ROPE_NTK = 2,        /* base' = base * s^(d/(d-2))                          */
    RCX_ROPE_DYN_NTK = 3,    /* base'(l) with l = L_target, factor 1 if l <= L_train */
    RCX_ROPE_NTK_PARTS = 4,  /* per-pair wavelength bands alpha/beta                 */
    RCX_ROPE_YARN = 5        /* NTK-by-parts frequencies + temperature t            */
} rcx_rope_scheme;

/* Which operands an attention call rotates in-kernel (rope_flags). */
enum { RCX_ROTATE_Q = 1, RCX_ROTATE_K = 2 };

typedef struct {
    void* ptr;           /* device pointer (host pointer for the *_host calls) */
    int32_t dtype;       /* rcx_dtype                                           */
    int64_t shape[4];
    int64_t stride[4];   /* in elements                                         */
} rcx_tensor;

/* Version of the ABI (major * 100 + minor). */
int rcx_abi_version(void);

/* Human-readable name of a status code (static string). */
const char* rcx_status_string(int status);

/*
 * rcx_rope_freqs -- per-pair rotation frequencies theta'_i, i < d/2, and the
 * attention temperature t, in float64 on the host.
 *
 *   theta_i = base^(-2i/d)              ("Context Extension" concept page,
 *                                        RoPE scaling schemes / Technical principles)
 *   s = L_target / L_train
 *   PI:        theta_i / s              ("Context window extension: 4K to 1M" 2.1;
 *                                        the page's m -> m/s, folded into theta)
 *   NTK:       base' = base s^(d/(d-2)) (same page 2.2)
 *   DYN_NTK:   base'(l), l = L_target; factor 1 when l <= L_train (same page 3)
 *   NTK_PARTS: theta_i * f(lambda_i), lambda_i = 2 pi / theta_i; f = 1 below
 *              L_train/beta, 1/s above L_train/alpha, linear in lambda between
 *              (same page 2.3, band reading of the garbled code)
 *   YARN:      NTK_PARTS frequencies and t = 0.1 ln s + 1 (same page 2.4)
 * t = 1 for every scheme but YARN.
 *
 * d: even, 2..256.  L_train, L_target > 0.  alpha, beta used by NTK_PARTS and
 * YARN only (0 < alpha < beta).  inv_freq_out: caller-owned host array of d/2
 * doubles.  temperature_out: host double, may be NULL.
 * Returns RCX_ERR_INVALID_ARG on a bad argument (outputs untouched).
 */
int rcx_rope_freqs(int scheme, double base, int d, int64_t L_train, int64_t L_target,
                   double alpha, double beta, double* inv_freq_out, double* temperature_out);

/*
 * rcx_rope_freqs_per_pair -- per-plane rescaled frequencies
 * theta'_i = base^(-2i/d) / factors[i], i < d/2, in float64 on the host.
 * "Context window extension: 4K to 1M" 2.5 (LongRoPE): each 2D rotation
 * plane gets its own scaling factor; plane i interpolates positions by its
 * factor (m -> m / factors[i]).  The factors come from the caller (the
 * pages' evolutionary search for them is not part of this library).
 * d: even, 2..256; factors: HOST array of d/2 positive finite doubles;
 * inv_freq_out: caller-owned host array of d/2 doubles.
 * Returns RCX_ERR_INVALID_ARG on a bad argument (output untouched).
 */
int rcx_rope_freqs_per_pair(double base, int d, const double* factors, double* inv_freq_out);

/*
 * rcx_rope_apply -- rotate Q and/or K by R(m) ("Context Extension" concept page,
 * Technical principles: each pair of dimensions (2i, 2i+1) turns by
 * phi = m * theta'_i; q_m = R(m) W_q x_m, k_n = R(n) W_k x_n).
 *
 * q, k: [B, N, H, d] inputs (bf16 or f32); q_out, k_out: outputs of the same
 * shape and dtype (out.ptr == in.ptr rotates in place; an operand whose
 * in.ptr is NULL is skipped).  d <= 256 and a multiple of 8 (bf16) or 4
 * (f32); base pointers 16-byte aligned and strides multiples of 16 bytes, else
 * RCX_ERR_ALIGNMENT.  positions: device int64 array of n_positions
 * >= N entries, position of token n is positions[n]; NULL means m = n.
 * inv_freq: HOST array of d/2 doubles (from rcx_rope_freqs).
 * Angles are reduced modulo 2 pi in float64 before an fp32 sincos, so the
 * applied angle is within about 5e-7 rad of m * theta' for every m < 2^24.
 * Memory-bound; data path: read x, write x' once.
 */
int rcx_rope_apply(rcx_tensor q, rcx_tensor k, rcx_tensor q_out, rcx_tensor k_out,
                   const int64_t* positions, int64_t n_positions,
                   const double* inv_freq, void* stream);

/*
 * rcx_attn_blockwise_fwd -- causal attention forward with an online softmax
 * over KV tiles ("Context Extension" concept page, FlashAttention section:
 * B_r x B_c tiles in on-chip memory, running max, O(n) memory), GQA
 * (query head h reads KV head h / (Hq/Hkv)), optional sliding window of
 * `window` keys with `n_sink` StreamingLLM sink keys ("Context window
 * extension: 4K to 1M" 4.1 and 4.2), logits scaled by 1/(sqrt(d) t)
 * (t from rcx_rope_freqs, same page 2.4).
 *
 * q: [B, Nq, Hq, d]; k, v: [B, Nk, Hkv, d]; o: [B, Nq, Hq, d] (bf16 or f32);
 * lse: [B, Hq, Nq, 1] fp32 natural-log LSE of the scaled logits, ptr may be
 * NULL.  Query row i is global token q_start + i, key j is k_start + j; the
 * mask is  j <= i  and (window == 0 or i - window < j or j < n_sink).
 * A row with no visible key gets O = 0 and lse = -inf.
 *
 * kv_block: Ring-Attention block size in keys (0 = the whole sequence is one
 * block).  The KV tiles of a query tile in shard r = i / kv_block are visited
 * in ring order, blocks (r - t) mod P for t = 0, 1, ... ("Context window
 * extension: 4K to 1M" 5.3, kwkr.cn 2.2); the online softmax merges them.
 * The result does not depend on kv_block beyond rounding.
 *
 * rope_flags: RCX_ROTATE_Q / RCX_ROTATE_K rotate that operand in-kernel with
 * inv_freq (HOST, d/2 doubles) at positions[global token] (device int64,
 * n_positions entries; NULL = identity).  rope_flags == 0: Q and K are taken
 * as already rotated.
 *
 * Paths: bf16 inputs with d == 128 run the tcgen05/TMEM tensor-core kernel;
 * it rotates Q in its tile load and needs K pre-rotated (RCX_ROTATE_K returns
 * RCX_ERR_UNSUPPORTED there: rotate K once with rcx_rope_apply).  Other
 * inputs (f32, or bf16 with d != 128) run a SIMT fp32-arithmetic kernel for
 * d in {32, 64, 128}; other d return RCX_ERR_UNSUPPORTED.
 * Alignment: bf16 tensor-core path needs 16-byte aligned base pointers and
 * token/head strides that are multiples of 8 elements.
 */
int rcx_attn_blockwise_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o,
                           rcx_tensor lse, int64_t kv_block, int64_t window, int64_t n_sink,
                           double temperature, int64_t q_start, int64_t k_start,
                           const int64_t* positions, int64_t n_positions,
                           const double* inv_freq, int rope_flags, void* stream);

/*
 * rcx_attn_blockwise_merge_fwd -- one step of the Ring-Attention loop: the
 * attention of rcx_attn_blockwise_fwd over this call's keys, merged in the
 * kernel's epilogue into a previous partial result over other keys by the
 * rule of rcx_merge_partials ("Context window extension: 4K to 1M" 5.3,
 * "output += block_output" made exact by the LSE weights; kwkr.cn 2.2,
 * online aggregation).  No partial buffer is written and no merge pass runs.
 *
 * acc: fp32 [B, Nq, Hq, d], the previous partial's normalised O, 16-byte
 * aligned base and token/head/batch strides that are multiples of 4
 * elements; acc_lse: its [B, Hq, Nq, 1] natural-log LSE (-inf marks a row
 * with no keys so far).  o, lse: the merged result (o f32 or bf16); o may be
 * acc itself and lse may be acc_lse (in-place accumulation: keep lse non-NULL
 * until the last step, or the accumulator's LSE is not updated).  Every other
 * argument, the mask and the paths are as rcx_attn_blockwise_fwd.  A row
 * with no visible key in either partial gets O = 0 and lse = -inf.
 */
int rcx_attn_blockwise_merge_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o,
                                 rcx_tensor lse, rcx_tensor acc, rcx_tensor acc_lse,
                                 int64_t kv_block, int64_t window, int64_t n_sink,
                                 double temperature, int64_t q_start, int64_t k_start,
                                 const int64_t* positions, int64_t n_positions,
                                 const double* inv_freq, int rope_flags, void* stream);

/*
 * rcx_attn_decode_fwd -- attention of one new query token per (batch, head)
 * against a KV cache ("Context Extension" concept page, KV-cache section:
 * each generated token computes Q, K, V, appends K, V to the cache and
 * attends with its Q to the whole cache).  The keys are global tokens
 * 0 .. Nk-1 as stored (already rotated when they were appended, e.g. with
 * rcx_rope_apply); the query is global token q_index; mask, GQA, temperature
 * and LSE as rcx_attn_blockwise_fwd.  The key range is split across CTAs and
 * the partial results are merged with the LSE rule of rcx_merge_partials.
 *
 * q, o: [B, 1, Hq, 128] (q bf16; o bf16 or f32); k, v: [B, Nk, Hkv, 128]
 * bf16 with Hq / Hkv in {1, 2, 4, 8}; lse: [B, Hq, 1, 1] fp32 or ptr NULL.
 * rope_flags: RCX_ROTATE_Q (rotate q at positions[q_index]) or 0;
 * RCX_ROTATE_K returns RCX_ERR_UNSUPPORTED (the cache holds rotated keys).
 * workspace: device buffer of rcx_attn_decode_workspace_size(q, k) bytes,
 * 256-byte aligned, caller-owned.  Memory-bound: reads the cache once.
 */
int64_t rcx_attn_decode_workspace_size(rcx_tensor q, rcx_tensor k);
int rcx_attn_decode_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                        int64_t window, int64_t n_sink, double temperature, int64_t q_index,
                        const int64_t* positions, int64_t n_positions, const double* inv_freq,
                        int rope_flags, void* workspace, int64_t workspace_bytes, void* stream);

/*
 * rcx_kv_quantize_int8 -- int8 KV-cache codes of a bf16 cache
 * ("Context window extension: 4K to 1M" 6.1: the KV cache held in INT8
 * instead of 16-bit floats, half the memory; the "Context Extension" concept
 * page lists the same compression).  Per row of d = 128 values (one token of
 * one head): amax = max |x|, scale = amax / 127, code = rint(x * (127 / amax))
 * clamped to [-127, 127]; a zero row gets scale 0 and zero codes.  The codes
 * are decided in IEEE fp32 (correctly rounded division and product,
 * round-half-to-even), so any fp32 implementation of the same rule gives the
 * same bytes.
 *
 * x: [B, N, H, 128] bf16, 8-byte aligned rows.  codes: [B, N, H, 128]
 * RCX_I8, same shape, 4-byte aligned rows.  scale: device fp32 [B, H, N],
 * contiguous and head-major (row (b, n, h) at (b * H + h) * N + n, so one
 * head's scales for consecutive tokens are adjacent), caller-owned.  Memory
 * bound: reads x once, writes codes and scales once.  Launches are timed
 * under RCX_KERNEL_DECODE.
 */
int rcx_kv_quantize_int8(rcx_tensor x, rcx_tensor codes, float* scale, void* stream);

/*
 * rcx_attn_decode_int8_fwd -- rcx_attn_decode_fwd over an int8 KV cache made
 * by rcx_kv_quantize_int8: key j of KV head h stands for k_codes[j] *
 * k_scale[h, j] (and likewise V).  Same query, mask, GQA, temperature, LSE,
 * rope_flags and split-KV merge as rcx_attn_decode_fwd.  The logits come
 * from int8 products of the stored K codes with each head's rotated query
 * split into two int8 parts (15 bits of its largest element), times the
 * scales; P V runs in fp16 with fp32 accumulation over the V codes with the V
 * scales folded into P, so the result is the attention over the dequantised
 * cache up to those roundings.
 *
 * q, o: [B, 1, Hq, 128] (q bf16; o bf16 or f32); k, v: [B, Nk, Hkv, 128]
 * RCX_I8, 16-byte aligned rows (base and strides multiples of 16 bytes);
 * k_scale, v_scale: device fp32 [B, Hkv, Nk] contiguous (the layout
 * rcx_kv_quantize_int8 writes); Hq / Hkv in
 * {1, 2, 4, 8}; lse: [B, Hq, 1, 1] fp32 or ptr NULL.  workspace: device
 * buffer of rcx_attn_decode_int8_workspace_size(q, k) bytes, 256-byte
 * aligned, caller-owned.  Memory-bound: reads each code and scale once (half
 * the bytes of the bf16 cache).
 */
int64_t rcx_attn_decode_int8_workspace_size(rcx_tensor q, rcx_tensor k);
int rcx_attn_decode_int8_fwd(rcx_tensor q, rcx_tensor k, const float* k_scale, rcx_tensor v,
                             const float* v_scale, rcx_tensor o, rcx_tensor lse, int64_t window,
                             int64_t n_sink, double temperature, int64_t q_index,
                             const int64_t* positions, int64_t n_positions, const double* inv_freq,
                             int rope_flags, void* workspace, int64_t workspace_bytes, void* stream);

/*
 * rcx_merge_partials -- LSE-weighted merge of two partial results over
 * disjoint key sets: m = max(lse_a, lse_b), w = exp(lse - m),
 * o = (w_a o_a + w_b o_b) / (w_a + w_b), lse = m + ln(w_a + w_b).
 * This is the page's "output += block_output" of the Ring Attention loop
 * ("Context window extension: 4K to 1M" 5.3) made exact, and the online
 * aggregation of kwkr.cn 2.2.
 *
 * o_a, o_b: [B, N, H, d] fp32; lse_a, lse_b: [B, H, N, 1] fp32.
 * o_out / lse_out: result (o_out f32 or bf16); o_out.ptr == NULL writes the
 * result back into (o_a, lse_a).  Two -inf partials give o = 0, lse = -inf.
 * Memory-bound.
 */
int rcx_merge_partials(rcx_tensor o_a, rcx_tensor lse_a, rcx_tensor o_b, rcx_tensor lse_b,
                       rcx_tensor o_out, rcx_tensor lse_out, void* stream);

/*
 * rcx_ring_attn_fwd -- the Ring-Attention schedule on one device: the
 * sequence is cut into P = ceil(N / kv_block) blocks; at step t every query
 * shard r attends to KV block (r - t) mod P ("Context window extension: 4K to
 * 1M" 5.3: send to rank + 1, receive from rank - 1; kwkr.cn 2.2: roll the
 * chunks by one), blocks with no visible key are skipped, and each step's
 * partial is merged into an fp32 accumulator with rcx_merge_partials' rule.
 * The final O is written in o's dtype, lse (optional) as for the attention call.
 *
 * q, k, v, o, lse, window, n_sink, temperature, positions, inv_freq,
 * rope_flags: as rcx_attn_blockwise_fwd (q_start = k_start = 0).  With
 * RCX_ROTATE_K on the bf16 path, K is rotated once into the workspace.
 * workspace: device buffer of at least rcx_ring_workspace_size() bytes,
 * 256-byte aligned, owned by the caller.
 */
int64_t rcx_ring_workspace_size(rcx_tensor q, rcx_tensor k, int64_t kv_block, int rope_flags);
int rcx_ring_attn_fwd(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                      int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
                      const int64_t* positions, int64_t n_positions, const double* inv_freq,
                      int rope_flags, void* workspace, int64_t workspace_bytes, void* stream);

/*
 * rcx_ring_attn_fwd_noalloc -- rcx_ring_attn_fwd for callers that cannot
 * allocate device memory, so cannot supply a workspace.  (The source pages
 * have no counterpart: this exists for deployments, not for the method.)
 * Typical such callers run inside a framework whose caching allocator owns
 * the whole device heap, or in a serving loop with a fixed memory budget and
 * a latency bar that cudaMalloc, which can synchronise the device, would break.
 *
 * Same arguments and result as rcx_ring_attn_fwd, minus workspace and
 * workspace_bytes; the caller still passes q, k, v, o and lse.  The scratch
 * (fp32 accumulator, one shard's fp32 partial, their LSEs and the rotated K)
 * lives in a file-scope device array of RCX_NOALLOC_SCRATCH_BYTES that every
 * GPU which loads this library holds until the process exits.  A request whose
 * rcx_ring_workspace_size() exceeds that returns RCX_ERR_UNSUPPORTED (with a
 * message on stderr) before anything is launched.  The call itself makes no
 * cudaMalloc/cudaFree and calls no allocating library routine.
 *
 * Every call looks up the array's device address on the current device with
 * cudaGetSymbolAddress (a host-side query: no allocation, no synchronisation),
 * so the address stays right if the device's context is torn down and
 * re-created.  The first call on a device may load the library's device code
 * there; make that first call before any stream capture.
 * Every call uses the same array and leaves its last contents there; nothing
 * in it has to start at zero, because each call writes every scratch byte it
 * reads.  Calls whose work overlaps on the GPU (different streams, or
 * different host threads) race on the array: serialise them.
 */
#define RCX_NOALLOC_SCRATCH_BYTES (32ll << 20)
int rcx_ring_attn_fwd_noalloc(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                              int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
                              const int64_t* positions, int64_t n_positions, const double* inv_freq,
                              int rope_flags, void* stream);

/*
 * Host<->device convenience for callers without device memory management:
 * same as rcx_ring_attn_fwd but q, k, v, o (and lse if non-NULL) are HOST
 * buffers (pinned for full copy speed; dense [B, N, H, d] and [B, H, N, 1]);
 * the call stages device copies and the workspace, streams the inputs in
 * (K first, then each query shard with its V block) and each shard's output
 * out as soon as it is final, on two copy streams of its own joined to
 * `stream` by events, and returns when everything is back on the host.
 * positions is a HOST array here.  The staging memory comes from a
 * library-owned memory pool of the current device that keeps it after the
 * call, so that repeated calls do not map it again (mapping ~73 GB costs
 * about a second on B200); rcx_release_staging() hands it back.  Because the
 * call synchronises, it also reads (and clears) the device status words: a
 * bounded wait that ran out in one of its kernels returns
 * RCX_ERR_DEVICE_TIMEOUT (o and lse then hold incomplete results).
 */
int rcx_ring_attn_fwd_host(rcx_tensor q, rcx_tensor k, rcx_tensor v, rcx_tensor o, rcx_tensor lse,
                           int64_t kv_block, int64_t window, int64_t n_sink, double temperature,
                           const int64_t* positions, int64_t n_positions, const double* inv_freq,
                           int rope_flags, void* stream);

/*
 * Returns the device memory that rcx_ring_attn_fwd_host keeps between calls
 * (every device's pool is trimmed to zero; memory of a call still running is
 * not touched).  Safe to call at any time; RCX_ERR_CUDA if the runtime
 * refuses.
 */
int rcx_release_staging(void);

/*
 * Device status word: kernels with bounded waits record the first
 * RCX_ERR_DEVICE_TIMEOUT here instead of hanging.  rcx_device_status()
 * synchronises `stream`, stores the word in *status_out and clears it.
 */
int rcx_device_status(void* stream, int* status_out);

/*
 * Test hook: make the next tensor-core attention launches wait on a barrier
 * that nothing arrives at, for `spins` iterations, so that the bounded-wait
 * path is exercised (the kernel records RCX_ERR_DEVICE_TIMEOUT and returns).
 * 0 switches it off.  Host-selected; no fault or trap is involved.
 */
int rcx_debug_inject_wait_timeout(int64_t spins);

/*
 * Launch accounting, for measurement.  Every kernel launch is counted per
 * kind.  With timing on, each launch is also bracketed by two CUDA events
 * recorded on the stream it is launched on; rcx_stats_read() waits for the
 * last of them and returns the summed elapsed time.  Events are host-side
 * CUDA objects (no device memory); the pool is kept until process exit.
 */
typedef enum {
    RCX_KERNEL_ROPE = 0,       /* rope_apply                   */
    RCX_KERNEL_ATTN_TC = 1,    /* tcgen05 bf16 attention       */
    RCX_KERNEL_ATTN_SIMT = 2,  /* SIMT fp32 attention          */
    RCX_KERNEL_MERGE = 3,      /* merge_partials               */
    RCX_KERNEL_DECODE = 4,     /* decode attention + combine   */
    RCX_KERNEL_KINDS = 5
} rcx_kernel_kind;

int rcx_stats_enable_timing(int on);
int rcx_stats_reset(void);
int rcx_stats_read(int kind, int64_t* launches_out, double* elapsed_ms_out);

#ifdef __cplusplus
}
#endif

#endif /* RCX_H */

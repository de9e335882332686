/*
 * fa.h -- C ABI of libfa.so: exact tiled softmax attention for NVIDIA B200 (sm_100a).
 *
 * What is computed (flash-attention README, "How to use FlashAttention"):
 *     O = softmax(softmax_scale * Q K^T + mask) V
 * computed tile by tile with an online softmax, so the Sq x Sk score matrix
 * never reaches device memory.  Every forward entry point also returns the
 * per-row log-sum-exp (kernels-community/flash-attn2 Hub card, "Low-level
 * ops": the low-level ops always return the softmax LSE):
 *     LSE_i = ln( sum_j exp(softmax_scale * q_i . k_j) )   over allowed keys j,
 * natural log, scale included, -inf for a row with no allowed key.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Element type: q, k, v, out, dout, dq, dk, dv, caches are bfloat16; lse is
 *   float32; cu_seqlens / cache_seqlens are int32.  All tensors are dense and
 *   contiguous with the head dimension D innermost.
 * - Pointers are DEVICE pointers of the current CUDA device, 16-byte aligned
 *   (tile loads use the tensor memory accelerator).  The caller owns every
 *   buffer; the library never allocates, never frees and never synchronises.
 *   Outputs are overwritten, never accumulated into.
 * - `stream` is a cudaStream_t passed as void*; all work is enqueued on it and
 *   the call returns as soon as it is enqueued.  NULL means the legacy default
 *   stream.
 * - Heads: Hq must be a multiple of Hkv; query head h reads KV head
 *   h / (Hq / Hkv) (flash-attention README, flash_attn_func docstring, MQA/GQA:
 *   6 query heads over 2 KV heads -> query heads 0-2 read KV head 0).
 * - Causal masking is aligned to the bottom-right corner: key j is allowed for
 *   query i iff j <= i + Sk - Sq (README, flash_attn_with_kvcache docstring and
 *   changelog 2.1).  A query row with no allowed key produces O = 0 and
 *   LSE = -inf; its gradients are zero.
 * - Head dims supported: D in {64, 128, 256} (the README caps head dims at 256).
 * - softmax_scale is explicit; the Python binding supplies 1/sqrt(D) by default.
 * - Workspace: each entry point that needs device scratch takes
 *   (workspace, workspace_bytes); the matching *_workspace_size() returns the
 *   bytes required (0 = none; workspace may then be NULL).  Workspace must be
 *   256-byte aligned and is not preserved between calls.
 * - Per-device state (the status word's address, the SM count, the kernels'
 *   shared-memory attributes) is looked up on the first call on a device and
 *   kept for the life of the process: a cudaDeviceReset of that device after
 *   the first call is not supported.
 *
 * Errors: every entry point returns an fa_status.  Arguments are validated
 * before anything is enqueued; a non-zero status means nothing was launched,
 * except FA_ERR_CUDA (a launch failed; the CUDA error is left pending for the
 * caller).  Kernels never trap: a wait that runs out of time records
 * FA_ERR_TIMEOUT in a per-device status word and the kernel returns; read it
 * with fa_get_device_status().
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

typedef void* fa_stream_t; /* a cudaStream_t */

enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* non-positive sizes, Hq % Hkv != 0, NULL pointer, bad page size / table */
    FA_ERR_UNSUPPORTED = 2,  /* head dim outside {64, 128, 256}, or a size beyond the int32 index range */
    FA_ERR_ALIGNMENT = 3,    /* a tensor pointer is not 16-byte aligned / workspace not 256-byte aligned */
    FA_ERR_WORKSPACE = 4,    /* workspace_bytes smaller than the *_workspace_size() figure */
    FA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    FA_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up (reported by fa_get_device_status) */
};

/* ------------------------------------------------------------------------- dense forward
 * fa_fwd: batched attention over equal-length sequences.
 *   q    [B, Sq, Hq,  D]      k, v [B, Sk, Hkv, D]      out [B, Sq, Hq, D]
 *   lse  [B, Hq, Sq] float32 (required: the backward consumes it)
 * Source: README, "How to use FlashAttention" (definition) and the
 * flash_attn_func docstring (shapes, GQA, causal).
 * Workspace: optional.  With fa_fwd_workspace_size() bytes (256) the persistent
 * kernel takes its work units from a counter there as CTAs finish (balanced on
 * unequal sequence lengths; heads grouped so their K and V stay in L2), zeroed
 * on `stream` by the call itself; with workspace = NULL the units are dealt
 * statically.  The result does not depend on the choice (each unit's
 * arithmetic is the same either way).
 */
FA_API size_t fa_fwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D);
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
           int B, int Hq, int Hkv, int Sq, int Sk, int D,
           float softmax_scale, int causal,
           void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- dense backward
 * fa_bwd: gradients of sum(out * dout) with respect to q, k, v, recomputing
 * the scores from q, k, v and lse (README, section on IO-aware tiling and
 * recomputation; FlashAttention fork v1.4 notes, section 4: the backward
 * re-applies the exponential against the stored statistics).
 *   q, dq [B, Sq, Hq, D]   k, v, dk, dv [B, Sk, Hkv, D]   out, dout [B, Sq, Hq, D]
 *   lse [B, Hq, Sq] float32 as written by fa_fwd.
 * With GQA, dk/dv of a KV head are summed over the query heads that read it.
 * Workspace (fa_bwd_workspace_size): float32 dq accumulator and per-row
 * statistics.  dq accumulation order is not fixed, so dq is not bit-reproducible
 * run to run; dk and dv are.
 */
FA_API size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D);
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
           const float* lse, void* dq, void* dk, void* dv,
           int B, int Hq, int Hkv, int Sq, int Sk, int D,
           float softmax_scale, int causal,
           void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- varlen forward
 * fa_varlen_fwd: packed batch of num_seqs independent sequences (names from the
 * Hub card's function list, flash_attn_varlen_func).  Sequence s occupies rows
 * cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 of q/out and cu_seqlens_k[s] ..
 * cu_seqlens_k[s+1]-1 of k/v; cu_seqlens_*[0] = 0, non-decreasing, last entry
 * = total_*.  Both arrays are DEVICE int32 [num_seqs + 1].  max_seqlen_* must
 * bound every sequence length (they size the grid).
 *   q, out [total_q, Hq, D]    k, v [total_k, Hkv, D]    lse [Hq, total_q] float32
 * Workspace: optional, as for fa_fwd (the dynamic schedule balances unequal lengths).
 */
FA_API size_t fa_varlen_fwd_workspace_size(int num_seqs, int total_q, int total_k, int Hq, int Hkv, int D);
FA_API int fa_varlen_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                  int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                  int Hq, int Hkv, int D, float softmax_scale, int causal,
                  void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- varlen backward
 * fa_varlen_bwd: backward of fa_varlen_fwd; layouts as there, plus
 *   dout, dq [total_q, Hq, D]   dk, dv [total_k, Hkv, D]
 */
FA_API size_t fa_varlen_bwd_workspace_size(int num_seqs, int total_q, int total_k, int Hq, int Hkv, int D);
FA_API int fa_varlen_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                  int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                  int Hq, int Hkv, int D, float softmax_scale, int causal,
                  void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- sliding window, deterministic backward
 * The *_ex entry points are the four calls above with the remaining options of
 * flash_attn_func / flash_attn_varlen_func (README, flash_attn_func docstring);
 * the calls above are the *_ex calls with window_left = window_right = -1 and
 * deterministic = 0.  Workspace needs and sizes are those of the plain calls.
 *
 * window_left, window_right: sliding window local attention (README changelog
 *   2.3, flash_attn_func docstring).  Query i of a sequence keeps only the keys
 *   j with  i + Sk - Sq - window_left <= j <= i + Sk - Sq + window_right
 *   (bottom-right aligned like the causal mask; Sq, Sk the lengths of that
 *   sequence).  A negative side (-1) is unbounded; (-1, -1) is no window.  With
 *   causal != 0 the keys kept are those both rules keep, i.e. the right side is
 *   0.  Rows left with no key give out = 0, lse = -inf and zero gradients.
 * deterministic (backward only): 0 accumulates dq with float32 reduce-adds whose
 *   order varies from run to run; 1 computes dq in a separate pass in which each
 *   query tile sums its key tiles in a fixed order, so dq, dk and dv are
 *   bit-identical across runs on the same inputs (README: the deterministic
 *   backward is slightly slower; the forward is always deterministic).
 * Errors as for the plain calls; sequence lengths above 2^30 are
 * FA_ERR_UNSUPPORTED on every dense and varlen entry point.
 */
FA_API int fa_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                     int B, int Hq, int Hkv, int Sq, int Sk, int D,
                     float softmax_scale, int causal, int window_left, int window_right,
                     void* workspace, size_t workspace_bytes, fa_stream_t stream);
FA_API int fa_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv,
                     int B, int Hq, int Hkv, int Sq, int Sk, int D,
                     float softmax_scale, int causal, int window_left, int window_right, int deterministic,
                     void* workspace, size_t workspace_bytes, fa_stream_t stream);
FA_API int fa_varlen_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                            int Hq, int Hkv, int D, float softmax_scale, int causal,
                            int window_left, int window_right,
                            void* workspace, size_t workspace_bytes, fa_stream_t stream);
FA_API int fa_varlen_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout,
                            const float* lse, void* dq, void* dk, void* dv,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                            int Hq, int Hkv, int D, float softmax_scale, int causal,
                            int window_left, int window_right, int deterministic,
                            void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- KV-cache decode
 * fa_fwd_kvcache: new queries against a contiguous KV cache (README,
 * flash_attn_with_kvcache docstring; changelog 2.2: the cache load is split
 * across thread blocks and a separate kernel combines the pieces).
 *   q [B, Sq, Hq, D]   k_cache, v_cache [B, cache_capacity, Hkv, D]
 *   cache_seqlens DEVICE int32 [B]: batch row b uses keys 0 .. cache_seqlens[b]-1,
 *   each in [0, cache_capacity]; rows beyond it are never read into the result.
 *   out [B, Sq, Hq, D]   lse [B, Hq, Sq] float32, or NULL if not wanted.
 * Sq >= 1 new query tokens per row; with causal != 0 token i of row b sees
 * keys 0 .. i + cache_seqlens[b] - Sq (bottom-right aligned; for Sq = 1 that is
 * every valid key).  num_splits = 0 picks the split of the cache
 * automatically; > 0 asks for that many splits of cache_capacity.  The result
 * does not depend on the split except through float32 rounding.
 * Workspace (fa_fwd_kvcache_workspace_size): float32 partial outputs and LSEs.
 * Head dims 64, 128 and 256.  No backward (the docstring states the same).
 * The automatic split (num_splits = 0) is sized for 148 SMs (B200) whatever
 * the device, so the workspace size does not depend on the device it runs on.
 */
FA_API size_t fa_fwd_kvcache_workspace_size(int B, int Hq, int Hkv, int Sq, int cache_capacity, int D, int num_splits);
FA_API int fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_seqlens,
                   void* out, float* lse,
                   int B, int Hq, int Hkv, int Sq, int cache_capacity, int D,
                   float softmax_scale, int causal, int num_splits,
                   void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- KV-cache: append, pages, windows
 * fa_fwd_kvcache_ex: the rest of flash_attn_with_kvcache (README docstring),
 * without rotary embedding.  In order, on `stream`:
 *  1. If k_new / v_new [B, seqlen_new, Hkv, D] are given (both, seqlen_new > 0),
 *     they are written into k_cache / v_cache IN PLACE at logical rows
 *     cache_seqlens[b] .. cache_seqlens[b] + seqlen_new - 1 of sequence b.
 *     Rows past what the sequence can hold are not written.  cache_seqlens is
 *     not modified (the caller advances it).
 *  2. Sequence b attends to its first min(cache_seqlens[b] + seqlen_new, cap)
 *     logical rows, with the bottom-right aligned causal mask and sliding window
 *     of fa_fwd_ex, where cap = cache_capacity (contiguous) or
 *     max_blocks_per_seq * page_block_size (paged).
 * Cache layouts:
 *  - contiguous (block_table = NULL): caches [cache_batch, cache_capacity, Hkv, D];
 *    sequence b uses cache row cache_batch_idx[b] (DEVICE int32 [B]) or b when
 *    cache_batch_idx is NULL.  With repeated indices and k_new given, which
 *    sequence's rows end up in the cache is unspecified (as in the docstring).
 *  - paged: caches [cache_batch = num_blocks, cache_capacity = page_block_size,
 *    Hkv, D], page_block_size a multiple of 256 (README); block_table DEVICE
 *    int32 [B, max_blocks_per_seq]: logical rows i*page .. i*page+page-1 of
 *    sequence b live in block block_table[b][i] (the reading taken of the
 *    docstring's block_table).  cache_batch_idx must then be NULL.
 *  q [B, Sq, Hq, D] and out [B, Sq, Hq, D]; lse [B, Hq, Sq] float32 or NULL.
 * A block id or cache_batch_idx entry outside the cache is not dereferenced:
 * the kernels record FA_ERR_INVALID_ARG in the device status word
 * (fa_get_device_status) and such rows read as zeros / the sequence as empty.
 * Workspace: fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, Sq, D, cache_capacity,
 * max_blocks_per_seq (0 for a contiguous cache), num_splits).
 */
FA_API size_t fa_fwd_kvcache_ex_workspace_size(int B, int Hq, int Hkv, int Sq, int D, int cache_capacity,
                                               int max_blocks_per_seq, int num_splits);
FA_API int fa_fwd_kvcache_ex(const void* q, void* k_cache, void* v_cache, const int32_t* cache_seqlens,
                             const void* k_new, const void* v_new, int seqlen_new,
                             const int32_t* cache_batch_idx, const int32_t* block_table, int max_blocks_per_seq,
                             int cache_batch, int cache_capacity,
                             void* out, float* lse, int B, int Hq, int Hkv, int Sq, int D,
                             float softmax_scale, int causal, int window_left, int window_right, int num_splits,
                             void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* ------------------------------------------------------------------------- merging partial attention results
 * fa_merge_lse: attention over the union of disjoint key sets from the results
 * over each set (for context-parallel / ring attention, where each rank attends
 * to one shard of the keys):
 *     LSE = ln sum_c exp(LSE_c),   out = sum_c exp(LSE_c - LSE) O_c
 * (README changelog 2.2: the split-KV decode merges its pieces the same way;
 * the forward's LSE output is what makes it possible).  Parts with LSE_c = -inf
 * contribute nothing; a row with every part empty gets out = 0, LSE = -inf.
 *   o_parts   [num_parts, B, S, H, D], bf16 (parts_fp32 = 0) or float32 (1)
 *   lse_parts [num_parts, B, H, S] float32 (the layout fa_fwd writes; a varlen
 *             result [H, total] is B = 1, S = total)
 *   out       [B, S, H, D], bf16 (out_fp32 = 0) or float32 (1)
 *   lse       [B, H, S] float32, or NULL
 * D in {64, 128, 256}.  out may be the memory of one of the parts (and lse of
 * one of the LSE parts): each row is read completely before it is written.
 */
FA_API int fa_merge_lse(const void* o_parts, const float* lse_parts, int num_parts, int B, int S, int H, int D,
                        int parts_fp32, void* out, float* lse, int out_fp32, fa_stream_t stream);

/* ------------------------------------------------------------------------- KV-cache decode without caller memory
 * fa_fwd_kvcache_noalloc: the same computation as fa_fwd_kvcache, for callers
 * that cannot allocate device memory when they decode -- for example a plugin or
 * inference runtime that plans its device memory ahead of time and only receives
 * the tensors it owns, or a C program with no allocator of its own.  The source
 * pages have no counterpart of this entry point; it is an interface addition.
 *
 * The per-split partial results live in one array compiled into the library
 * (fa_fwd_kvcache_noalloc_scratch_bytes() bytes, 16 MiB).  Every GPU that loads
 * the library holds that array until the process exits.  The caller still
 * passes q, the caches, cache_seqlens, out and (optionally) lse exactly as for
 * fa_fwd_kvcache; no workspace argument, and nothing is allocated or freed.
 *   - The first call on a device looks up the array's device address there
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is kept for the life of the process: calling it again after a
 *     cudaDeviceReset of that device is not supported.
 *   - All calls share the array: calls that overlap on the GPU (other streams,
 *     other host threads) race on it and must be serialised by the caller.
 *     Nothing in it needs to start at zero; each call writes what it reads.
 *   - With num_splits = 0 the split is chosen as for fa_fwd_kvcache; when its
 *     partials do not fit, the largest smaller split count n whose partials fit
 *     is used, split exactly as fa_fwd_kvcache splits with num_splits = n, so the
 *     result is bit-identical to that call's (and to the num_splits = 0 call's
 *     when no coarsening is needed).  If they cannot fit (an explicit
 *     num_splits too large, or B * Sq * Hq * (D + 1) * 4 bytes beyond the array),
 *     the call returns FA_ERR_WORKSPACE and launches nothing.
 */
FA_API size_t fa_fwd_kvcache_noalloc_scratch_bytes(void);
FA_API int fa_fwd_kvcache_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* cache_seqlens, void* out, float* lse,
                                  int B, int Hq, int Hkv, int Sq, int cache_capacity, int D,
                                  float softmax_scale, int causal, int num_splits, fa_stream_t stream);

/* ------------------------------------------------------------------------- helpers
 * fa_status_string: static English text for a status code (never NULL).
 */
FA_API const char* fa_status_string(int status);

/* fa_get_device_status: enqueues a read of the current device's status word on
 * `stream`, SYNCHRONISES that stream, clears the word, and returns FA_OK or the
 * first error a kernel recorded since the last call (FA_ERR_TIMEOUT).  Returns
 * FA_ERR_CUDA if the read itself fails.  Diagnostic; not for the hot path.
 */
FA_API int fa_get_device_status(fa_stream_t stream);

/* fa_set_wait_timeout_ns: time limit for every bounded device-side wait in
 * kernels launched after this call (process-wide; default 2e9 ns).  0 restores
 * the default.  Returns the previous value.
 */
FA_API unsigned long long fa_set_wait_timeout_ns(unsigned long long ns);

/* Kernel timing with CUDA events, for benchmarks.  fa_profile_begin(1) makes
 * every later launch of the main kernel of fa_fwd / fa_varlen_fwd (id 0), the
 * main backward kernel of fa_bwd / fa_varlen_bwd (id 1), the split kernel of
 * fa_fwd_kvcache (id 2) and the dQ pass of the deterministic backward (id 3)
 * record a pair of CUDA events around itself, and every fa_bwd / fa_varlen_bwd
 * call records one pair around all of its launches (id 4: preprocess, main
 * kernel and dQ convert or dQ pass), on the
 * launching stream (up to 1024 launches per id; later ones are not recorded),
 * and clears earlier records; fa_profile_begin(0) stops recording.
 * fa_profile_read, after the caller has synchronised those streams, returns the
 * number of recorded launches of `kernel_id` and the sum of their durations in
 * milliseconds.  Events are created on first use; no device memory is allocated.
 */
enum fa_kernel_id {
    FA_KERNEL_FWD = 0, FA_KERNEL_BWD = 1, FA_KERNEL_DECODE = 2, FA_KERNEL_BWD_DQ = 3, FA_KERNEL_BWD_ALL = 4
};
FA_API int fa_profile_begin(int enable);
FA_API int fa_profile_read(int kernel_id, int* launches, float* total_ms);

/* fa_debug_wait_timeout_selftest: launches one block whose wait on a barrier
 * nobody arrives at runs out after timeout_ns; the kernel records
 * FA_ERR_TIMEOUT and returns.  Used by the tests to show that a stuck wait ends
 * with a status instead of a hang.  Asynchronous on `stream`.
 */
FA_API int fa_debug_wait_timeout_selftest(unsigned long long timeout_ns, fa_stream_t stream);

/* fa_debug_umma_selftest: one 128x128x128 bf16 tensor-core product on one CTA,
 * for checking shared-memory descriptor, tensor-memory and operand-packing
 * conventions.  a, b: bf16 [128][128] row-major; c: float32 [128][128].
 *   mode 0: c = a . b^T     (both operands K-major in shared memory)
 *   mode 1: c = a . b       (b N-major in shared memory)
 *   mode 2: c = a . b       (a copied into tensor memory as bf16, b N-major)
 */
FA_API int fa_debug_umma_selftest(const void* a, const void* b, float* c, int mode, fa_stream_t stream);

/* fa_debug_exp2_selftest: y[i] = 2^x[i] for n (even) device floats, computed with the
 * FMA-pipe exponential the softmax kernels use for part of their exponentials, so that
 * its accuracy can be checked against CUDA's exp2f.  Asynchronous on `stream`.
 */
FA_API int fa_debug_exp2_selftest(const float* x, float* y, int n, fa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FA_H_ */

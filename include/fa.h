/*
 * fa.h -- C ABI of libfa.so: exact, IO-aware scaled-dot-product attention on B200.
 *
 * The operation (youngju.dev "attention variants", section 1 cost analysis and the
 * gqa_attention example of section 2; toolsku.com generation 1 MHA formula):
 *
 *     O = softmax(Q K^T * scale [+ causal mask]) V,     LSE = ln sum_j exp(s_ij)
 *
 * computed without ever writing the (N, N) score matrix to memory: Q, K and V are
 * staged tile by tile into on-chip memory and the softmax is accumulated online with a
 * running row maximum and sum (youngju.dev section 3, FlashAttention).  Grouped-query
 * sharing (youngju.dev section 2; toolsku.com generation 2): with Hq query heads and
 * Hkv key/value heads (Hkv = G on the pages; G = Hq is MHA, G = 1 is MQA), query head h
 * reads key/value head h / (Hq / Hkv), the repeat_interleave mapping.
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major, in device memory, and owned by the caller; the
 *     library allocates nothing per call and keeps no pointer after it returns.
 *   - q, k, v, kcache, vcache and o must be 16-byte aligned (the TMA engine requires it).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call only
 *     enqueues work on that stream and returns without synchronising.
 *   - Errors in the arguments are returned synchronously and nothing is launched.
 *     Errors the device detects (a pipeline wait that exceeded its time limit, a cache
 *     length out of range) are recorded in a device error word that fa_get_error reads.
 *   - Threads: the calls are thread-safe; the last error message is per host thread.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID = 1,      /* bad argument: null pointer, size <= 0, Hq % Hkv != 0,
                                causal with Nq > Nk, scale not finite and > 0 */
    FA_ERR_UNSUPPORTED = 2,  /* valid but not supported: d not in {64, 128}, a pointer that
                                is not 16-byte aligned, no sm_100 device */
    FA_ERR_WORKSPACE = 3,    /* decode workspace null or smaller than required */
    FA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed; see fa_last_error_message */
    FA_ERR_TIMEOUT = 5,      /* a kernel pipeline wait exceeded its time limit (fa_get_error) */
    FA_ERR_DEVICE_ARG = 6,   /* the device found seqlens[b] outside [0, Nmax] and clamped it,
                                or a block-table entry outside the page pool */
    FA_ERR_DEBUG_CHECK = 7   /* debug builds only: a global-memory index computed by a kernel
                                failed its bounds check; the access was skipped */
} fa_status;

typedef enum { FA_BF16 = 0, FA_F32 = 1 } fa_dtype;

/*
 * Prefill / generic forward attention, bf16 output.
 *   q   (B, Hq,  Nq, d) bf16          k, v (B, Hkv, Nk, d) bf16
 *   o   (B, Hq,  Nq, d) bf16 (written)
 *   lse (B, Hq,  Nq)    fp32 (written), natural log of sum_j exp(scale * q_i . k_j)
 *   scale: multiplies q.k; pass 1/sqrt(d) for the usual softmax(QK^T/sqrt(d_k)).
 *   causal != 0: row i sees keys j <= i + (Nk - Nq) (bottom-right alignment; equal to
 *   the usual lower-triangular mask when Nq == Nk).  Requires Nq <= Nk.
 * Supported: d in {64, 128}; any B, Hq, Hkv with Hq % Hkv == 0; any Nq, Nk >= 1.
 */
FA_API int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
           void *stream);

/* As fa_fwd, with the output element type chosen by o_dtype (FA_BF16 or FA_F32). */
FA_API int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
              int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
              int o_dtype, void *stream);

/*
 * Sliding-window causal attention (youngju.dev "attention variants", section 4: every
 * token attends only to the W most recent tokens, itself included, so the cost falls
 * from N^2 to N x W; with W = 3, query 5 sees keys 3, 4 and 5).  With the bottom-right
 * alignment of fa_fwd, row i sees keys j with i + (Nk - Nq) - W < j <= i + (Nk - Nq);
 * Nq < Nk is chunked prefill (youngju.dev section 5): the Nq new rows are the last Nq
 * positions of a sequence whose first Nk - Nq keys are already cached.
 *   window: W >= 1 (FA_ERR_INVALID otherwise); W >= Nk gives plain causal attention.
 *   Key tiles that lie wholly outside every row's window are neither loaded nor
 *   multiplied.  Other arguments, layouts, ownership and errors as fa_fwd_ex.
 */
FA_API int fa_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                  int o_dtype, void *stream);

/*
 * Forward attention over FP8 (E4M3) Q, K and V.  FP8 is among the data types of
 * FlashAttention-3 in the toolsku.com "attention mechanism evolution" FlashAttention
 * generations table; the pages fix no scale convention, and this library's is one
 * dequantization scale per head:
 *   q[b,h,i,:] = q_scale[h] * e4m3(q8[b,h,i,:]),  k[b,g,j,:] = k_scale[g] * e4m3(k8[b,g,j,:]),
 *   v[b,g,j,:] = v_scale[g] * e4m3(v8[b,g,j,:]),
 * and the result is the attention of these tensors (masks, alignment and LSE as fa_fwd_ex
 * and fa_fwd_window).
 *   q  (B, Hq,  Nq, d) uint8 E4M3 bytes ("e4m3fn": bias 7, no infinities), device
 *   k, v (B, Hkv, Nk, d) uint8 E4M3 bytes, device
 *   q_scale (Hq), k_scale (Hkv), v_scale (Hkv): fp32, device
 *   o   (B, Hq, Nq, d) written, bf16 or fp32 (o_dtype); lse (B, Hq, Nq) fp32 written
 *   causal, window: as fa_fwd_window (window 0 for none; a window needs causal != 0).
 * S = Q K^T is computed exactly in fp32 from the E4M3 codes on the tensor cores; P is
 * rounded to fp16 for P V (V widened to fp16 on chip, exactly).  d must be 128
 * (FA_ERR_UNSUPPORTED otherwise); a null scale pointer is FA_ERR_INVALID.  E4M3 NaN bytes
 * are not special-cased.  Ownership, alignment and the other errors as fa_fwd_ex.
 */
FA_API int fa_fwd_fp8(const void *q, const void *k, const void *v, const float *q_scale,
                      const float *k_scale, const float *v_scale, void *o, float *lse, int B, int Hq,
                      int Hkv, int Nq, int Nk, int d, float scale, int causal, int window, int o_dtype,
                      void *stream);

/*
 * Forward attention on (batch, sequence, heads, dim) tensors, the layout of the
 * flash_attn_func call in toolsku.com "attention mechanism evolution", FlashAttention
 * usage example (its layer views the projections as (B, S, H, d) and passes them on with
 * no transpose):
 *   q   (B, Nq, Hq,  d) bf16          k, v (B, Nk, Hkv, d) bf16
 *   o   (B, Nq, Hq,  d) written, bf16 or fp32 (o_dtype)
 *   lse (B, Hq,  Nq)    fp32 written (the head-major layout of fa_fwd)
 *   causal, scale: as fa_fwd.  window: 0 for none, else W >= 1 with causal != 0, as
 *   fa_fwd_window (FA_ERR_INVALID for W < 0 or a window without causal).
 * The result equals fa_fwd_ex / fa_fwd_window on the same tensors transposed to
 * (B, H, N, d): the kernel reads the same tiles through strided TMA descriptors, so no
 * transposed copy is made.  Supported sizes and errors as fa_fwd_ex.
 */
FA_API int fa_fwd_bshd(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                int window, int o_dtype, void *stream);

/*
 * Bytes of device workspace fa_decode needs for these sizes (fp32 partial outputs and
 * partial log-sum-exps of the split-KV chunks).  0 if the sizes are invalid.
 */
FA_API size_t fa_decode_workspace_size(int B, int Hq, int Nmax, int d);

/*
 * Decode step over a KV cache (one query row per sequence and head): youngju.dev
 * section 7 (decode reads the whole cache every step) and the past_kv path of the
 * toolsku.com MHA/GQA modules (the cached keys are concatenated before the scores).
 *   q        (B, Hq, d) bf16            kcache, vcache (B, Hkv, Nmax, d) bf16
 *   seqlens  int32[B] in device memory, each in [0, Nmax]: sequence b attends cached
 *            keys 0 .. seqlens[b]-1, unmasked.  seqlens[b] == 0 gives o = 0, lse = -inf.
 *   o        (B, Hq, d) bf16 (written);  lse (B, Hq) fp32 (written) or NULL.
 *   workspace/workspace_bytes: caller-owned device scratch of at least
 *            fa_decode_workspace_size(B, Hq, Nmax, d) bytes, 16-byte aligned; its contents
 *            need no initialisation and are overwritten.  Calls that share a workspace
 *            must be ordered (same stream, or synchronised).
 * The cache is split into chunks of 256 keys processed in parallel; the partial results
 * are combined exactly by a log-sum-exp merge.
 */
FA_API int fa_decode(const void *q, const void *kcache, const void *vcache, const int *seqlens,
              void *o, float *lse, int B, int Hq, int Hkv, int Nmax, int d, float scale,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * As fa_decode, with the output element type chosen by o_dtype: FA_BF16 or FA_F32 (o is
 * then (B, Hq, d) fp32).  The fp32 output keeps partial results exact enough to be merged
 * again, as fa_merge_lse does for a cache split across devices.
 */
FA_API int fa_decode_ex(const void *q, const void *kcache, const void *vcache, const int *seqlens,
                 void *o, float *lse, int B, int Hq, int Hkv, int Nmax, int d, float scale,
                 int o_dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Log-sum-exp merge of P partial attention results over disjoint key sets (the same
 * rescaling the online softmax applies between key blocks, youngju.dev "attention
 * variants" section 3, applied across parts): for every row,
 *     M = max_p lse_p,  w_p = exp(lse_p - M),  o = sum_p w_p o_p / sum_p w_p,
 *     lse = M + ln sum_p w_p.
 * Used for context-parallel decode: each device decodes its own slab of every sequence's
 * keys (fa_decode_ex with FA_F32), the (o, lse) pairs are all-gathered, and this call
 * combines them into the result over the whole cache.
 *   o_parts   (P, rows, d) fp32 device memory;  lse_parts (P, rows) fp32, natural log,
 *             -inf for a part that saw no key (its o_p is ignored).
 *   o         (rows, d) written, bf16 or fp32 (o_dtype);  lse (rows) written, or NULL.
 *   A row whose every part is -inf gets o = 0 and lse = -inf.  d in {64, 128}.
 * This library adds it: the pages merge only the blocks of one pass.
 */
FA_API int fa_merge_lse(const float *o_parts, const float *lse_parts, int P, int rows, int d,
                 void *o, float *lse, int o_dtype, void *stream);

/*
 * Decode step over a paged KV cache (youngju.dev "attention variants", section 5: the
 * cache is cut into fixed-size blocks managed like virtual-memory pages, which removes
 * fragmentation).  The page layout is this library's choice:
 *   kpages, vpages  (num_pages, Hkv, page_size, d) bf16: a page holds page_size
 *                   consecutive tokens of one sequence for every K/V head;
 *   block_table     int32 (B, max_pages) in device memory: token t of sequence b is row
 *                   t % page_size of page block_table[b * max_pages + t / page_size].
 *                   Only the entries of pages 0 .. ceil(seqlens[b] / page_size) - 1 are
 *                   read; each must lie in [0, num_pages).  An entry outside it is
 *                   reported by fa_get_error as FA_ERR_DEVICE_ARG, and the keys of that
 *                   page read as zeros (no memory outside the pool is touched).
 *   seqlens         int32[B], each in [0, page_size * max_pages].
 *   page_size       a multiple of 16 (FA_ERR_UNSUPPORTED otherwise).
 *   workspace       at least fa_decode_workspace_size(B, Hq, page_size * max_pages, d)
 *                   bytes, as for fa_decode.
 * q, o, lse, scale, stream and the result are exactly those of fa_decode on the cache the
 * pages spell out.
 */
FA_API int fa_decode_paged(const void *q, const void *kpages, const void *vpages,
                    const int *block_table, const int *seqlens, void *o, float *lse,
                    int B, int Hq, int Hkv, int num_pages, int page_size, int max_pages,
                    int d, float scale, void *workspace, size_t workspace_bytes,
                    void *stream);

/*
 * Decode step over an FP8 KV cache (youngju.dev "attention variants", sections 5 and 7:
 * storing the cache in FP8 halves its bytes, and decode is bound by reading them).  The
 * pages fix no scale convention; this library's is one dequantization scale per K/V head
 * for K and one for V:
 *   kcache, vcache  (B, Hkv, Nmax, d) bytes, each an OCP FP8 E4M3 ("e4m3fn") value;
 *   k_scale, v_scale float32[Hkv] in device memory: key j of head g is
 *                   k_scale[g] * e4m3(kcache[b, g, j, :]), likewise V with v_scale
 *                   (a single per-tensor scale is the case of equal entries).
 * q (bf16), o (bf16), lse, seqlens, workspace (fa_decode_workspace_size(B, Hq, Nmax, d)),
 * scale and stream are those of fa_decode, and so is the result on the dequantized cache.
 * Supported: d = 128 (FA_ERR_UNSUPPORTED otherwise).  Inside, every E4M3 value is
 * converted exactly to fp16 and multiplied with fp16 operands (fp32 accumulation); q
 * enters as fp16 after an exact power-of-two scaling of each row, and the softmax
 * weights P as fp16.
 */
FA_API int fa_decode_fp8(const void *q, const void *kcache, const void *vcache,
                  const float *k_scale, const float *v_scale, const int *seqlens, void *o,
                  float *lse, int B, int Hq, int Hkv, int Nmax, int d, float scale,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * The FP8 decode over a paged cache: kpages/vpages (num_pages, Hkv, page_size, d) E4M3
 * bytes with the page layout and block table of fa_decode_paged, and the per-head scales
 * of fa_decode_fp8.  Workspace: fa_decode_workspace_size(B, Hq, page_size * max_pages, d).
 */
FA_API int fa_decode_paged_fp8(const void *q, const void *kpages, const void *vpages,
                        const float *k_scale, const float *v_scale, const int *block_table,
                        const int *seqlens, void *o, float *lse, int B, int Hq, int Hkv,
                        int num_pages, int page_size, int max_pages, int d, float scale,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode step that allocates nothing and takes no workspace (no counterpart on the
 * pages: an addition of this library for callers that cannot hand it device scratch).
 * Some callers have no way to allocate device memory at the point of the call: plugins
 * that only receive device pointers from a host framework that owns the allocator,
 * serving loops that must not call cudaMalloc (it can synchronise the whole device and
 * stall other streams), or memory pools that are fully reserved up front.  This entry
 * point computes exactly what fa_decode computes, with the same arguments minus the
 * workspace; its split-KV partials go to a fixed scratch array that the library keeps in
 * device memory (FA_NOALLOC_SCRATCH_BYTES = 32 MiB on every GPU that loads libfa.so,
 * held until the process exits).
 *   - Limit: fa_decode_workspace_size(B, Hq, Nmax, d) must be <= FA_NOALLOC_SCRATCH_BYTES
 *     (e.g. B * Hq * ceil(Nmax / 256) * (d + 1) * 4 bytes, each part rounded up to 256);
 *     larger problems are rejected with FA_ERR_WORKSPACE and nothing is launched.
 *   - The first call on each device looks up the device address of the scratch array
 *     (cudaGetSymbolAddress) with that device current; make that first call before any
 *     stream capture begins.  The lookup is repeated when the device's context has
 *     changed since (after a cudaDeviceReset, whose module reload moves the array).
 *   - Every call, on every stream, shares the one scratch array and leaves its contents
 *     behind.  Nothing in it needs to start at zero (each call writes every partial it
 *     reads), but calls whose kernels overlap on the GPU race on it: order them (one
 *     stream, or events) just as calls that share one fa_decode workspace.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
FA_API int fa_decode_noalloc(const void *q, const void *kcache, const void *vcache,
                             const int *seqlens, void *o, float *lse, int B, int Hq, int Hkv,
                             int Nmax, int d, float scale, void *stream);

/*
 * Synchronises `stream`, then reads and clears the device error word.  Returns FA_OK,
 * FA_ERR_TIMEOUT, FA_ERR_DEVICE_ARG, FA_ERR_DEBUG_CHECK (debug builds), or FA_ERR_CUDA if
 * the synchronisation itself failed.
 */
FA_API int fa_get_error(void *stream);

/*
 * Limit, in nanoseconds, on any single pipeline wait inside the kernels launched from
 * now on by this process (default 2e9 = 2 s).  A wait that runs out records
 * FA_ERR_TIMEOUT, makes every role of the kernel stop at its next wait, frees the
 * kernel's tensor memory and returns.  0 restores the default.
 */
FA_API void fa_set_wait_limit_ns(unsigned long long ns);

/*
 * Self-test of the time-limit path: launches the prefill kernel on the given (valid)
 * arguments with its matrix-multiply warp told never to signal that a score tile is
 * ready, so the softmax warps' first wait must run out after the wait limit.  The
 * outputs are left unspecified; fa_get_error afterwards returns FA_ERR_TIMEOUT.
 */
FA_API int fa_fwd_selftest_timeout(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                            int causal, void *stream);

/*
 * Self-test of the time-limit path of the decode kernels: runs the decode of fa_decode
 * (k_scale = v_scale = NULL: bf16 caches) or of fa_decode_fp8 (both scales given: E4M3
 * caches) on the given (valid) arguments, with the producer warp of every split-kernel CTA
 * withholding its first copy, so that the consumers' first wait must run out after the
 * wait limit; the merge kernel that follows runs on whatever the partials hold.  The
 * outputs are left unspecified; fa_get_error afterwards returns FA_ERR_TIMEOUT.  Nothing
 * faults or hangs: every wait is bounded and every copy that was issued lands before the
 * kernel exits.
 */
FA_API int fa_decode_selftest_timeout(const void *q, const void *kcache, const void *vcache,
                                      const float *k_scale, const float *v_scale, const int *seqlens,
                                      void *o, float *lse, int B, int Hq, int Hkv, int Nmax, int d,
                                      float scale, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Build flags of this library: bit 0 set in the debug build (libfa_debug.so, compiled with
 * FA_DEBUG_CHECKS), whose kernels check every global-memory index they compute by hand
 * (outputs, decode partials, scales, q rows, block-table entries) against the size of its
 * buffer, skip the access on a failure and report FA_ERR_DEBUG_CHECK through fa_get_error.
 * The results are the release build's; only speed differs.
 */
FA_API int fa_build_flags(void);

/*
 * Self-test of the debug build's bounds checks: runs the prefill of fa_fwd on the given
 * (valid) arguments with every LSE index moved out of its buffer, so each LSE store must
 * fail its check and be skipped (lse is left as it was; O is computed normally);
 * fa_get_error afterwards returns FA_ERR_DEBUG_CHECK.  In a release build (no checks
 * compiled in) it returns FA_ERR_UNSUPPORTED and launches nothing.
 */
FA_API int fa_debug_selftest_bounds(const void *q, const void *k, const void *v, void *o, float *lse,
                                    int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                                    int causal, void *stream);

/* Human-readable name of a status code (static storage). */
FA_API const char *fa_status_str(int status);

/* Message of the last error returned on this host thread ("" if none). */
FA_API const char *fa_last_error_message(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */

/*
 * jetlong.h -- C ABI of libjetlong.so: Jet-Long dynamic bifocal RoPE attention
 * on NVIDIA B200 (sm_100a).
 *
 * Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
 * RoPE" (Tang, Wang, Gu, Han, Cai, 2026), as summarised on the pages
 * "Resumen Técnico: Jet-Long", "Jet-Long: Efficient Long-Context Extension with
 * Dynamic Bifocal RoPE" and "技術要約: Jet-Long" (Methodology sections 1 and 2)
 * and in the abstract of "Jet-Long : Extension efficace de long contexte avec
 * RoPE bifocale dynamique".
 *
 * Notation.  L: length of a sequence (prefill) or of the cache including the
 * current token (decode).  w_pretrained: pretraining window.  w0: local window.
 * G = max(1, ceil(L / w_pretrained)); f(x) = floor(x / G).  A (query i, key j)
 * pair with 0 <= i - j < w0 is LOCAL and scores <R(i)q, R(j)k>; any other
 * causal pair is REMOTE and scores <R(f(i))q, R(f(j))k>.  R(p) is RoPE in the
 * rotate-half pairing (c, c + d/2) with theta_c = rope_base^(-2c/d).
 * Query head h reads KV head floor(h / (Hq / Hkv)).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them.  bf16 tensors are token-major and contiguous.
 *    Every tensor pointer must be 16-byte aligned.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Nothing blocks the host except jl_sync_status.
 *  - Arguments are validated before anything is launched.  A failed check
 *    returns JL_ERR_INVALID (or JL_ERR_UNSUPPORTED for a valid but unbuilt
 *    shape) and sets a thread-local message readable with jl_last_error().
 *    A CUDA launch failure returns JL_ERR_CUDA.
 *  - Kernels never trap.  Every wait inside a kernel is bounded; a wait that
 *    runs out records JL_ERR_TIMEOUT in a device status word and the kernel
 *    returns.  jl_sync_status() reports and clears that word.
 *  - Only sm_100a is built.  There is no CPU fallback.
 */
#ifndef JETLONG_H
#define JETLONG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* jl_stream_t;

typedef enum {
  JL_OK = 0,
  JL_ERR_INVALID = 1,     /* bad argument; nothing was launched                */
  JL_ERR_UNSUPPORTED = 2, /* valid request for a shape this build does not have */
  JL_ERR_CUDA = 3,        /* a CUDA call failed                                 */
  JL_ERR_TIMEOUT = 4      /* a bounded in-kernel wait ran out                   */
} jl_status;

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char* jl_last_error(void);

/* G = max(1, ceil(L / w_pretrained)) (Methodology section 1, dynamic grouping).
 * Host helper; returns -1 if w_pretrained < 1 or L < 0. */
int64_t jl_group_size(int64_t L, int64_t w_pretrained);

/* Synchronises `stream`, then returns and clears the device status word:
 * JL_OK; JL_ERR_TIMEOUT if a bounded wait ran out; JL_ERR_INVALID if a cache
 * writer met a position outside the cache or the tables; JL_ERR_CUDA if the
 * synchronisation itself failed. */
jl_status jl_sync_status(jl_stream_t stream);

/*
 * Debug-bounds build (no counterpart in the paper; a diagnostic of this library).
 * Returns 1 in the library built with -DJL_DEBUG_BOUNDS (libjetlong_bounds.so),
 * 0 otherwise.  That build checks on the device every index its kernels derive
 * there -- RoPE table rows (remote rows < w_pretrained, every row < n_tab_rows),
 * TMA tile coordinates against the sequence or cache they belong to, cache and
 * page positions, workspace slots -- and records a failed check in the status
 * word instead of trapping; jl_sync_status() then returns JL_ERR_INVALID.  The
 * checks are compiled out of the normal build.
 */
int jl_debug_bounds_enabled(void);

/*
 * Single-launch decode build (no counterpart in the paper; a variant of this
 * library).  Returns 1 in the library built with -DJL_DECODE_LAST_CTA_MERGE=1
 * (libjetlong_lastcta.so), 0 otherwise.  In that build the head_dim-128 decode is
 * one kernel launch: the last split CTA of each (entry, KV head) merges the split
 * partials (see jl_bifocal_decode).  The normal build merges them in a second,
 * small kernel, which measured faster on B200: the last CTA's atomic ticket and
 * its reads of the other CTAs' partials are serial L2 round trips that cost more
 * than the kernel boundary they save.
 */
int jl_decode_single_launch_enabled(void);

/*
 * Failure-detection self-test (no counterpart in the paper; it exercises this
 * library's bounded waits).  Launches one thread that waits on a shared-memory
 * barrier that nothing ever completes, giving up after limit_cycles SM clock
 * cycles: the kernel records JL_ERR_TIMEOUT in the device status word and
 * returns normally, so no GPU fault or hang is involved.  A following
 * jl_sync_status() reports JL_ERR_TIMEOUT and clears the word; until then,
 * later launches of the attention kernels see the word and skip their work.
 * limit_cycles must be in [1000, 2000000000].
 */
jl_status jl_selftest_wait_timeout(int64_t limit_cycles, jl_stream_t stream);

/*
 * RoPE cos/sin tables (Methodology section 1, "Dynamic Bifocal RoPE": the local
 * window keeps classical RoPE at the true positions, and positions beyond it
 * are rotated at the remote positions f(x); both rotations are rows of this one
 * table).  Fills cos_out[p][c] = cos(p * theta_c) and
 * sin_out[p][c] = sin(p * theta_c) for p in [0, n_pos), c in [0, head_dim/2),
 * row-major fp32 [n_pos][head_dim/2].  Angles and cos/sin are computed in fp64
 * on the device and rounded to fp32 once.  Both the base rotations R(i) and the
 * remote rotations R(f(i)) read these rows (remote rows are < w_pretrained);
 * decode also reads rows n = x - f(x) for its correction rotations.
 * Requirements: n_pos >= 1, head_dim in {64, 128}, rope_base > 1.
 */
jl_status jl_rope_tables(float* cos_out, float* sin_out, int64_t n_pos, int32_t head_dim, double rope_base,
                         jl_stream_t stream);

/*
 * Scaled RoPE tables for the frequency-interpolation variant:
 * cos/sin(p * theta_c * freq_scale[c]), fp64 angle rounded to fp32 once.
 * freq_scale: HOST array of head_dim/2 positive factors (1/G for position
 * interpolation; a ramp between 1/s and 1 for a YaRN-style by-parts rule).
 */
jl_status jl_rope_tables_scaled(float* cos_out, float* sin_out, int64_t n_pos, int32_t head_dim, double rope_base,
                                const double* freq_scale, jl_stream_t stream);

/*
 * Frequency-interpolation variant of the remote window (the pages' ablation of
 * position aliasing against interpolation, Results; kernel only).  Local pairs
 * (0 <= i-j < w0) keep base RoPE from cos_tab/sin_tab; every other causal pair
 * scores <R'(i) q, R'(j) k> with R' read from cos_rem/sin_rem at the raw
 * positions (from jl_rope_tables_scaled).  No G or f: the caller's table sets
 * the compression.  Same layout, conventions, key workspace (its remote rows are
 * the interpolated rotation at the raw position) and kernel as
 * jl_bifocal_prefill; n_rem_rows >= max_seqlen.
 */
jl_status jl_interp_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                            int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                            int32_t w0, const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                            const float* cos_rem, const float* sin_rem, int64_t n_rem_rows, float softmax_scale,
                            void* out, float* lse, void* workspace, size_t workspace_bytes,
                            jl_stream_t stream);

/*
 * Bifocal prefill (Methodology section 2, inclusion-exclusion attention merge).
 * Computes, for every token i of every packed sequence and every query head,
 *   out = softmax_j(scale * s(i, j)) V   over j <= i, with s the routed score,
 * which equals the inclusion-exclusion merge of the three flash passes
 * (local/base + causal/remote - local/remote) on their log-sum-exp statistics.
 *
 *   q           bf16 [total_tokens][Hq][head_dim], RAW (not rotated)
 *   k, v        bf16 [total_tokens][Hkv][head_dim], k RAW
 *   cu_seqlens  device int32 [batch + 1], cu_seqlens[0] = 0, non-decreasing,
 *               cu_seqlens[batch] = total_tokens.  Positions restart at 0 in
 *               every sequence; G is computed per sequence from its length.
 *   max_seqlen  >= every sequence length (sizes the grid)
 *   w0          >= 0 (0 = no local window); w_pretrained >= 1
 *   cos_tab, sin_tab  from jl_rope_tables with n_tab_rows >= max_seqlen
 *   softmax_scale     <= 0 selects 1/sqrt(head_dim)
 *   out         bf16 [total_tokens][Hq][head_dim]
 *   lse         fp32 [Hq][total_tokens], natural-log log-sum-exp of the scaled
 *               routed scores of each row; may be NULL.
 *   workspace   NULL, or device scratch of at least
 *               jl_bifocal_prefill_workspace_size(total_tokens, Hkv, head_dim)
 *               bytes, 16-byte aligned, owned by the caller; its contents on
 *               entry do not matter.  With a workspace the keys are rotated once,
 *               before the attention kernel: the workspace receives R(j) k_j and,
 *               for sequences with G > 1, R(f(j)) k_j, and the kernel reads those
 *               for its local and remote visits.  Without one (NULL, 0) the
 *               kernel rotates each key tile on every visit (no global scratch).
 *               Both give the routed scores of the method; they may differ in the
 *               last bf16 bit of a rotated key (table row against a rotation
 *               recurrence), well inside the parity tolerance.
 * Supported: head_dim in {64, 128}; Hq % Hkv == 0; batch >= 0 (0 is a no-op).
 */
jl_status jl_bifocal_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                             int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv,
                             int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                             const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, jl_stream_t stream);

/* Bytes of the jl_bifocal_prefill / jl_plain_prefill workspace: two rotated key rows
 * (base and remote) per token and KV head, 2 * total_tokens * Hkv * head_dim * 2.
 * 0 for non-positive sizes. */
size_t jl_bifocal_prefill_workspace_size(int64_t total_tokens, int32_t Hkv, int32_t head_dim);

/*
 * jl_bifocal_prefill that also writes the base-RoPE KV cache the decode reads
 * (Methodology section 2: the cache holds the base keys R(j) k_j at their exact
 * positions and is never rewritten afterwards).  The attention result equals
 * jl_bifocal_prefill's; in addition, for every sequence b and position j:
 *   k_cache[b][j][h] = bf16(R(j) k_j), v_cache[b][j][h] = v_j
 *   k_cache, v_cache  bf16 [batch][cache_stride][Hkv][head_dim], caller-owned,
 *                     16-byte aligned; positions >= the sequence length are not written
 *   cache_stride      >= max_seqlen
 *   workspace, workspace_bytes  as for jl_bifocal_prefill.  With a workspace the
 *                     keys are rotated once into it, the attention is exactly
 *                     jl_bifocal_prefill's with a workspace, and the cache writer
 *                     (jl_kv_cache_fill) fills the cache.  Without one (NULL, 0)
 *                     the kernel rotates the keys itself and writes each key tile
 *                     while it holds it rotated for its own query block (one CTA
 *                     per KV head and block), so the cache costs no extra pass
 *                     over K; w0 = 0 has no base-position visit when G > 1, and
 *                     then the cache writer fills the cache after the attention.
 */
jl_status jl_bifocal_prefill_and_cache(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                       int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t Hq,
                                       int32_t Hkv, int32_t head_dim, int32_t w0, int32_t w_pretrained,
                                       const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                                       float softmax_scale, void* out, float* lse, void* k_cache, void* v_cache,
                                       int64_t cache_stride, void* workspace, size_t workspace_bytes,
                                       jl_stream_t stream);

/*
 * Chunked prefill against a base-RoPE cache (a prompt processed in pieces, or
 * a long continuation of a conversation).  Entry b already holds past_lens[b]
 * keys/values in the caches, and this chunk's n_b = cu_seqlens[b+1] -
 * cu_seqlens[b] tokens have been appended after them (jl_kv_cache_fill with
 * past_lens).  Each chunk query at absolute position i = past_lens[b] + r
 * attends to cached keys j <= i with the bifocal routing of the current length
 * L = past_lens[b] + n_b (G = max(1, ceil(L / w_pretrained)), Methodology
 * section 1).  Local keys are used as cached; remote keys get the correction
 * rotation R(f(j) - j) in shared memory, the query is rotated by R(f(i)) -- the
 * cache is never rewritten (Methodology section 2).  The result for a chunk
 * equals the rows past_lens[b] .. L-1 of a full jl_bifocal_prefill over the
 * first L tokens.
 *   q            bf16 [total_tokens][Hq][head_dim], the chunks' RAW queries
 *   cu_seqlens   device int32 [batch + 1] over the chunks; max_seqlen >= every n_b
 *   past_lens    device int32 [batch]; max_total >= every past_lens[b] + n_b
 *   k_cache, v_cache  bf16 [batch][cache_stride][Hkv][head_dim], read only
 *   out, lse     as for jl_bifocal_prefill, over the chunks' packed tokens
 * Requirements: cache_stride >= max_total, n_tab_rows >= max_total,
 * batch * cache_stride < 2^31.
 */
jl_status jl_bifocal_prefill_chunk(const void* q, const int32_t* cu_seqlens, const int32_t* past_lens, int32_t batch,
                                   int64_t total_tokens, int32_t max_seqlen, int32_t max_total, const void* k_cache,
                                   const void* v_cache, int64_t cache_stride, int32_t Hq, int32_t Hkv,
                                   int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                                   const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out,
                                   float* lse, jl_stream_t stream);

/*
 * The pages' literal realisation of the bifocal prefill (Methodology section 2):
 * three flash passes -- pass 1 local window (0 <= i-j < w0) with base
 * positions, pass 2 full causal with remote positions, pass 3 local window
 * with remote positions -- each writing its output and log-sum-exp, then the
 * inclusion-exclusion merge
 *   M = max(lse1, lse2), a_p = e^(lse_p - M),
 *   out = (a1 O1 + a2 O2 - a3 O3) / (a1 + a2 - a3), lse = M + ln(a1 + a2 - a3).
 * Same arguments and result as jl_bifocal_prefill, plus a caller workspace of
 * jl_bifocal_prefill_three_pass_workspace_size() bytes that afterwards holds
 * the passes: O_p fp32 [3][total_tokens][Hq][head_dim] (fp32 because the merge
 * subtracts pass 3 from pass 2), then lse_p fp32 [3][Hq][total_tokens].  It does more work than the fused kernel (pass 3
 * repeats the window) and exists to run the merge as written.
 */
jl_status jl_bifocal_prefill_three_pass(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                        int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t Hq,
                                        int32_t Hkv, int32_t head_dim, int32_t w0, int32_t w_pretrained,
                                        const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                                        float softmax_scale, void* out, float* lse, void* workspace,
                                        size_t workspace_bytes, jl_stream_t stream);
size_t jl_bifocal_prefill_three_pass_workspace_size(int64_t total_tokens, int32_t Hq, int32_t head_dim);

/* Plain causal RoPE prefill (every causal pair LOCAL), built from the same
 * kernel; the comparator for bifocal prefill.  Same conventions, workspace
 * included (only its base rows are written). */
jl_status jl_plain_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                           int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                           const float* cos_tab, const float* sin_tab, int64_t n_tab_rows, float softmax_scale,
                           void* out, float* lse, void* workspace, size_t workspace_bytes, jl_stream_t stream);

/*
 * Single-query bifocal decode with the on-the-fly correction rotation
 * (Methodology section 2).  One new token per batch entry b sits at position
 * i = seqlens[b] - 1 of a base-RoPE KV cache.
 *
 *   q            bf16 [B][Hq][head_dim], ALREADY rotated by R(i) (base RoPE)
 *   k_cache      bf16 [B][cache_stride][Hkv][head_dim]: keys rotated by R(j)
 *                at their absolute positions j; the caller has already
 *                appended the current token.  READ ONLY: never written.
 *   v_cache      bf16 [B][cache_stride][Hkv][head_dim], read only
 *   seqlens      device int32 [B], 1 <= seqlens[b] <= max_seqlen
 *   max_seqlen   <= cache_stride; sizes the split-K grid (the call does not
 *                read seqlens on the host, so it can be captured in a CUDA
 *                graph and replayed across G changes)
 *   cos_tab, sin_tab  from jl_rope_tables, n_tab_rows >= max_seqlen
 *   out          bf16 [B][Hq][head_dim]
 *   lse          fp32 [B][Hq] natural-log LSE; may be NULL
 *   workspace    device scratch of at least jl_bifocal_decode_workspace_size()
 *                bytes, 16-byte aligned, owned by the caller; its contents on
 *                entry do not matter; calls sharing it must not overlap.
 * The keys are split across CTAs; a second, small kernel merges the split
 * partials.  In the single-launch build (jl_decode_single_launch_enabled) the
 * head_dim-128 call is one kernel launch instead: the last CTA of each (entry,
 * KV head) to finish merges them.  It is found through two counter words per
 * (entry, KV head) in the workspace: a count that the last CTA puts back to a
 * marked zero, and, for a workspace whose count word is not marked yet, a second
 * count tagged with a value unique to the call (a word with another tag counts
 * as zero).  So the workspace needs no clearing in either build, and a CUDA
 * graph replaying the call finds the count clear.  A CTA that gives up on a
 * bounded wait still counts.  In both builds out and lse are written as NaN when
 * a kernel of the call gave up.
 * Local keys (i - j < w0) score q . k_cache[j] unchanged; remote keys score
 * (R(f(i) - i) q) . (R(f(j) - j) k_cache[j]), both corrections applied in
 * registers.  G = max(1, ceil(seqlens[b] / w_pretrained)) is computed on the
 * device every call.
 * Supported: head_dim 128 (tensor cores) or 64 (CUDA cores), 1 to 16 query
 * heads per KV head; more returns JL_ERR_UNSUPPORTED.
 */
jl_status jl_bifocal_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                            int32_t B, int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv,
                            int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                            const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, jl_stream_t stream);

/* Bytes of workspace jl_bifocal_decode / jl_plain_decode need for these sizes,
 * whatever the KV-head count: the split count depends on Hkv (as many splits as
 * fit one wave of CTAs), so the size is the largest over every Hkv dividing Hq.
 * 0 for non-positive sizes. */
size_t jl_bifocal_decode_workspace_size(int32_t B, int32_t Hq, int32_t head_dim, int32_t max_seqlen);

/* Plain causal decode (no correction rotation), built from the same kernel;
 * the comparator for the decode overhead.  Same conventions. */
jl_status jl_plain_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                          int32_t B, int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv,
                          int32_t head_dim, const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                          float softmax_scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                          jl_stream_t stream);

/*
 * Base-RoPE KV cache writers (Methodology section 2: the cache holds the
 * un-compressed base keys R(j) k_j at their absolute positions and is written
 * once per token; the bifocal decode only reads it).
 *
 * jl_kv_cache_fill: for every token t of packed sequence b (position
 * p = past_lens[b] + t - cu_seqlens[b]), k_cache[b][p] = R(p) k[t] (fp32 math,
 * rounded to bf16) and v_cache[b][p] = v[t], for every KV head.
 *   k, v        bf16 [total_tokens][Hkv][head_dim], k RAW
 *   cu_seqlens  device int32 [batch + 1] as for jl_bifocal_prefill
 *   past_lens   device int32 [batch]: tokens already in each entry (a prompt
 *               continued in chunks); NULL means 0
 *   k_cache, v_cache  bf16 [batch][cache_stride][Hkv][head_dim]
 * A position >= cache_stride or >= n_tab_rows is skipped and reported by
 * jl_sync_status() as JL_ERR_INVALID (the lengths live on the device).
 */
jl_status jl_kv_cache_fill(const void* k, const void* v, const int32_t* cu_seqlens, const int32_t* past_lens,
                           int32_t batch, int64_t total_tokens, int32_t Hkv, int32_t head_dim, const float* cos_tab,
                           const float* sin_tab, int64_t n_tab_rows, void* k_cache, void* v_cache,
                           int64_t cache_stride, jl_stream_t stream);

/*
 * One decode step's inputs: entry b's new token sits at i = seqlens[b] - 1
 * (seqlens already counts it).  q_out[b] = R(i) q[b] (the base-rotated query
 * jl_bifocal_decode takes), k_cache[b][i] = R(i) k[b], v_cache[b][i] = v[b].
 *   q      bf16 [B][Hq][head_dim] raw;  k, v  bf16 [B][Hkv][head_dim], k raw
 *   q_out  bf16 [B][Hq][head_dim];  caches as for jl_bifocal_decode (written
 *          only at position i)
 * Out-of-range positions are skipped and reported like jl_kv_cache_fill.
 */
jl_status jl_decode_append(const void* q, const void* k, const void* v, const int32_t* seqlens, int32_t B,
                           int32_t Hq, int32_t Hkv, int32_t head_dim, const float* cos_tab, const float* sin_tab,
                           int64_t n_tab_rows, void* q_out, void* k_cache, void* v_cache, int64_t cache_stride,
                           jl_stream_t stream);

/*
 * Paged caches.  The caches are a pool of pages, bf16 [num_pages][page_size]
 * [Hkv][head_dim] (k_pool base-RoPE, v_pool values), and entry b's position j
 * lives in page block_table[b * max_pages + j / page_size] at row
 * j % page_size.  block_table: device int32 [B][max_pages].  The writers skip
 * and report (jl_sync_status: JL_ERR_INVALID) a page index outside
 * [0, num_pages); the decode reads such a page as zeros.  page_size must be a
 * multiple of 128 for the decode (a 128-key tile never crosses a page).
 */
jl_status jl_bifocal_decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                                  const int32_t* seqlens, int32_t B, int32_t max_pages, int32_t page_size,
                                  int32_t num_pages, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                                  int32_t w0, int32_t w_pretrained, const float* cos_tab, const float* sin_tab,
                                  int64_t n_tab_rows, float softmax_scale, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, jl_stream_t stream);
jl_status jl_kv_cache_fill_paged(const void* k, const void* v, const int32_t* cu_seqlens, const int32_t* past_lens,
                                 int32_t batch, int64_t total_tokens, int32_t Hkv, int32_t head_dim,
                                 const float* cos_tab, const float* sin_tab, int64_t n_tab_rows, void* k_pool,
                                 void* v_pool, const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                 int32_t num_pages, jl_stream_t stream);
jl_status jl_decode_append_paged(const void* q, const void* k, const void* v, const int32_t* seqlens, int32_t B,
                                 int32_t Hq, int32_t Hkv, int32_t head_dim, const float* cos_tab,
                                 const float* sin_tab, int64_t n_tab_rows, void* q_out, void* k_pool, void* v_pool,
                                 const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                 int32_t num_pages, jl_stream_t stream);

/*
 * jl_bifocal_decode without a caller workspace.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory, for
 * example an engine plugin that is handed only its input and output buffers,
 * or a serving loop that forbids cudaMalloc once it is running.  It computes
 * exactly what jl_bifocal_decode computes and takes the same arguments minus
 * the workspace.  It allocates nothing: the split-K scratch is a file-scope
 * device array of jl_bifocal_decode_noalloc_scratch_bytes() bytes (8 MiB) that
 * every GPU loading the library holds until the process exits.
 *  - Sizes whose scratch would exceed that maximum (B * n_split * Hq *
 *    (head_dim + 2) * 4 bytes of partials plus B * Hq * 16 bytes of merge
 *    counters, see jl_bifocal_decode_workspace_size) return
 *    JL_ERR_INVALID with a message; B = 1, Hq = 32, head_dim = 128 fits up to
 *    max_seqlen = 131072.
 *  - The stream, the current device and q must be on one device; a mismatch
 *    returns JL_ERR_INVALID (the array's address is only valid on its own
 *    device).  Each call outside stream capture looks the address up again with
 *    cudaGetSymbolAddress, so a reset device context is picked up; a call made
 *    during a capture uses the address from the last uncaptured call on that
 *    device, so make the first call on a device before any stream capture.
 *  - If a kernel of the call gives up on a bounded wait (jl_sync_status then
 *    reports JL_ERR_TIMEOUT), out and lse are written as NaN.
 *  - All calls on a device share the one array, and it keeps whatever the last
 *    call left there (nothing in it needs to start at zero).  Calls whose
 *    executions overlap on the GPU -- on different streams, or from different
 *    host threads -- race on it: order them on one stream or use
 *    jl_bifocal_decode with separate workspaces.
 */
jl_status jl_bifocal_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                                    int32_t B, int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv,
                                    int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                                    const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out,
                                    float* lse, jl_stream_t stream);

/* Bytes of the static scratch behind jl_bifocal_decode_noalloc (per device). */
size_t jl_bifocal_decode_noalloc_scratch_bytes(void);

#ifdef __cplusplus
}
#endif
#endif /* JETLONG_H */

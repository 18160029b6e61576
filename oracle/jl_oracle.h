/*
 * jl_oracle.h -- CPU oracle for Jet-Long dynamic bifocal RoPE attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously correct fp64
 * restatement of what the attention path computes.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or constant with the CUDA library, and it never reads a
 * value produced by the CUDA library.
 *
 * Sources (the paper "Jet-Long: Efficient Long-Context Extension with Dynamic
 * Bifocal RoPE", Tang, Wang, Gu, Han, Cai, 2026, as summarised on the pages
 * "Resumen Técnico: Jet-Long", "Jet-Long: Efficient Long-Context Extension with
 * Dynamic Bifocal RoPE", "技術要約: Jet-Long" and "Jet-Long : Extension efficace
 * de long contexte avec RoPE bifocale dynamique"):
 *   - Methodology, section 1 "Dynamic Bifocal RoPE": the local window of w0
 *     keeps classical RoPE; positions beyond it use the remote map
 *     f(x) = floor(x / G) with G = max(1, ceil(L / w_pretrained)).
 *   - Methodology, section 2 "Inference efficiency": the on-the-fly correction
 *     rotation applied to the active query and the cached base keys; the
 *     inclusion-exclusion merge of three flash-style passes on LogSumExp
 *     statistics, which yields the exact distance-routed output.
 *
 * Readings of points the pages leave open:
 *   C1 local  <=>  0 <= i - j < w0   (distance, strict; w0 keys incl. self)
 *   C2 the remote score rotates the query by f(i) and the key by f(j)
 *   C3 positions are 0-based per sequence; L is the sequence length (prefill)
 *      or the cache length including the current token (decode: query at L-1)
 *   C4 rotate-half pairing (c, c + d/2), theta_c = base^(-2c/d), scale 1/sqrt(d)
 *   C6 query head h reads KV head floor(h / (Hq / Hkv))
 *   C7 an empty pass has lse = -inf and contributes nothing
 *
 * Every function computes in fp64.  Inputs are read through jlo_view, which
 * accepts fp64, fp32 or raw bf16 bit patterns; bf16 and fp32 values are upcast
 * to fp64 exactly.  Return value: 0 on success, negative on invalid arguments.
 *
 * Parity status: every function here is pinned by the CPU test suite (closed
 * forms, invariants, library special cases, brute force); see the pins listed
 * beside each test.
 */
#ifndef JL_ORACLE_H
#define JL_ORACLE_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

enum { JLO_F64 = 0, JLO_BF16 = 1, JLO_F32 = 2 };

/* Strided view of a [positions][heads][d] tensor; the channel stride is 1.
 * Element (pos, head, c) lives at data[pos*stride_pos + head*stride_head + c]. */
typedef struct {
  const void* data;
  int64_t stride_pos;
  int64_t stride_head;
  int32_t dtype;
  int32_t pad_;
} jlo_view;

/* G = max(1, ceil(L / w_pretrained)) in integer arithmetic. */
int64_t jlo_group_size(int64_t L, int64_t w_pretrained);
/* f(x) = floor(x / G) for x >= 0. */
int64_t jlo_remote_pos(int64_t x, int64_t G);
/* theta_c = base^(-2c/d), c = 0..d/2-1. */
void jlo_inv_freq(int32_t d, double rope_base, double* theta);
/* cos/sin(p * theta_c) for p = 0..n_pos-1, row-major [n_pos][d/2]. */
void jlo_rope_cos_sin(int64_t n_pos, int32_t d, double rope_base, double* cos_out, double* sin_out);
/* y = R(pos) x, rotate-half convention; pos may be negative (R(-n) = R(n)^T). */
void jlo_rotate(const double* x, int32_t d, int64_t pos, double rope_base, double* y);

/* y_r = R(pos_r) x_r for n rows of width d (x, y: [n][d] fp64; pos may be negative). */
void jlo_rotate_rows(const double* x, const int64_t* pos, int64_t n, int32_t d, double rope_base, double* y);

/*
 * Direct definition for one sequence of length L.  For each selected row r
 * (query position i = row_pos[r], query head h = row_head[r]) build the
 * explicit routed score row over j = 0..L-1 against KV head floor(h*Hkv/Hq):
 *     mask(i,j) = MASKED        if j > i
 *               = LOCAL         if 0 <= i - j < w0
 *               = REMOTE        otherwise
 *     s(i,j)    = scale * <R(i) q_i, R(j) k_j>          (LOCAL)
 *               = scale * <R(f(i)) q_i, R(f(j)) k_j>    (REMOTE)
 * and return lse_r = log sum_j exp s(i,j) (natural log) and
 * out_r = sum_j exp(s(i,j) - lse_r) v_j.  q, k, v hold RAW (un-rotated)
 * vectors.  G comes from L.  w0 may be 0 (no local window) or >= L.
 * plain != 0 routes every causal pair LOCAL (plain causal RoPE attention).
 * out: [n_rows][d], lse: [n_rows].
 */
int jlo_bifocal_rows(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d,
                     int32_t n_q_heads, int32_t n_kv_heads,
                     const int64_t* row_pos, const int32_t* row_head, int64_t n_rows,
                     int64_t w0, int64_t w_pretrained, double rope_base, double scale, int plain,
                     double* out, double* lse);

/*
 * Frequency-interpolation variant of the remote window (the pages' ablation:
 * interpolation, YaRN-style, against position aliasing).  Local pairs
 * (0 <= i - j < w0) keep base RoPE; every other causal pair scores
 *     scale * < R'(i) q_i , R'(j) k_j >,   R'(p): angle p * theta_c * lambda_c
 * with caller-given per-frequency factors lambda [d/2] (lambda_c = 1/G is
 * position interpolation; a ramp between 1/s and 1 is YaRN's by-parts rule).
 * No G or f is involved.  Same layout and outputs as jlo_bifocal_rows.
 */
int jlo_interp_rows(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d, int32_t n_q_heads,
                    int32_t n_kv_heads, const int64_t* row_pos, const int32_t* row_head, int64_t n_rows,
                    int64_t w0, double rope_base, const double* lambda, double scale, double* out, double* lse);

/*
 * The pages' own realisation: three softmax passes merged by inclusion-
 * exclusion on their LogSumExp statistics.
 *   pass 1: local window (0 <= i-j < w0), base positions
 *   pass 2: full causal (j <= i), remote positions
 *   pass 3: local window, remote positions (subtracted)
 *   M = max(lse1, lse2); Z = e^(lse1-M) + e^(lse2-M) - e^(lse3-M)
 *   out = (e^(lse1-M) o1 + e^(lse2-M) o2 - e^(lse3-M) o3) / Z; lse = M + log Z
 * Same arguments as jlo_bifocal_rows; pass_lse [n_rows][3] may be NULL.
 */
int jlo_bifocal_rows_three_pass(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d,
                                int32_t n_q_heads, int32_t n_kv_heads,
                                const int64_t* row_pos, const int32_t* row_head, int64_t n_rows,
                                int64_t w0, int64_t w_pretrained, double rope_base, double scale,
                                double* out, double* lse, double* pass_lse);

/*
 * Decode step on a base-RoPE cache of length L (the current token included):
 * the query sits at i = L-1 and G = max(1, ceil(L / w_pretrained)).
 * q_tilde: query heads already rotated by R(L-1) (head h at
 * data[h*stride_head]; stride_pos is ignored).  k_cache: keys already rotated
 * by R(j) at their absolute positions j; v_cache: values.  Local keys use the
 * cached representation unchanged; remote keys use the correction rotations
 *     s = scale * < R(f(i) - i) q_tilde , R(f(j) - j) k_tilde_j >.
 * plain != 0 makes every key local (plain causal decode).
 * out: [n_q_heads][d], lse: [n_q_heads].
 */
int jlo_decode_step(jlo_view q_tilde, jlo_view k_cache, jlo_view v_cache, int64_t L, int32_t d,
                    int32_t n_q_heads, int32_t n_kv_heads,
                    int64_t w0, int64_t w_pretrained, double rope_base, double scale, int plain,
                    double* out, double* lse);

/* Threads the oracle's parallel loops use (OpenMP), for reporting. */
int jlo_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif

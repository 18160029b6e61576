/*
 * jl_oracle.c -- CPU oracle for Jet-Long dynamic bifocal RoPE attention.
 *
 * TEST INFRASTRUCTURE ONLY (see jl_oracle.h).  Plain C99 + OpenMP, fp64.
 * The only precomputation is of quantities the definition names directly:
 * cos/sin(p*theta_c) and the rotated vectors R(p)x.  There is no tiling,
 * blocking, online softmax or fusion: every score row is materialised in full
 * with its explicit routing mask, then normalised with a max-subtracted
 * log-sum-exp.
 */
#include "jl_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { MASKED = 0, LOCAL = 1, REMOTE = 2 };

/* ---- element access -------------------------------------------------------- */

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double view_at(const jlo_view* t, int64_t pos, int64_t head, int64_t c) {
  int64_t off = pos * t->stride_pos + head * t->stride_head + c;
  switch (t->dtype) {
    case JLO_BF16: return bf16_bits_to_double(((const uint16_t*)t->data)[off]);
    case JLO_F32: return (double)((const float*)t->data)[off];
    default: return ((const double*)t->data)[off];
  }
}

static void view_row(const jlo_view* t, int64_t pos, int64_t head, int32_t d, double* x) {
  for (int32_t c = 0; c < d; ++c) x[c] = view_at(t, pos, head, c);
}

/* ---- position map (Methodology section 1, equations for G and f) ---------- */

int64_t jlo_group_size(int64_t L, int64_t w_pretrained) {
  if (w_pretrained <= 0) return -1;
  int64_t g = (L + w_pretrained - 1) / w_pretrained; /* ceil for L >= 0 */
  return g < 1 ? 1 : g;
}

int64_t jlo_remote_pos(int64_t x, int64_t G) { return x / G; /* x >= 0, G >= 1: floor */ }

/* ---- RoPE (rotate-half pairing (c, c + d/2)) ------------------------------- */

void jlo_inv_freq(int32_t d, double rope_base, double* theta) {
  for (int32_t c = 0; c < d / 2; ++c) theta[c] = pow(rope_base, -2.0 * (double)c / (double)d);
}

void jlo_rope_cos_sin(int64_t n_pos, int32_t d, double rope_base, double* cos_out, double* sin_out) {
  int32_t h = d / 2;
  double* theta = (double*)malloc(sizeof(double) * (size_t)h);
  jlo_inv_freq(d, rope_base, theta);
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < n_pos; ++p)
    for (int32_t c = 0; c < h; ++c) {
      double a = (double)p * theta[c];
      cos_out[p * h + c] = cos(a);
      sin_out[p * h + c] = sin(a);
    }
  free(theta);
}

/* y_c = x_c cos(p t_c) - x_{c+h} sin(p t_c);  y_{c+h} = x_{c+h} cos(p t_c) + x_c sin(p t_c) */
static void rotate_with(const double* x, int32_t d, const double* cs, const double* sn, double sign,
                        double* y) {
  int32_t h = d / 2;
  for (int32_t c = 0; c < h; ++c) {
    double co = cs[c], si = sign * sn[c];
    double a = x[c], b = x[c + h];
    y[c] = a * co - b * si;
    y[c + h] = b * co + a * si;
  }
}

void jlo_rotate(const double* x, int32_t d, int64_t pos, double rope_base, double* y) {
  int32_t h = d / 2;
  double* theta = (double*)malloc(sizeof(double) * (size_t)h * 3);
  double* cs = theta + h;
  double* sn = cs + h;
  jlo_inv_freq(d, rope_base, theta);
  int64_t n = pos < 0 ? -pos : pos;
  for (int32_t c = 0; c < h; ++c) {
    double a = (double)n * theta[c];
    cs[c] = cos(a);
    sn[c] = sin(a);
  }
  rotate_with(x, d, cs, sn, pos < 0 ? -1.0 : 1.0, y);
  free(theta);
}

void jlo_rotate_rows(const double* x, const int64_t* pos, int64_t n, int32_t d, double rope_base, double* y) {
  int32_t h = d / 2;
  double* theta = (double*)malloc(sizeof(double) * (size_t)h);
  jlo_inv_freq(d, rope_base, theta);
#pragma omp parallel
  {
    double* cs = (double*)malloc(sizeof(double) * (size_t)h * 2);
    double* sn = cs + h;
#pragma omp for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
      int64_t m = pos[r] < 0 ? -pos[r] : pos[r];
      for (int32_t c = 0; c < h; ++c) {
        double a = (double)m * theta[c];
        cs[c] = cos(a);
        sn[c] = sin(a);
      }
      rotate_with(x + r * d, d, cs, sn, pos[r] < 0 ? -1.0 : 1.0, y + r * d);
    }
    free(cs);
  }
  free(theta);
}

static double dot(const double* a, const double* b, int32_t d) {
  double s = 0.0;
  for (int32_t c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

/* Softmax over the unmasked entries of one explicit score row; writes out/lse. */
static void softmax_row(const double* s, const unsigned char* mask, int64_t n, const jlo_view* v,
                        int64_t kv_head, int32_t d, double* out, double* lse) {
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j)
    if (mask[j] != MASKED && s[j] > m) m = s[j];
  for (int32_t c = 0; c < d; ++c) out[c] = 0.0;
  if (m == -INFINITY) { /* empty set: lse = -inf, out = 0 */
    *lse = -INFINITY;
    return;
  }
  double z = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    if (mask[j] == MASKED) continue;
    double p = exp(s[j] - m);
    z += p;
    for (int32_t c = 0; c < d; ++c) out[c] += p * view_at(v, j, kv_head, c);
  }
  for (int32_t c = 0; c < d; ++c) out[c] /= z;
  *lse = m + log(z);
}

/* Rotated keys R(j) k_j and R(f(j)) k_j for j = 0..n-1 of one KV head. */
static void rotate_keys(const jlo_view* k, int64_t kv_head, int64_t n, int32_t d, int64_t G,
                        const double* cs, const double* sn, double* kb, double* kr) {
  int32_t h = d / 2;
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
      view_row(k, j, kv_head, d, x);
      rotate_with(x, d, cs + j * h, sn + j * h, 1.0, kb + j * d);
      int64_t fj = jlo_remote_pos(j, G);
      rotate_with(x, d, cs + fj * h, sn + fj * h, 1.0, kr + j * d);
    }
    free(x);
  }
}

static int check_common(int64_t L, int32_t d, int32_t hq, int32_t hkv, int64_t w0, int64_t w_pre) {
  if (L < 0 || d <= 0 || (d & 1) || hq <= 0 || hkv <= 0 || hq % hkv || w0 < 0 || w_pre < 1) return -1;
  return 0;
}

/* Shared driver for the direct definition (mode 0) and the three-pass merge (mode 1). */
static int rows_impl(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d, int32_t hq, int32_t hkv,
                     const int64_t* row_pos, const int32_t* row_head, int64_t n_rows, int64_t w0,
                     int64_t w_pre, double base, double scale, int plain, int mode, double* out,
                     double* lse, double* pass_lse) {
  if (check_common(L, d, hq, hkv, w0, w_pre)) return -1;
  int64_t imax = -1;
  for (int64_t r = 0; r < n_rows; ++r) {
    if (row_pos[r] < 0 || row_pos[r] >= L || row_head[r] < 0 || row_head[r] >= hq) return -2;
    if (row_pos[r] > imax) imax = row_pos[r];
  }
  if (n_rows == 0) return 0;
  const int32_t h = d / 2;
  const int64_t npos = imax + 1;
  const int64_t G = plain ? 1 : jlo_group_size(L, w_pre);
  const int32_t group = hq / hkv;

  double* cs = (double*)malloc(sizeof(double) * (size_t)(npos * h));
  double* sn = (double*)malloc(sizeof(double) * (size_t)(npos * h));
  double* kb = (double*)malloc(sizeof(double) * (size_t)(npos * d));
  double* kr = (double*)malloc(sizeof(double) * (size_t)(npos * d));
  if (!cs || !sn || !kb || !kr) {
    free(cs); free(sn); free(kb); free(kr);
    return -3;
  }
  jlo_rope_cos_sin(npos, d, base, cs, sn);

  for (int32_t kvh = 0; kvh < hkv; ++kvh) {
    int any = 0;
    for (int64_t r = 0; r < n_rows && !any; ++r) any = (row_head[r] / group == kvh);
    if (!any) continue;
    rotate_keys(&k, kvh, npos, d, G, cs, sn, kb, kr);

#pragma omp parallel
    {
      double* x = (double*)malloc(sizeof(double) * (size_t)d * 3);
      double* qb = x + d;
      double* qr = qb + d;
      double* s = (double*)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1) * 2);
      double* s2 = s + npos;
      unsigned char* mask = (unsigned char*)malloc((size_t)(npos > 0 ? npos : 1) * 2);
      unsigned char* mask2 = mask + npos;
      double* o = (double*)malloc(sizeof(double) * (size_t)d * 3);
#pragma omp for schedule(dynamic, 1)
      for (int64_t r = 0; r < n_rows; ++r) {
        if (row_head[r] / group != kvh) continue;
        const int64_t i = row_pos[r];
        const int64_t fi = jlo_remote_pos(i, G);
        view_row(&q, i, row_head[r], d, x);
        rotate_with(x, d, cs + i * h, sn + i * h, 1.0, qb);
        rotate_with(x, d, cs + fi * h, sn + fi * h, 1.0, qr);
        if (mode == 0) {
          /* explicit routed score row with its mask; keys beyond the largest
             selected position are MASKED for every selected row, so the row
             stops there */
          for (int64_t j = 0; j < npos; ++j) {
            int64_t dist = i - j;
            if (dist < 0) mask[j] = MASKED;
            else if (plain || dist < w0) mask[j] = LOCAL;
            else mask[j] = REMOTE;
            if (mask[j] == LOCAL) s[j] = scale * dot(qb, kb + j * d, d);
            else if (mask[j] == REMOTE) s[j] = scale * dot(qr, kr + j * d, d);
            else s[j] = 0.0;
          }
          softmax_row(s, mask, npos, &v, kvh, d, out + r * d, lse + r);
        } else {
          /* three passes: o[0..d) pass 1, o[d..2d) pass 2, o[2d..3d) pass 3 */
          double l[3];
          for (int64_t j = 0; j < npos; ++j) { /* pass 1: window, base */
            int64_t dist = i - j;
            mask[j] = (dist >= 0 && dist < w0) ? LOCAL : MASKED;
            s[j] = mask[j] ? scale * dot(qb, kb + j * d, d) : 0.0;
          }
          softmax_row(s, mask, npos, &v, kvh, d, o, &l[0]);
          for (int64_t j = 0; j < npos; ++j) { /* pass 2: causal, remote */
            mask2[j] = (i - j >= 0) ? REMOTE : MASKED;
            s2[j] = mask2[j] ? scale * dot(qr, kr + j * d, d) : 0.0;
          }
          softmax_row(s2, mask2, npos, &v, kvh, d, o + d, &l[1]);
          for (int64_t j = 0; j < npos; ++j) /* pass 3: window, remote (same set as pass 1) */
            s[j] = mask[j] ? scale * dot(qr, kr + j * d, d) : 0.0;
          softmax_row(s, mask, npos, &v, kvh, d, o + 2 * d, &l[2]);
          double M = l[0] > l[1] ? l[0] : l[1];
          double a1 = l[0] == -INFINITY ? 0.0 : exp(l[0] - M);
          double a2 = l[1] == -INFINITY ? 0.0 : exp(l[1] - M);
          double a3 = l[2] == -INFINITY ? 0.0 : exp(l[2] - M);
          double Z = a1 + a2 - a3;
          for (int32_t c = 0; c < d; ++c) out[r * d + c] = (a1 * o[c] + a2 * o[d + c] - a3 * o[2 * d + c]) / Z;
          lse[r] = M + log(Z);
          if (pass_lse) {
            pass_lse[r * 3 + 0] = l[0];
            pass_lse[r * 3 + 1] = l[1];
            pass_lse[r * 3 + 2] = l[2];
          }
        }
      }
      free(x); free(s); free(mask); free(o);
    }
  }
  free(cs); free(sn); free(kb); free(kr);
  return 0;
}

int jlo_bifocal_rows(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d, int32_t n_q_heads,
                     int32_t n_kv_heads, const int64_t* row_pos, const int32_t* row_head, int64_t n_rows,
                     int64_t w0, int64_t w_pretrained, double rope_base, double scale, int plain,
                     double* out, double* lse) {
  return rows_impl(q, k, v, L, d, n_q_heads, n_kv_heads, row_pos, row_head, n_rows, w0, w_pretrained,
                   rope_base, scale, plain, 0, out, lse, NULL);
}

int jlo_bifocal_rows_three_pass(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d,
                                int32_t n_q_heads, int32_t n_kv_heads, const int64_t* row_pos,
                                const int32_t* row_head, int64_t n_rows, int64_t w0,
                                int64_t w_pretrained, double rope_base, double scale, double* out,
                                double* lse, double* pass_lse) {
  return rows_impl(q, k, v, L, d, n_q_heads, n_kv_heads, row_pos, row_head, n_rows, w0, w_pretrained,
                   rope_base, scale, 0, 1, out, lse, pass_lse);
}

/* ---- frequency-interpolation variant (Results, ablation: aliasing vs interpolation) ---- */

int jlo_interp_rows(jlo_view q, jlo_view k, jlo_view v, int64_t L, int32_t d, int32_t hq, int32_t hkv,
                    const int64_t* row_pos, const int32_t* row_head, int64_t n_rows, int64_t w0, double base,
                    const double* lambda, double scale, double* out, double* lse) {
  if (check_common(L, d, hq, hkv, w0, 1) || !lambda) return -1;
  int64_t imax = -1;
  for (int64_t r = 0; r < n_rows; ++r) {
    if (row_pos[r] < 0 || row_pos[r] >= L || row_head[r] < 0 || row_head[r] >= hq) return -2;
    if (row_pos[r] > imax) imax = row_pos[r];
  }
  if (n_rows == 0) return 0;
  const int32_t h = d / 2;
  const int64_t npos = imax + 1;
  const int32_t group = hq / hkv;
  double* theta = (double*)malloc(sizeof(double) * (size_t)h);
  double* cb = (double*)malloc(sizeof(double) * (size_t)(npos * h));  /* base cos/sin */
  double* sb = (double*)malloc(sizeof(double) * (size_t)(npos * h));
  double* ci = (double*)malloc(sizeof(double) * (size_t)(npos * h));  /* interpolated cos/sin */
  double* si = (double*)malloc(sizeof(double) * (size_t)(npos * h));
  double* kb = (double*)malloc(sizeof(double) * (size_t)(npos * d));
  double* ki = (double*)malloc(sizeof(double) * (size_t)(npos * d));
  if (!theta || !cb || !sb || !ci || !si || !kb || !ki) {
    free(theta); free(cb); free(sb); free(ci); free(si); free(kb); free(ki);
    return -3;
  }
  jlo_inv_freq(d, base, theta);
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < npos; ++p)
    for (int32_t c = 0; c < h; ++c) {
      cb[p * h + c] = cos((double)p * theta[c]);
      sb[p * h + c] = sin((double)p * theta[c]);
      ci[p * h + c] = cos((double)p * theta[c] * lambda[c]);
      si[p * h + c] = sin((double)p * theta[c] * lambda[c]);
    }
  for (int32_t kvh = 0; kvh < hkv; ++kvh) {
    int any = 0;
    for (int64_t r = 0; r < n_rows && !any; ++r) any = (row_head[r] / group == kvh);
    if (!any) continue;
#pragma omp parallel
    {
      double* x = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
      for (int64_t j = 0; j < npos; ++j) {
        view_row(&k, j, kvh, d, x);
        rotate_with(x, d, cb + j * h, sb + j * h, 1.0, kb + j * d);
        rotate_with(x, d, ci + j * h, si + j * h, 1.0, ki + j * d);
      }
      free(x);
    }
#pragma omp parallel
    {
      double* x = (double*)malloc(sizeof(double) * (size_t)d * 3);
      double* qb = x + d;
      double* qi = qb + d;
      double* s = (double*)malloc(sizeof(double) * (size_t)npos);
      unsigned char* mask = (unsigned char*)malloc((size_t)npos);
#pragma omp for schedule(dynamic, 1)
      for (int64_t r = 0; r < n_rows; ++r) {
        if (row_head[r] / group != kvh) continue;
        const int64_t i = row_pos[r];
        view_row(&q, i, row_head[r], d, x);
        rotate_with(x, d, cb + i * h, sb + i * h, 1.0, qb);
        rotate_with(x, d, ci + i * h, si + i * h, 1.0, qi);
        for (int64_t j = 0; j < npos; ++j) {
          const int64_t dist = i - j;
          if (dist < 0) { mask[j] = MASKED; s[j] = 0.0; }
          else if (dist < w0) { mask[j] = LOCAL; s[j] = scale * dot(qb, kb + j * d, d); }
          else { mask[j] = REMOTE; s[j] = scale * dot(qi, ki + j * d, d); }
        }
        softmax_row(s, mask, npos, &v, kvh, d, out + r * d, lse + r);
      }
      free(x); free(s); free(mask);
    }
  }
  free(theta); free(cb); free(sb); free(ci); free(si); free(kb); free(ki);
  return 0;
}

/* ---- decode (Methodology section 2, on-the-fly correction rotation) ------- */

int jlo_decode_step(jlo_view q_tilde, jlo_view k_cache, jlo_view v_cache, int64_t L, int32_t d,
                    int32_t n_q_heads, int32_t n_kv_heads, int64_t w0, int64_t w_pretrained,
                    double rope_base, double scale, int plain, double* out, double* lse) {
  if (check_common(L, d, n_q_heads, n_kv_heads, w0, w_pretrained) || L < 1) return -1;
  const int32_t h = d / 2;
  const int64_t i = L - 1;
  const int64_t G = plain ? 1 : jlo_group_size(L, w_pretrained);
  const int32_t group = n_q_heads / n_kv_heads;
  /* correction angles are |f(x) - x| <= L - 1: tabulate cos/sin(n theta) for n < L */
  double* cs = (double*)malloc(sizeof(double) * (size_t)(L * h));
  double* sn = (double*)malloc(sizeof(double) * (size_t)(L * h));
  double* kc = (double*)malloc(sizeof(double) * (size_t)(L * d));
  double* s = (double*)malloc(sizeof(double) * (size_t)L);
  unsigned char* mask = (unsigned char*)malloc((size_t)L);
  if (!cs || !sn || !kc || !s || !mask) {
    free(cs); free(sn); free(kc); free(s); free(mask);
    return -3;
  }
  jlo_rope_cos_sin(L, d, rope_base, cs, sn);
  const int64_t nq = i - jlo_remote_pos(i, G); /* query correction R(f(i) - i) = R(-nq) */

  for (int32_t kvh = 0; kvh < n_kv_heads; ++kvh) {
    /* corrected keys: R(f(j) - j) k_tilde_j for remote keys, k_tilde_j for local */
#pragma omp parallel
    {
      double* x = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
      for (int64_t j = 0; j < L; ++j) {
        view_row(&k_cache, j, kvh, d, x);
        int local = plain || (i - j < w0);
        mask[j] = local ? LOCAL : REMOTE;
        if (local) {
          memcpy(kc + j * d, x, sizeof(double) * (size_t)d);
        } else {
          int64_t nk = j - jlo_remote_pos(j, G); /* R(f(j) - j) = R(-nk) */
          rotate_with(x, d, cs + nk * h, sn + nk * h, -1.0, kc + j * d);
        }
      }
      free(x);
    }
    for (int32_t hh = 0; hh < group; ++hh) {
      int32_t qh = kvh * group + hh;
      double* qt = (double*)malloc(sizeof(double) * (size_t)d * 2);
      double* qc = qt + d;
      view_row(&q_tilde, 0, qh, d, qt);
      rotate_with(qt, d, cs + nq * h, sn + nq * h, -1.0, qc);
#pragma omp parallel for schedule(static)
      for (int64_t j = 0; j < L; ++j) s[j] = scale * dot(mask[j] == LOCAL ? qt : qc, kc + j * d, d);
      softmax_row(s, mask, L, &v_cache, kvh, d, out + (int64_t)qh * d, lse + qh);
      free(qt);
    }
  }
  free(cs); free(sn); free(kc); free(s); free(mask);
  return 0;
}

int jlo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

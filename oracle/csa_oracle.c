/*
 * csa_oracle.c -- CPU oracle of the CSA / HCA compressed attention layer.
 *
 * TEST INFRASTRUCTURE ONLY (see csa_oracle.h for the contract and sources).
 * Written for a reader to check against the pages by eye: one loop per
 * definition, double precision, no blocking or fusion.  OpenMP is used only
 * across independent query rows / entries.
 */
#include "csa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static double ld_elem(const void* p, int dt, int64_t i) {
  switch (dt) {
    case ORC_F64: return ((const double*)p)[i];
    case ORC_F32: return (double)((const float*)p)[i];
    default: {
      uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
      float f;
      memcpy(&f, &bits, sizeof f);
      return (double)f;
    }
  }
}

int64_t orc_n_visible(int64_t t, int m, int64_t n_entries) {
  int64_t v = (t + 1) / m;
  if (v < 0) v = 0;
  return v < n_entries ? v : n_entries;
}

/* ---------------------------------------------------------------- pooling */
int orc_pool(int T, int C, int m, int overlap, int in_dt, const void* kv, const void* z,
             const float* bias, double* out) {
  const int E = T / m;
  const int S = overlap ? 2 * m : m;
#pragma omp parallel for schedule(static)
  for (int j = 0; j < E; ++j) {
    double* a = (double*)malloc(sizeof(double) * S);
    int* tok = (int*)malloc(sizeof(int) * S);
    for (int c = 0; c < C; ++c) {
      /* slot s -> token; previous-group slots of entry 0 do not exist */
      int first_tok = overlap ? m * (j - 1) : m * j;
      double amax = -INFINITY;
      for (int s = 0; s < S; ++s) {
        tok[s] = first_tok + s;
        if (tok[s] < 0) { a[s] = -INFINITY; continue; }
        a[s] = ld_elem(z, in_dt, (int64_t)tok[s] * C + c) + (double)bias[(int64_t)s * C + c];
        if (a[s] > amax) amax = a[s];
      }
      double den = 0.0, num = 0.0;
      for (int s = 0; s < S; ++s) {
        if (tok[s] < 0) continue;
        double e = exp(a[s] - amax);
        den += e;
        num += e * ld_elem(kv, in_dt, (int64_t)tok[s] * C + c);
      }
      out[(int64_t)j * C + c] = num / den;
    }
    free(a);
    free(tok);
  }
  return E;
}

/* ---------------------------------------------------------------- RMSNorm */
void orc_rmsnorm(int64_t rows, int C, double eps, double* x) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double* v = x + r * C;
    double ss = 0.0;
    for (int c = 0; c < C; ++c) ss += v[c] * v[c];
    double inv = 1.0 / sqrt(ss / C + eps);
    for (int c = 0; c < C; ++c) v[c] *= inv;
  }
}

/* ------------------------------------------------------------------- RoPE */
void orc_rope(int64_t rows, int C, int rope_dims, double theta, const int64_t* pos, double* x) {
  if (rope_dims <= 0) return;
  const int base = C - rope_dims;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double* v = x + r * C + base;
    for (int i = 0; i < rope_dims / 2; ++i) {
      double ang = (double)pos[r] * pow(theta, -2.0 * i / rope_dims);
      double cs = cos(ang), sn = sin(ang);
      double a = v[2 * i], b = v[2 * i + 1];
      v[2 * i] = a * cs - b * sn;
      v[2 * i + 1] = a * sn + b * cs;
    }
  }
}

/* ------------------------------------------------------------------ MXFP4 */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* smallest E with amax <= 6 * 2^E, clamped to [-127, 127] */
static int mx_block_exponent(double amax) {
  if (amax == 0.0) return -127;
  int E = -127;
  while (E < 127 && amax > 6.0 * ldexp(1.0, E)) ++E;
  return E;
}

/* round-to-nearest-even of a (>= 0, already divided by 2^E) onto the E2M1 magnitudes */
static int mx_magnitude_code(double a) {
  int best = 0;
  double best_err = fabs(a - kE2M1[0]);
  for (int c = 1; c < 8; ++c) {
    double err = fabs(a - kE2M1[c]);
    if (err < best_err || (err == best_err && (c % 2) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return best;
}

void orc_mxfp4_quantize(int64_t rows, int cols, const float* x, uint8_t* packed, uint8_t* scales) {
  const int nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int b = 0; b < nb; ++b) {
      const float* blk = x + r * cols + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i)
        if (fabs((double)blk[i]) > amax) amax = fabs((double)blk[i]);
      int E = mx_block_exponent(amax);
      scales[r * nb + b] = (uint8_t)(E + 127);
      for (int i = 0; i < 32; ++i) {
        double y = ldexp((double)blk[i], -E);
        int code = mx_magnitude_code(fabs(y)) | (signbit(blk[i]) ? 8 : 0);
        uint8_t* byte = packed + r * (cols / 2) + (b * 32 + i) / 2;
        if (i % 2 == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
        else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
      }
    }
  }
}

void orc_mxfp4_dequantize(int64_t rows, int cols, const uint8_t* packed, const uint8_t* scales,
                          double* out) {
  const int nb = cols / 32;
  for (int64_t r = 0; r < rows; ++r)
    for (int c = 0; c < cols; ++c) {
      uint8_t byte = packed[r * (cols / 2) + c / 2];
      int code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      double v = kE2M1[code & 7] * ((code & 8) ? -1.0 : 1.0);
      out[r * cols + c] = ldexp(v, (int)scales[r * nb + c / 32] - 127);
    }
}

/* ------------------------------------------------------------ indexer */
int64_t orc_index_scores(int nq, int Hi, int Di, const uint8_t* q_packed, const uint8_t* q_scales,
                         const float* w, const int32_t* q_seq, const int32_t* n_vis, int E_max,
                         const uint8_t* k_packed, const uint8_t* k_scales, float* s32, double* s64) {
  int64_t inexact = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : inexact)
  for (int n = 0; n < nq; ++n) {
    double* qd = (double*)malloc(sizeof(double) * Hi * Di);
    double* kd = (double*)malloc(sizeof(double) * Di);
    orc_mxfp4_dequantize((int64_t)Hi, Di, q_packed + (int64_t)n * Hi * (Di / 2),
                         q_scales + (int64_t)n * Hi * (Di / 32), qd);
    const int64_t kbase = (int64_t)q_seq[n] * E_max;
    for (int j = 0; j < n_vis[n]; ++j) {
      orc_mxfp4_dequantize(1, Di, k_packed + (kbase + j) * (Di / 2), k_scales + (kbase + j) * (Di / 32), kd);
      double acc64 = 0.0;
      float acc32 = 0.0f;
      for (int h = 0; h < Hi; ++h) {
        double d = 0.0;
        for (int c = 0; c < Di; ++c) d += qd[h * Di + c] * kd[c];
        float df = (float)d;
        if ((double)df != d) ++inexact;
        acc64 += (double)w[(int64_t)n * Hi + h] * (d > 0.0 ? d : 0.0);
        acc32 = fmaf(w[(int64_t)n * Hi + h], df > 0.0f ? df : 0.0f, acc32);
      }
      s32[(int64_t)n * E_max + j] = acc32;
      if (s64) s64[(int64_t)n * E_max + j] = acc64;
    }
    free(qd);
    free(kd);
  }
  return inexact;
}

/* ---------------------------------------------------------------- top-k */
typedef struct {
  float s;
  int32_t j;
} cand_t;

static int cand_order(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->s > b->s) return -1; /* score descending */
  if (a->s < b->s) return 1;
  return (a->j < b->j) ? -1 : (a->j > b->j); /* ties: index ascending */
}

static int idx_ascending(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

void orc_topk(int nq, int E_stride, const float* scores, const int32_t* n_vis, int k,
              int32_t* idx, int32_t* cnt, float* kth) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int n = 0; n < nq; ++n) {
    const int nv = n_vis[n];
    int32_t* out = idx + (int64_t)n * k;
    for (int r = 0; r < k; ++r) out[r] = -1;
    if (kth) kth[2 * n] = kth[2 * n + 1] = NAN;
    if (nv <= k) {
      for (int r = 0; r < nv; ++r) out[r] = r;
      cnt[n] = nv;
      continue;
    }
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * nv);
    for (int j = 0; j < nv; ++j) {
      c[j].s = scores[(int64_t)n * E_stride + j];
      c[j].j = j;
    }
    qsort(c, nv, sizeof(cand_t), cand_order);
    for (int r = 0; r < k; ++r) out[r] = c[r].j;
    qsort(out, k, sizeof(int32_t), idx_ascending);
    cnt[n] = k;
    if (kth) {
      kth[2 * n] = c[k - 1].s;
      kth[2 * n + 1] = c[k].s;
    }
    free(c);
  }
}

/* ------------------------------------------------------------- attention */
void orc_attention(int nq, int H, int D, double scale, int q_dt, const void* q, const int64_t* q_pos,
                   const int32_t* q_seq, int E_max, int e_dt, const void* entries, int k,
                   const int32_t* idx, const int32_t* cnt, int W, int Tw, int w_dt, const void* window,
                   const int64_t* wbase, double* out, double* lse) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int n = 0; n < nq; ++n) {
    const int b = q_seq[n];
    const int64_t t = q_pos[n];
    /* the key set: selected entries, then window rows */
    int64_t u_lo = t - W + 1;
    if (u_lo < 0) u_lo = 0;
    if (u_lo < wbase[b]) u_lo = wbase[b];
    int64_t u_hi = t;
    if (u_hi > wbase[b] + Tw - 1) u_hi = wbase[b] + Tw - 1;
    const int n_win = (W > 0 && u_hi >= u_lo) ? (int)(u_hi - u_lo + 1) : 0;
    const int n_sel = cnt[n];
    const int nk = n_sel + n_win;
    /* element offsets of each key row, with its source tensor */
    int64_t* row_off = (int64_t*)malloc(sizeof(int64_t) * (nk > 0 ? nk : 1));
    int* row_src = (int*)malloc(sizeof(int) * (nk > 0 ? nk : 1));
    for (int r = 0; r < n_sel; ++r) {
      row_off[r] = ((int64_t)b * E_max + idx[(int64_t)n * k + r]) * D;
      row_src[r] = 0;
    }
    for (int r = 0; r < n_win; ++r) {
      row_off[n_sel + r] = ((int64_t)b * Tw + (u_lo + r - wbase[b])) * D;
      row_src[n_sel + r] = 1;
    }
    double* logit = (double*)malloc(sizeof(double) * (nk > 0 ? nk : 1));
    for (int h = 0; h < H; ++h) {
      const int64_t qoff = ((int64_t)n * H + h) * D;
      double* o = out + qoff;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (nk == 0) {
        if (lse) lse[(int64_t)n * H + h] = -INFINITY;
        continue;
      }
      double mx = -INFINITY;
      for (int r = 0; r < nk; ++r) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) {
          double kv = row_src[r] ? ld_elem(window, w_dt, row_off[r] + d) : ld_elem(entries, e_dt, row_off[r] + d);
          dot += ld_elem(q, q_dt, qoff + d) * kv;
        }
        logit[r] = scale * dot;
        if (logit[r] > mx) mx = logit[r];
      }
      double den = 0.0;
      for (int r = 0; r < nk; ++r) den += exp(logit[r] - mx);
      for (int r = 0; r < nk; ++r) {
        double p = exp(logit[r] - mx) / den;
        for (int d = 0; d < D; ++d) {
          double kv = row_src[r] ? ld_elem(window, w_dt, row_off[r] + d) : ld_elem(entries, e_dt, row_off[r] + d);
          o[d] += p * kv;
        }
      }
      if (lse) lse[(int64_t)n * H + h] = mx + log(den);
    }
    free(logit);
    free(row_off);
    free(row_src);
  }
}

void orc_grouped_out_proj(int T, int H, int D, int G, int R, int d_model, int in_dt, const void* o, const void* A,
                          const void* Bm, double* z, double* y) {
  const int64_t Kg = (int64_t)(H / G) * D;  /* inputs per group */
  const int64_t HD = (int64_t)H * D;
  const int64_t GR = (int64_t)G * R;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    /* each group: its heads' outputs times the group's own matrix */
    for (int g = 0; g < G; ++g) {
      for (int r = 0; r < R; ++r) {
        double acc = 0.0;
        for (int64_t i = 0; i < Kg; ++i)
          acc += ld_elem(o, in_dt, (int64_t)t * HD + g * Kg + i) * ld_elem(A, in_dt, ((int64_t)g * R + r) * Kg + i);
        z[(int64_t)t * GR + (int64_t)g * R + r] = acc;
      }
    }
    /* the groups' results, concatenated, times the dense matrix */
    for (int n = 0; n < d_model; ++n) {
      double acc = 0.0;
      for (int64_t j = 0; j < GR; ++j) acc += z[(int64_t)t * GR + j] * ld_elem(Bm, in_dt, (int64_t)n * GR + j);
      y[(int64_t)t * d_model + n] = acc;
    }
  }
}

/*
 * csa2_oracle.c -- CPU oracle for the CSA2 decode step over an FP4 global KV
 * cache.  TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU leg).
 * See csa2_oracle.h for the source tags [REL] [CNB] [YOM] [TUC] and for the
 * contract of every function.  Compile without fast-math and with
 * -ffp-contract=off so that every float operation is a single IEEE rounding.
 */
#include "csa2_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ formats */

double csa2o_bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

uint16_t csa2o_bf16_round(double v) {
  /* Round to the nearest bf16 by comparing the two neighbours of v in the
   * bf16 grid; ties pick the pattern with an even last bit. */
  float f = (float)v; /* only used to find the binade; refined below */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t lo = (uint16_t)(u >> 16);
  /* candidates: lo, and its neighbours towards +inf and -inf */
  uint16_t cands[3] = {lo, (uint16_t)(lo + 1), (uint16_t)(lo - 1)};
  uint16_t best = lo;
  double bestd = INFINITY;
  for (int i = 0; i < 3; i++) {
    uint16_t c = cands[i];
    if ((c & 0x7F80) == 0x7F80) continue; /* skip inf / nan patterns */
    if ((c ^ lo) & 0x8000) continue;      /* stay on the sign of v */
    double d = fabs(csa2o_bf16_value(c) - v);
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    }
  }
  if (v == 0.0) best = signbit(v) ? 0x8000 : 0x0000;
  return best;
}

double csa2o_e2m1_value(uint8_t code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m                       /* subnormal: 2^(1-1) * m/2 */
                        : ldexp(1.0 + 0.5 * m, e - 1);  /* normal: 2^(e-1) * (1+m/2) */
  return s ? -mag : mag;
}

double csa2o_e4m3_value(uint8_t bits) {
  int s = (bits >> 7) & 1, e = (bits >> 3) & 15, m = bits & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp(m / 8.0, -6)            /* subnormal: 2^(1-7) * m/8 */
                        : ldexp(1.0 + m / 8.0, e - 7);  /* normal: 2^(e-7) * (1+m/8) */
  return s ? -mag : mag;
}

uint8_t csa2o_e2m1_encode(float q) {
  double a = fabs((double)q);
  uint8_t sign = signbit(q) ? 0x8 : 0x0;
  /* Saturation: nothing is nearer than the largest magnitude.  Stated
   * explicitly because far-away distances are not exact in fp64. */
  if (a >= 6.0) return (uint8_t)(0x7 | sign);
  uint8_t best = 0;
  double bestd = INFINITY;
  for (uint8_t c = 0; c < 8; c++) {
    double d = fabs(a - csa2o_e2m1_value(c));
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    }
  }
  return (uint8_t)(best | sign);
}

uint8_t csa2o_e4m3_encode(float t) {
  if (isnan(t)) return 0x7F;
  double a = fabs((double)t);
  uint8_t sign = signbit(t) ? 0x80 : 0x00;
  if (a >= 448.0) return (uint8_t)(0x7E | sign); /* satfinite, as above */
  uint8_t best = 0;
  double bestd = INFINITY;
  for (int c = 0; c <= 0x7E; c++) { /* every finite non-negative code */
    double d = fabs(a - csa2o_e4m3_value((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = (uint8_t)c;
      bestd = d;
    }
  }
  return (uint8_t)(best | sign);
}

/* ----------------------------------------------------------- A1/A2 codec */

int csa2o_quantize_fp4(const uint16_t *x, int64_t rows, int32_t ch,
                       uint8_t *codes, uint8_t *scales) {
  if (rows < 0 || ch <= 0 || ch % 16 != 0) return CSA2O_EARG;
  for (int64_t r = 0; r < rows; r++) {
    const uint16_t *xr = x + r * ch;
    uint8_t *cr = codes + r * (ch / 2);
    uint8_t *sr = scales + r * (ch / 16);
    for (int g = 0; g < ch / 16; g++) {
      float amax = 0.0f;
      for (int i = 0; i < 16; i++) {
        float v = fabsf((float)csa2o_bf16_value(xr[16 * g + i]));
        if (v > amax) amax = v;
      }
      volatile float t = amax / 6.0f; /* one fp32 rounding */
      uint8_t sb = csa2o_e4m3_encode(t);
      float s = (float)csa2o_e4m3_value(sb);
      sr[g] = sb;
      uint8_t code[16];
      for (int i = 0; i < 16; i++) {
        if (s == 0.0f) {
          code[i] = 0x0;
        } else {
          volatile float qv = (float)csa2o_bf16_value(xr[16 * g + i]) / s;
          code[i] = csa2o_e2m1_encode(qv);
        }
      }
      for (int j = 0; j < 8; j++)
        cr[8 * g + j] = (uint8_t)(code[2 * j] | (code[2 * j + 1] << 4));
    }
  }
  return CSA2O_OK;
}

int csa2o_dequantize_fp4(const uint8_t *codes, const uint8_t *scales,
                         int64_t rows, int32_t ch, double *y) {
  if (rows < 0 || ch <= 0 || ch % 16 != 0) return CSA2O_EARG;
  for (int64_t r = 0; r < rows; r++)
    for (int i = 0; i < ch; i++) {
      uint8_t byte = codes[r * (ch / 2) + i / 2];
      uint8_t code = (i & 1) ? (byte >> 4) : (byte & 0xF);
      y[r * ch + i] = csa2o_e2m1_value(code) *
                      csa2o_e4m3_value(scales[r * (ch / 16) + i / 16]);
    }
  return CSA2O_OK;
}

/* --------------------------------------------------------- KV cache view */

int64_t csa2o_row_of(const csa2o_kv *kv, int32_t b, int64_t p) {
  int64_t row;
  if (kv->page_table == NULL) {
    row = (int64_t)b * kv->seq_stride + p;
  } else {
    int64_t page = p / kv->page_rows;
    if (page >= kv->max_pages) return -1;
    int64_t pid = kv->page_table[(int64_t)b * kv->max_pages + page];
    row = pid * kv->page_rows + p % kv->page_rows;
  }
  if (row < 0 || row >= kv->pool_rows) return -1;
  return row;
}

/* ------------------------------------------------------------- indexer */

/* s(p) for one position, fp64 over the bf16 values (products are exact). */
static double score_one(const uint16_t *k, const csa2o_dims *dm,
                        const uint16_t *q_idx, const float *w) {
  double acc = 0.0;
  for (int h = 0; h < dm->hi; h++) {
    double dot = 0.0;
    for (int d = 0; d < dm->di; d++)
      dot += csa2o_bf16_value(q_idx[h * dm->di + d]) * csa2o_bf16_value(k[d]);
    acc += (double)w[h] * (dot > 0.0 ? dot : 0.0);
  }
  return acc;
}

int csa2o_scores(const csa2o_kv *kv, const csa2o_dims *dm, int32_t b, int64_t C,
                 const uint16_t *q_idx, const float *w, double *s) {
  for (int64_t p = 0; p < C; p++) {
    int64_t row = csa2o_row_of(kv, b, p);
    if (row < 0) return CSA2O_EARG;
    s[p] = score_one(kv->idxk + row * dm->di, dm, q_idx, w);
  }
  return CSA2O_OK;
}

int csa2o_block_max(const double *s, int64_t C, int32_t blk, double *bm) {
  if (blk <= 0) return CSA2O_EARG;
  int64_t nblk = (C + blk - 1) / blk;
  for (int64_t j = 0; j < nblk; j++) {
    double m = -INFINITY;
    for (int64_t p = j * blk; p < C && p < (j + 1) * blk; p++)
      if (s[p] > m) m = s[p];
    bm[j] = m;
  }
  return CSA2O_OK;
}

typedef struct {
  double v;
  int64_t id;
} vid_t;

static int cmp_desc_then_id(const void *a, const void *b) {
  const vid_t *x = (const vid_t *)a, *y = (const vid_t *)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

static int cmp_i32(const void *a, const void *b) {
  int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

int64_t csa2o_select_topk(const double *v, const int64_t *ids, int64_t n,
                          int64_t k, int32_t *out) {
  if (n <= 0 || k <= 0) return 0;
  vid_t *a = (vid_t *)malloc((size_t)n * sizeof *a);
  for (int64_t i = 0; i < n; i++) {
    a[i].v = v[i];
    a[i].id = ids ? ids[i] : i;
  }
  qsort(a, (size_t)n, sizeof *a, cmp_desc_then_id);
  int64_t m = k < n ? k : n;
  for (int64_t i = 0; i < m; i++) out[i] = (int32_t)a[i].id;
  free(a);
  qsort(out, (size_t)m, sizeof *out, cmp_i32);
  return m;
}

int64_t csa2o_pool(const double *bm, int64_t nblk, int32_t pool_blocks,
                   int32_t *pool) {
  return csa2o_select_topk(bm, NULL, nblk, pool_blocks, pool);
}

/* ----------------------------------------------------------- attention */

int csa2o_attention(const csa2o_kv *kv, const csa2o_dims *dm, int32_t b,
                    const uint16_t *q, const int32_t *idx, int32_t n_idx,
                    const uint8_t *swa, int32_t swa_len, double sm_scale,
                    double *out) {
  const int D = dm->d;
  const int nk = n_idx + swa_len;
  memset(out, 0, sizeof(double) * (size_t)dm->h * D);
  if (nk == 0) return CSA2O_OK;
  double *R = (double *)malloc(sizeof(double) * (size_t)nk * D);
  for (int j = 0; j < n_idx; j++) {
    int64_t row = csa2o_row_of(kv, b, idx[j]);
    if (row < 0) {
      free(R);
      return CSA2O_EARG;
    }
    csa2o_dequantize_fp4(kv->codes + row * (D / 2), kv->scales + row * (D / 16),
                         1, D, R + (size_t)j * D);
  }
  for (int j = 0; j < swa_len; j++)
    for (int c = 0; c < D; c++)
      R[(size_t)(n_idx + j) * D + c] = csa2o_e4m3_value(swa[(size_t)j * D + c]);
  double *l = (double *)malloc(sizeof(double) * (size_t)nk);
  for (int h = 0; h < dm->h; h++) {
    double m = -INFINITY;
    for (int j = 0; j < nk; j++) {
      double dot = 0.0;
      for (int c = 0; c < D; c++)
        dot += csa2o_bf16_value(q[h * D + c]) * R[(size_t)j * D + c];
      l[j] = dot * sm_scale;
      if (l[j] > m) m = l[j];
    }
    double den = 0.0;
    for (int j = 0; j < nk; j++) {
      l[j] = exp(l[j] - m);
      den += l[j];
    }
    for (int j = 0; j < nk; j++)
      for (int c = 0; c < D; c++)
        out[h * D + c] += (l[j] / den) * R[(size_t)j * D + c];
  }
  free(l);
  free(R);
  return CSA2O_OK;
}

/* ----------------------------------------------------------- layer group */

int csa2o_layer_group(const csa2o_kv *kv, const csa2o_dims *dm, int32_t B,
                      const int64_t *n_rows, int32_t L, const int32_t *modes,
                      const uint16_t *q_idx, const float *w, const uint16_t *q,
                      const uint8_t *swa, const int32_t *swa_len, int32_t top_k,
                      int32_t pool_blocks, double sm_scale, int32_t *idx,
                      int32_t *idx_count, int32_t *pool, int32_t *pool_count,
                      double *out) {
  const int HI = dm->hi, DI = dm->di, H = dm->h, D = dm->d, W = dm->w;
  int rc = CSA2O_OK;
  for (int l = 0; l < L; l++)
    if (modes[l] < CSA2O_FULL || modes[l] > CSA2O_REUSE) return CSA2O_EARG;
  /* A Reindex or Reuse layer needs an earlier Full layer whose cache it
   * reuses [REL §CSA2: "reuses the previous Full layer's main KV"]. */
  if (L > 0 && modes[0] != CSA2O_FULL) return CSA2O_EARG;
  for (int b = 0; b < B; b++) pool_count[b] = 0;

  for (int b = 0; b < B && rc == CSA2O_OK; b++) {
    const int64_t C = n_rows[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    int64_t nblk = (C + dm->blk - 1) / dm->blk;
    double *bm = (double *)malloc(sizeof(double) * (size_t)(nblk > 0 ? nblk : 1));
    int32_t *cur_pool = (int32_t *)malloc(sizeof(int32_t) * (size_t)(pool_blocks > 0 ? pool_blocks : 1));
    int64_t cur_pool_n = 0;
    int32_t *latest = (int32_t *)malloc(sizeof(int32_t) * (size_t)top_k);
    int64_t latest_n = 0;

    for (int l = 0; l < L && rc == CSA2O_OK; l++) {
      const uint16_t *qi = q_idx + ((size_t)l * B + b) * HI * DI;
      const float *wl = w + ((size_t)l * B + b) * HI;
      if (modes[l] == CSA2O_FULL) {
        /* Score every visible position; exact Top-k by a full sort over all
         * of them ("fresh Top-512", [REL §CSA2], [YOM §二 table]). */
        rc = csa2o_scores(kv, dm, b, C, qi, wl, s);
        if (rc) break;
        latest_n = csa2o_select_topk(s, NULL, C, top_k, latest);
        if (pool_blocks > 0) {
          /* HSI pool: top blocks of blk positions by block max [YOM §二]. */
          csa2o_block_max(s, C, dm->blk, bm);
          cur_pool_n = csa2o_pool(bm, nblk, pool_blocks, cur_pool);
        }
      } else if (modes[l] == CSA2O_REINDEX) {
        /* Rescore with this layer's own indexer query, only inside the pool
         * (all positions when there is no pool) [REL §CSA2; YOM §二]. */
        int64_t ncand = 0;
        int64_t *ids;
        if (pool_blocks > 0) {
          ids = (int64_t *)malloc(sizeof(int64_t) * (size_t)(cur_pool_n * dm->blk + 1));
          for (int64_t i = 0; i < cur_pool_n; i++)
            for (int64_t p = (int64_t)cur_pool[i] * dm->blk;
                 p < ((int64_t)cur_pool[i] + 1) * dm->blk && p < C; p++)
              ids[ncand++] = p;
        } else {
          ids = (int64_t *)malloc(sizeof(int64_t) * (size_t)(C + 1));
          for (int64_t p = 0; p < C; p++) ids[ncand++] = p;
        }
        double *v = (double *)malloc(sizeof(double) * (size_t)(ncand + 1));
        for (int64_t i = 0; i < ncand && rc == CSA2O_OK; i++) {
          int64_t row = csa2o_row_of(kv, b, ids[i]);
          if (row < 0) rc = CSA2O_EARG;
          else v[i] = score_one(kv->idxk + row * DI, dm, qi, wl);
        }
        if (rc) {
          free(v);
          free(ids);
          break;
        }
        latest_n = csa2o_select_topk(v, ids, ncand, top_k, latest);
        free(v);
        free(ids);
      }
      /* REUSE: the latest indices as they are [REL §CSA2; YOM §二]. */
      int32_t *il = idx + ((size_t)l * B + b) * top_k;
      for (int i = 0; i < top_k; i++) il[i] = i < latest_n ? latest[i] : -1;
      idx_count[(size_t)l * B + b] = (int32_t)latest_n;

      /* Core attention over the sparse rows and this layer's SWA window. */
      rc = csa2o_attention(kv, dm, b, q + ((size_t)l * B + b) * H * D, latest,
                           (int32_t)latest_n, swa + ((size_t)l * B + b) * W * D,
                           swa_len[b], sm_scale, out + ((size_t)l * B + b) * H * D);
    }
    if (pool_blocks > 0) {
      for (int i = 0; i < pool_blocks; i++)
        pool[(size_t)b * pool_blocks + i] = i < cur_pool_n ? cur_pool[i] : -1;
      pool_count[b] = (int32_t)cur_pool_n;
    }
    free(latest);
    free(cur_pool);
    free(bm);
    free(s);
  }
  return rc;
}

/* ----------------------------------------------------------- cache append */

int csa2o_project_idxk(const uint16_t *x, const uint16_t *w_idx, int32_t d, int32_t di,
                       uint16_t *out) {
  if (d <= 0 || di <= 0) return CSA2O_EARG;
  for (int32_t j = 0; j < di; j++) {
    double acc = 0.0;
    for (int32_t c = 0; c < d; c++)
      acc += csa2o_bf16_value(x[c]) * csa2o_bf16_value(w_idx[(int64_t)c * di + j]);
    out[j] = csa2o_bf16_round(acc);
  }
  return CSA2O_OK;
}

int csa2o_cache_append(const csa2o_kv *kv, const csa2o_dims *dm, int32_t B,
                       uint8_t *codes, uint8_t *scales, uint16_t *idxk,
                       int64_t *n_rows, const uint16_t *x, const uint16_t *w_idx,
                       int32_t L, const uint16_t *x_swa, uint8_t *swa,
                       int64_t *swa_pos, int32_t *swa_len) {
  const int32_t d = dm->d, di = dm->di, w = dm->w;
  int rc = CSA2O_OK;
  for (int32_t b = 0; b < B; b++) {
    const int64_t p = n_rows[b];
    const int64_t cap = kv->page_table ? (int64_t)kv->max_pages * kv->page_rows
                                       : kv->seq_stride;
    const int64_t row = (p >= 0 && p < cap) ? csa2o_row_of(kv, b, p) : -1;
    if (row < 0) {
      rc = CSA2O_EARG;
      continue;
    }
    csa2o_quantize_fp4(x + (int64_t)b * d, 1, d, codes + row * (d / 2),
                       scales + row * (d / 16));
    csa2o_project_idxk(x + (int64_t)b * d, w_idx, d, di, idxk + row * di);
    n_rows[b] = p + 1;
  }
  for (int32_t b = 0; b < B && L > 0; b++) {
    const int64_t slot = swa_pos[b] % w;
    for (int32_t l = 0; l < L; l++) {
      const uint16_t *src = x_swa + ((int64_t)l * B + b) * d;
      uint8_t *dst = swa + (((int64_t)l * B + b) * w + slot) * d;
      for (int32_t c = 0; c < d; c++) dst[c] = csa2o_e4m3_encode((float)csa2o_bf16_value(src[c]));
    }
    swa_pos[b] += 1;
    swa_len[b] = (int32_t)(swa_pos[b] < w ? swa_pos[b] : w);
  }
  return rc;
}

/* ----------------------------------------------------- multi-query decode */

int csa2o_layer_group_multi(const csa2o_kv *kv, const csa2o_dims *dm, int32_t B, int32_t Q,
                            const int64_t *n_rows, int32_t L, const int32_t *modes,
                            const uint16_t *q_idx, const float *w, const uint16_t *q,
                            const uint8_t *swa, const int32_t *swa_len, int32_t top_k,
                            int32_t pool_blocks, double sm_scale, int32_t *idx,
                            int32_t *idx_count, int32_t *pool, int32_t *pool_count,
                            double *out) {
  if (B < 0 || Q < 1 || L < 0 || top_k < 1) return CSA2O_EARG;
  const int HI = dm->hi, DI = dm->di, H = dm->h, D = dm->d, W = dm->w;
  const int64_t WR = (int64_t)W + Q - 1; /* window rows per (layer, sequence) */
  const int pb = pool_blocks > 0 ? pool_blocks : 1;
  uint16_t *qi_t = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(L ? L : 1) * HI * DI);
  float *w_t = (float *)malloc(sizeof(float) * (size_t)(L ? L : 1) * HI);
  uint16_t *q_t = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(L ? L : 1) * H * D);
  uint8_t *swa_t = (uint8_t *)calloc((size_t)(L ? L : 1) * W * D, 1);
  int32_t *idx_t = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L ? L : 1) * top_k);
  int32_t *cnt_t = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L ? L : 1));
  int32_t *pool_t = (int32_t *)malloc(sizeof(int32_t) * (size_t)pb);
  double *out_t = (double *)malloc(sizeof(double) * (size_t)(L ? L : 1) * H * D);
  int rc = CSA2O_OK;
  for (int32_t b = 0; b < B && rc == CSA2O_OK; b++) {
    /* the view of sequence b alone, as batch entry 0 */
    csa2o_kv one = *kv;
    if (kv->page_table) {
      one.page_table = kv->page_table + (int64_t)b * kv->max_pages;
    } else {
      const int64_t off = (int64_t)b * kv->seq_stride;
      one.codes = kv->codes + off * (D / 2);
      one.scales = kv->scales + off * (D / 16);
      one.idxk = kv->idxk + off * DI;
      one.pool_rows = kv->pool_rows - off;
    }
    for (int32_t t = 0; t < Q && rc == CSA2O_OK; t++) {
      const int64_t v = (int64_t)b * Q + t; /* (b, t) on the flattened axis */
      int64_t C = n_rows[b] - (Q - 1 - t);
      if (C < 0) C = 0;
      int64_t e = (int64_t)swa_len[b] - (Q - 1 - t);
      if (e < 0) e = 0;
      const int64_t s0 = e > W ? e - W : 0;
      const int32_t len = (int32_t)(e - s0);
      for (int32_t l = 0; l < L; l++) {
        memcpy(qi_t + (size_t)l * HI * DI, q_idx + ((size_t)l * B * Q + v) * HI * DI,
               sizeof(uint16_t) * HI * DI);
        memcpy(w_t + (size_t)l * HI, w + ((size_t)l * B * Q + v) * HI, sizeof(float) * HI);
        memcpy(q_t + (size_t)l * H * D, q + ((size_t)l * B * Q + v) * H * D,
               sizeof(uint16_t) * H * D);
        memcpy(swa_t + (size_t)l * W * D, swa + (((size_t)l * B + b) * WR + s0) * D,
               (size_t)len * D);
      }
      rc = csa2o_layer_group(&one, dm, 1, &C, L, modes, qi_t, w_t, q_t, swa_t, &len, top_k,
                             pool_blocks, sm_scale, idx_t, cnt_t, pool_t, pool_count + v, out_t);
      for (int32_t l = 0; l < L; l++) {
        memcpy(idx + ((size_t)l * B * Q + v) * top_k, idx_t + (size_t)l * top_k,
               sizeof(int32_t) * top_k);
        idx_count[(size_t)l * B * Q + v] = cnt_t[l];
        memcpy(out + ((size_t)l * B * Q + v) * H * D, out_t + (size_t)l * H * D,
               sizeof(double) * H * D);
      }
      if (pool_blocks > 0)
        memcpy(pool + (size_t)v * pool_blocks, pool_t, sizeof(int32_t) * pool_blocks);
    }
  }
  free(qi_t);
  free(w_t);
  free(q_t);
  free(swa_t);
  free(idx_t);
  free(cnt_t);
  free(pool_t);
  free(out_t);
  return rc;
}

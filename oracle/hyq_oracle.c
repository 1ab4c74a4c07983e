/*
 * hyq_oracle.c -- plain CPU oracle for the HyQuant hybrid KV-cache decode
 * path.  TEST INFRASTRUCTURE ONLY (see hyq_oracle.h for scope and sources).
 *
 * Deliberately simple: one position at a time, fp64 accumulation, no
 * blocking or reordering.  The only parallelism is an OpenMP loop over
 * independent (batch, kv-head) units.
 */
#include "hyq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------
 * binary16 conversions (IEEE 754: 1 sign bit, 5 exponent bits with bias 15,
 * 10 fraction bits; exponent 0 = subnormal with weight 2^-24 per ulp).
 * ---------------------------------------------------------------------- */
double hyqo_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m | 0x400), e - 25);
  return sign ? -v : v;
}

uint16_t hyqo_float_to_half(float f) {
  uint32_t bits;
  memcpy(&bits, &f, 4);
  uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  double a = fabs((double)f);
  /* 65520 is halfway between 65504 (largest finite, odd significand) and
   * 2^16; ties go to the even neighbour, which is the overflow to inf. */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
  if (a < ldexp(1.0, -14)) {
    /* subnormal range: count units of 2^-24, round half to even */
    double u = rint(a * ldexp(1.0, 24));
    return (uint16_t)(sign | (uint16_t)u); /* u == 1024 is the smallest normal */
  }
  int E;
  double m = frexp(a, &E);          /* a = m * 2^E, m in [0.5, 1) */
  double u = rint(ldexp(m, 11));    /* 11 significant bits, ties to even */
  int e = E - 1 + 15;
  if (u == 2048.0) {
    u = 1024.0;
    e += 1;
  }
  if (e >= 31) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | (uint16_t)(e << 10) | ((uint16_t)u & 0x3ffu));
}

static float half_to_float(uint16_t h) { return (float)hyqo_half_to_double(h); }

/* ------------------------------------------------------------------------
 * Quantizer.  The pages fix only the bit width (4 bits, keys and values); the grid
 * used here is asymmetric min/max over groups of 32 contiguous channels of
 * one token, fp16 scale = (max-min)/15 and fp16 zero = min, codes by
 * round-half-to-even of (x - zero)/scale clamped to [0, 15], decided in fp32.
 * ---------------------------------------------------------------------- */
int hyqo_quantize_row(const uint16_t *x, uint8_t code[HYQO_D],
                      uint16_t scale_h[HYQO_NG], uint16_t zero_h[HYQO_NG]) {
  for (int c = 0; c < HYQO_D; ++c) {
    if (!isfinite(hyqo_half_to_double(x[c]))) return -1;
  }
  for (int g = 0; g < HYQO_NG; ++g) {
    float mn = half_to_float(x[g * HYQO_GROUP]);
    float mx = mn;
    for (int c = g * HYQO_GROUP; c < (g + 1) * HYQO_GROUP; ++c) {
      float v = half_to_float(x[c]);
      if (v < mn) mn = v;
      if (v > mx) mx = v;
    }
    float diff = mx - mn;            /* fp32, round to nearest even */
    float s32 = diff / 15.0f;        /* fp32 division */
    uint16_t sh = hyqo_float_to_half(s32);
    uint16_t zh = hyqo_float_to_half(mn); /* exact: mn is an fp16 value */
    if (zh == 0x8000u) zh = 0;       /* canonical +0 for a zero minimum */
    scale_h[g] = sh;
    zero_h[g] = zh;
    float sf = half_to_float(sh);
    float zf = half_to_float(zh);
    for (int c = g * HYQO_GROUP; c < (g + 1) * HYQO_GROUP; ++c) {
      int q = 0;
      if (sf != 0.0f) {
        float num = half_to_float(x[c]) - zf; /* fp32 subtraction */
        float r = num / sf;                   /* fp32 division, no FMA */
        float ri = rintf(r);                  /* ties to even (default mode) */
        if (ri < 0.0f) ri = 0.0f;
        if (ri > 15.0f) ri = 15.0f;
        q = (int)ri;
      }
      code[c] = (uint8_t)q;
    }
  }
  return 0;
}

/* Packed row format: 8 pieces of 8 bytes.  Piece p holds channels
 * 4p..4p+3 of every group.  Inside a piece, byte 4h + 2j + i carries group
 * 2h + i, channels 4p + 2j (low nibble) and 4p + 2j + 1 (high nibble). */
void hyqo_code_slot(int c, int *byte_index, int *high_nibble) {
  int g = c / HYQO_GROUP;
  int w = c % HYQO_GROUP;
  int p = w / 4;
  int j = (w / 2) % 2;
  int h = g / 2;
  int i = g % 2;
  *byte_index = 8 * p + 4 * h + 2 * j + i;
  *high_nibble = w % 2;
}

static void store_codes(const uint8_t code[HYQO_D], uint8_t *packed) {
  memset(packed, 0, HYQO_ROW_BYTES);
  for (int c = 0; c < HYQO_D; ++c) {
    int b, hi;
    hyqo_code_slot(c, &b, &hi);
    packed[b] |= (uint8_t)((code[c] & 0xF) << (hi ? 4 : 0));
  }
}

void hyqo_unpack_codes(const uint8_t *packed, uint8_t code[HYQO_D]) {
  for (int c = 0; c < HYQO_D; ++c) {
    int b, hi;
    hyqo_code_slot(c, &b, &hi);
    code[c] = (uint8_t)((packed[b] >> (hi ? 4 : 0)) & 0xF);
  }
}

int64_t hyqo_pack(const uint16_t *x, int64_t n_rows, int64_t row_stride,
                  uint8_t *codes, uint16_t *sz) {
  int64_t bad = 0;
  for (int64_t r = 0; r < n_rows; ++r) {
    uint8_t code[HYQO_D];
    uint16_t s[HYQO_NG], z[HYQO_NG];
    if (hyqo_quantize_row(x + r * row_stride, code, s, z) != 0) {
      memset(codes + r * HYQO_ROW_BYTES, 0, HYQO_ROW_BYTES);
      memset(sz + r * 8, 0, 8 * sizeof(uint16_t));
      ++bad;
      continue;
    }
    store_codes(code, codes + r * HYQO_ROW_BYTES);
    for (int g = 0; g < HYQO_NG; ++g) {
      sz[r * 8 + 2 * g] = s[g];
      sz[r * 8 + 2 * g + 1] = z[g];
    }
  }
  return bad;
}

void hyqo_dequant_row(const uint8_t *packed, const uint16_t *sz, double out[HYQO_D]) {
  uint8_t code[HYQO_D];
  hyqo_unpack_codes(packed, code);
  for (int c = 0; c < HYQO_D; ++c) {
    int g = c / HYQO_GROUP;
    double s = hyqo_half_to_double(sz[2 * g]);
    double z = hyqo_half_to_double(sz[2 * g + 1]);
    out[c] = z + (double)code[c] * s; /* exact in fp64 */
  }
}

/* ------------------------------------------------------------------------
 * Key/value view of one unit, as decode sees it.
 * ---------------------------------------------------------------------- */
typedef struct {
  const hyqo_cache *c;
  int b, kvh;
  int64_t unit;
  int32_t T;
  int32_t *slot_of; /* position -> VL slot, or -1; length max(T, 1) */
} unit_view;

static int view_open(unit_view *u, const hyqo_cache *c, int64_t unit) {
  u->c = c;
  u->unit = unit;
  u->b = (int)(unit / c->n_kv_heads);
  u->kvh = (int)(unit % c->n_kv_heads);
  u->T = c->seq_len[u->b];
  if (u->T < 0 || u->T > c->capacity) return -2;
  int32_t n = u->T > 0 ? u->T : 1;
  u->slot_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  if (!u->slot_of) return -9;
  for (int32_t p = 0; p < n; ++p) u->slot_of[p] = -1;
  int32_t cnt = c->vl_count[unit];
  int32_t n_old = u->T - c->window; /* positions eligible for VL */
  if (cnt < 0 || cnt > c->vl_capacity) return -3;
  if (cnt > 0 && n_old <= 0) return -3;
  const int32_t *pos = c->vl_pos + unit * (int64_t)c->vl_capacity;
  for (int32_t i = 0; i < cnt; ++i) {
    if (pos[i] < 0 || pos[i] >= n_old) return -4;
    if (i > 0 && pos[i] <= pos[i - 1]) return -5;
    u->slot_of[pos[i]] = i;
  }
  return 0;
}

static void view_close(unit_view *u) { free(u->slot_of); }

/* Fill k, v (fp64) for position p of the unit. */
static void view_row(const unit_view *u, int32_t p, double k[HYQO_D], double v[HYQO_D]) {
  const hyqo_cache *c = u->c;
  int32_t W = c->window;
  if (p >= u->T - W) { /* local window, FP16 */
    int64_t base = (u->unit * W + (p % W)) * (int64_t)HYQO_D;
    for (int d = 0; d < HYQO_D; ++d) {
      k[d] = hyqo_half_to_double(c->win_k[base + d]);
      v[d] = hyqo_half_to_double(c->win_v[base + d]);
    }
  } else if (u->slot_of[p] >= 0) { /* vertical-line token, FP16 */
    int64_t base = (u->unit * c->vl_capacity + u->slot_of[p]) * (int64_t)HYQO_D;
    for (int d = 0; d < HYQO_D; ++d) {
      k[d] = hyqo_half_to_double(c->vl_k[base + d]);
      v[d] = hyqo_half_to_double(c->vl_v[base + d]);
    }
  } else { /* quantized majority */
    int64_t row = u->unit * c->capacity + p;
    hyqo_dequant_row(c->k_codes + row * HYQO_ROW_BYTES, c->k_sz + row * 8, k);
    hyqo_dequant_row(c->v_codes + row * HYQO_ROW_BYTES, c->v_sz + row * 8, v);
  }
}

/* Whether position p is in the unit's key/value multiset: every position of
 * [0, T) for the hybrid decode; for the vertical-only ablation only the
 * vertical-line positions and the window. */
static int in_multiset(const unit_view *u, int32_t p, int vl_only) {
  if (!vl_only) return 1;
  return p >= u->T - u->c->window || u->slot_of[p] >= 0;
}

/* softmax(q . k_p / sqrt(d)) weighted sum of v_p over the positions of the
 * multiset.  Two plain passes: logits and their max, then weights and the
 * sum. */
static void attend_one_head(const unit_view *u, const double *qd, int vl_only, double *o, double *lse) {
  int32_t T = u->T;
  double scale = 1.0 / sqrt((double)HYQO_D);
  double *logit = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  double k[HYQO_D], v[HYQO_D];
  double m = -INFINITY;
  int32_t n = 0; /* positions in the multiset */
  for (int32_t p = 0; p < T; ++p) {
    if (!in_multiset(u, p, vl_only)) continue;
    view_row(u, p, k, v);
    double s = 0.0;
    for (int d = 0; d < HYQO_D; ++d) s += qd[d] * k[d];
    logit[p] = s * scale;
    if (logit[p] > m) m = logit[p];
    ++n;
  }
  double l = 0.0;
  double acc[HYQO_D];
  for (int d = 0; d < HYQO_D; ++d) acc[d] = 0.0;
  for (int32_t p = 0; p < T; ++p) {
    if (!in_multiset(u, p, vl_only)) continue;
    view_row(u, p, k, v);
    double w = exp(logit[p] - m);
    l += w;
    for (int d = 0; d < HYQO_D; ++d) acc[d] += w * v[d];
  }
  for (int d = 0; d < HYQO_D; ++d) o[d] = (n > 0) ? acc[d] / l : 0.0;
  *lse = (n > 0) ? m + log(l) : -INFINITY;
  free(logit);
}

static int64_t n_units_of(const hyqo_cache *c) {
  return (int64_t)c->batch * c->n_kv_heads;
}

static int decode_units(const hyqo_cache *c, const uint16_t *q, const int32_t *units,
                        int32_t n_units, int vl_only, double *o, double *lse) {
  if (c->n_q_heads % c->n_kv_heads != 0) return -1;
  int G = c->n_q_heads / c->n_kv_heads;
  int64_t total = units ? n_units : n_units_of(c);
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t iu = 0; iu < total; ++iu) {
    int64_t unit = units ? units[iu] : iu;
    unit_view u;
    int rc = view_open(&u, c, unit);
    if (rc != 0) {
#pragma omp atomic write
      err = rc;
      if (rc != -9 && rc != -2) view_close(&u);
      continue;
    }
    for (int hg = 0; hg < G; ++hg) {
      int64_t h = (int64_t)u.b * c->n_q_heads + (int64_t)u.kvh * G + hg;
      double qd[HYQO_D], od[HYQO_D], l;
      for (int d = 0; d < HYQO_D; ++d) qd[d] = hyqo_half_to_double(q[h * HYQO_D + d]);
      attend_one_head(&u, qd, vl_only, od, &l);
      if (o)
        for (int d = 0; d < HYQO_D; ++d) o[h * HYQO_D + d] = od[d];
      if (lse) lse[h] = l;
    }
    view_close(&u);
  }
  return err;
}

int hyqo_decode(const hyqo_cache *c, const uint16_t *q, const int32_t *units,
                int32_t n_units, double *o, double *lse) {
  return decode_units(c, q, units, n_units, 0, o, lse);
}

int hyqo_decode_vl_only(const hyqo_cache *c, const uint16_t *q, const int32_t *units,
                        int32_t n_units, double *o, double *lse) {
  return decode_units(c, q, units, n_units, 1, o, lse);
}

int hyqo_decode_fp16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *seq_len, int32_t B, int32_t Hq, int32_t Hkv,
                     int32_t cap, const int32_t *units, int32_t n_units,
                     double *o, double *lse) {
  if (Hq % Hkv != 0) return -1;
  int G = Hq / Hkv;
  int64_t total = units ? n_units : (int64_t)B * Hkv;
  double scale = 1.0 / sqrt((double)HYQO_D);
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t iu = 0; iu < total; ++iu) {
    int64_t unit = units ? units[iu] : iu;
    int b = (int)(unit / Hkv), kvh = (int)(unit % Hkv);
    int32_t T = seq_len[b];
    if (T < 0 || T > cap) {
#pragma omp atomic write
      err = -2;
      continue;
    }
    const uint16_t *ku = k + unit * (int64_t)cap * HYQO_D;
    const uint16_t *vu = v + unit * (int64_t)cap * HYQO_D;
    double *logit = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int hg = 0; hg < G; ++hg) {
      int64_t h = (int64_t)b * Hq + (int64_t)kvh * G + hg;
      double qd[HYQO_D];
      for (int d = 0; d < HYQO_D; ++d) qd[d] = hyqo_half_to_double(q[h * HYQO_D + d]);
      double m = -INFINITY;
      for (int32_t p = 0; p < T; ++p) {
        double s = 0.0;
        for (int d = 0; d < HYQO_D; ++d) s += qd[d] * hyqo_half_to_double(ku[(int64_t)p * HYQO_D + d]);
        logit[p] = s * scale;
        if (logit[p] > m) m = logit[p];
      }
      double l = 0.0, acc[HYQO_D];
      for (int d = 0; d < HYQO_D; ++d) acc[d] = 0.0;
      for (int32_t p = 0; p < T; ++p) {
        double w = exp(logit[p] - m);
        l += w;
        for (int d = 0; d < HYQO_D; ++d) acc[d] += w * hyqo_half_to_double(vu[(int64_t)p * HYQO_D + d]);
      }
      if (o)
        for (int d = 0; d < HYQO_D; ++d) o[h * HYQO_D + d] = (T > 0) ? acc[d] / l : 0.0;
      if (lse) lse[h] = (T > 0) ? m + log(l) : -INFINITY;
    }
    free(logit);
  }
  return err;
}

/* ------------------------------------------------------------------------
 * Vertical-line selection.  Reading of the detector description: the last
 * n_q queries of every query head of the group are scored against all keys
 * (the pages' periodic matrix product), each query row is turned into
 * attention probabilities by a causal softmax, and the probabilities are
 * summed down each key column (the pages' column totals).  The k
 * largest column sums among positions older than the window are kept.
 * ---------------------------------------------------------------------- */
typedef struct {
  double cs;
  int32_t p;
} cand_t;

static int cand_cmp(const void *a, const void *b) {
  const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
  if (x->cs > y->cs) return -1;
  if (x->cs < y->cs) return 1;
  return (x->p < y->p) ? -1 : (x->p > y->p);
}

static int int_cmp(const void *a, const void *b) {
  int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x < y) ? -1 : (x > y);
}

int hyqo_select_vl(const hyqo_cache *c, const uint16_t *q_sel, int32_t n_q,
                   const uint16_t *k_full, int32_t k, const int32_t *units,
                   int32_t n_units, int32_t *out_pos, double *out_colsum,
                   double *margin) {
  if (c->n_q_heads % c->n_kv_heads != 0) return -1;
  int G = c->n_q_heads / c->n_kv_heads;
  int64_t total = units ? n_units : n_units_of(c);
  double scale = 1.0 / sqrt((double)HYQO_D);
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t iu = 0; iu < total; ++iu) {
    int64_t unit = units ? units[iu] : iu;
    unit_view u;
    int rc = view_open(&u, c, unit);
    int32_t T = u.T;
    int32_t n_cand = T - c->window;
    if (rc == 0 && (T < n_q || n_cand < k || k < 0)) rc = -6;
    if (rc != 0) {
#pragma omp atomic write
      err = rc;
      if (rc != -9 && rc != -2) view_close(&u);
      continue;
    }
    /* materialize the key view in fp64 */
    double *K = (double *)malloc(sizeof(double) * (size_t)T * HYQO_D);
    double vtmp[HYQO_D];
    for (int32_t p = 0; p < T; ++p) {
      if (k_full) {
        const uint16_t *kr = k_full + (unit * (int64_t)c->capacity + p) * HYQO_D;
        for (int d = 0; d < HYQO_D; ++d) K[(int64_t)p * HYQO_D + d] = hyqo_half_to_double(kr[d]);
      } else {
        view_row(&u, p, K + (int64_t)p * HYQO_D, vtmp);
      }
    }
    double *cs = (double *)calloc((size_t)(n_cand > 0 ? n_cand : 1), sizeof(double));
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    for (int hg = 0; hg < G; ++hg) {
      int64_t h = (int64_t)u.b * c->n_q_heads + (int64_t)u.kvh * G + hg;
      for (int32_t i = 0; i < n_q; ++i) {
        const uint16_t *qr = q_sel + (h * n_q + i) * HYQO_D;
        double qd[HYQO_D];
        for (int d = 0; d < HYQO_D; ++d) qd[d] = hyqo_half_to_double(qr[d]);
        int32_t last = T - n_q + i; /* causal: keys 0..last */
        double m = -INFINITY;
        for (int32_t p = 0; p <= last; ++p) {
          double acc = 0.0;
          for (int d = 0; d < HYQO_D; ++d) acc += qd[d] * K[(int64_t)p * HYQO_D + d];
          s[p] = acc * scale;
          if (s[p] > m) m = s[p];
        }
        double l = 0.0;
        for (int32_t p = 0; p <= last; ++p) l += exp(s[p] - m);
        for (int32_t p = 0; p < n_cand && p <= last; ++p) cs[p] += exp(s[p] - m) / l;
      }
    }
    cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_cand > 0 ? n_cand : 1));
    for (int32_t p = 0; p < n_cand; ++p) {
      cand[p].cs = cs[p];
      cand[p].p = p;
    }
    qsort(cand, (size_t)(n_cand > 0 ? n_cand : 0), sizeof(cand_t), cand_cmp);
    int32_t *dst = out_pos + unit * (int64_t)k;
    for (int32_t j = 0; j < k; ++j) dst[j] = cand[j].p;
    qsort(dst, (size_t)k, sizeof(int32_t), int_cmp);
    if (margin) {
      if (k == 0 || k >= n_cand)
        margin[unit] = 1.0;
      else
        margin[unit] = (cand[k - 1].cs - cand[k].cs) / cand[k - 1].cs;
    }
    if (out_colsum) {
      double *oc = out_colsum + unit * (int64_t)c->capacity;
      for (int32_t p = 0; p < c->capacity; ++p) oc[p] = (p < n_cand) ? cs[p] : 0.0;
    }
    free(cand);
    free(s);
    free(cs);
    free(K);
    view_close(&u);
  }
  return err;
}

/* ------------------------------------------------------------------------
 * Prefill hybrid-precision attention (the prefill operator).  Reading of
 * the pages (explainer "Two Operational Modes / Prefill Stage": the quantized
 * majority is computed first and the high-precision vertical lines and
 * local window are overlaid; wpnews: the bulk of query, key and value is
 * quantized): causal attention in which the pair (query row i, key j <= i)
 * is high precision when j is a vertical line or lies in the query's
 * sliding window (j > i - W), and then uses the FP16 q_i, k_j, v_j;
 * otherwise it uses the INT4-dequantized q_i, k_j, v_j (the cache's grid).
 * One softmax over all keys j <= i, scale 1/sqrt(128), in fp64.
 * ---------------------------------------------------------------------- */
static int quant_dequant(const uint16_t *x, double out[HYQO_D]) {
  uint8_t code[HYQO_D];
  uint16_t s[HYQO_NG], z[HYQO_NG];
  if (hyqo_quantize_row(x, code, s, z) != 0) return -1;
  for (int c = 0; c < HYQO_D; ++c) {
    int g = c / HYQO_GROUP;
    out[c] = hyqo_half_to_double(z[g]) + (double)code[c] * hyqo_half_to_double(s[g]);
  }
  return 0;
}

int hyqo_prefill_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const int32_t *seq_len, int32_t B, int32_t Hq, int32_t Hkv,
                           int32_t cap, int32_t W, const int32_t *vl_pos,
                           const int32_t *vl_count, int32_t vl_stride, double *o,
                           double *lse) {
  if (Hkv <= 0 || Hq % Hkv != 0 || W < 0) return -1;
  int G = Hq / Hkv;
  double scale = 1.0 / sqrt((double)HYQO_D);
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t uh = 0; uh < (int64_t)B * Hq; ++uh) {
    int b = (int)(uh / Hq), h = (int)(uh % Hq), kvh = h / G;
    int64_t unit = (int64_t)b * Hkv + kvh;
    int32_t T = seq_len[b];
    if (T < 0 || T > cap) {
#pragma omp atomic write
      err = -2;
      continue;
    }
    int32_t n = T > 0 ? T : 1;
    char *is_vl = (char *)calloc((size_t)n, 1);
    double *kq = (double *)malloc(sizeof(double) * (size_t)n * HYQO_D);
    double *vq = (double *)malloc(sizeof(double) * (size_t)n * HYQO_D);
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    int bad = 0;
    if (vl_pos && vl_count) {
      int32_t cnt = vl_count[unit];
      for (int32_t i = 0; i < cnt; ++i) {
        int32_t p = vl_pos[unit * vl_stride + i];
        if (p < 0 || p >= T) bad = 1;
        else is_vl[p] = 1;
      }
    }
    const uint16_t *ku = k + unit * (int64_t)cap * HYQO_D, *vu = v + unit * (int64_t)cap * HYQO_D;
    for (int32_t j = 0; j < T && !bad; ++j)
      if (quant_dequant(ku + (int64_t)j * HYQO_D, kq + (int64_t)j * HYQO_D) ||
          quant_dequant(vu + (int64_t)j * HYQO_D, vq + (int64_t)j * HYQO_D))
        bad = 1;
    const uint16_t *qh = q + ((int64_t)b * Hq + h) * (int64_t)cap * HYQO_D;
    for (int32_t i = 0; i < T && !bad; ++i) {
      double qf[HYQO_D], qq[HYQO_D];
      for (int d = 0; d < HYQO_D; ++d) qf[d] = hyqo_half_to_double(qh[(int64_t)i * HYQO_D + d]);
      if (quant_dequant(qh + (int64_t)i * HYQO_D, qq)) {
        bad = 1;
        break;
      }
      double m = -INFINITY;
      for (int32_t j = 0; j <= i; ++j) {
        int high = is_vl[j] || j > i - W;
        double sdot = 0.0;
        for (int d = 0; d < HYQO_D; ++d)
          sdot += high ? qf[d] * hyqo_half_to_double(ku[(int64_t)j * HYQO_D + d])
                       : qq[d] * kq[(int64_t)j * HYQO_D + d];
        w[j] = sdot * scale;
        if (w[j] > m) m = w[j];
      }
      double l = 0.0, acc[HYQO_D];
      for (int d = 0; d < HYQO_D; ++d) acc[d] = 0.0;
      for (int32_t j = 0; j <= i; ++j) {
        int high = is_vl[j] || j > i - W;
        double e = exp(w[j] - m);
        l += e;
        for (int d = 0; d < HYQO_D; ++d)
          acc[d] += e * (high ? hyqo_half_to_double(vu[(int64_t)j * HYQO_D + d]) : vq[(int64_t)j * HYQO_D + d]);
      }
      double *orow = o + (((int64_t)b * Hq + h) * cap + i) * HYQO_D;
      for (int d = 0; d < HYQO_D; ++d) orow[d] = acc[d] / l;
      if (lse) lse[((int64_t)b * Hq + h) * cap + i] = m + log(l);
    }
    if (bad) {
#pragma omp atomic write
      err = -3;
    }
    free(is_vl);
    free(kq);
    free(vq);
    free(w);
  }
  return err;
}

/*
 * hyq_oracle.h -- plain, slow CPU oracle for the HyQuant hybrid-precision
 * KV-cache decode path.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark call it; the CUDA library
 * never links, includes or calls it, and it includes no GPU header.
 *
 * Source of the method: "HyQuant: Hybrid-Precision Quantization for LLM
 * Attention" (arXiv 2608.27875), as described on
 *   - aifromscratch.in explainer, "How It Works" (three token classes: K_VL,
 *     K_Win = last 128 tokens, K_Q = 4-bit keys and values) and
 *     "Two Operational Modes / Decode Stage" (fused dequant + attention);
 *   - wpnews.pro summary (the vertical-line detector keeps recent queries and
 *     every 64 tokens scores them against the keys, totalling each column);
 *   - hotpaper.ai summary (vertical lines chosen by column totals of
 *     attention, under 5% of tokens).
 * Where the pages leave a step open (quantizer grid, scale format, softmax
 * before the column sum, GQA grouping, re-selection semantics) the reading
 * used is stated at each function below.
 *
 * Floating point: fp64 everywhere, except the quantizer, whose integer codes
 * are decided in IEEE fp32 with round-to-nearest-even (the precision the
 * quantizer definition fixes), compiled with -ffp-contract=off.
 *
 * Every function here has at least one pin in tests/ that does not reuse this
 * code (brute force, closed forms, library routines).
 */
#ifndef HYQ_ORACLE_H
#define HYQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HYQO_D 128     /* head_dim */
#define HYQO_GROUP 32  /* channels per quantization group */
#define HYQO_NG 4      /* groups per row */
#define HYQO_ROW_BYTES 64

/* ---- fp16 <-> wider conversions, written from the IEEE 754 binary16 format */
double hyqo_half_to_double(uint16_t h);
uint16_t hyqo_float_to_half(float f); /* round to nearest, ties to even */

/* ---- quantizer (one row of 128 fp16 values) ----------------------------
 * Per group g of 32 contiguous channels: mn, mx = min/max (fp32, exact);
 * s32 = fp32(mx - mn) / 15 in fp32; scale_h = fp16(s32);  zero_h = mn
 * (with -0 written as +0); sf = float(scale_h); code = 0 if sf == 0 else
 * clamp(rint_even(fp32(x - zero) / sf), 0, 15).
 * Returns 0, or -1 when the row holds a non-finite value (codes undefined). */
int hyqo_quantize_row(const uint16_t *x, uint8_t code[HYQO_D],
                      uint16_t scale_h[HYQO_NG], uint16_t zero_h[HYQO_NG]);

/* Byte position and nibble of channel c inside a 64-byte packed row (the
 * interchange format of the library's C ABI; see include/hyq.h). */
void hyqo_code_slot(int c, int *byte_index, int *high_nibble);

/* Quantize n rows (x[i*row_stride + c]) into packed codes [n][64] and
 * scale/zero [n][8] = {s0,z0,s1,z1,s2,z2,s3,z3}.  Returns the number of rows
 * that held a non-finite value (those rows are left as zero bytes). */
int64_t hyqo_pack(const uint16_t *x, int64_t n_rows, int64_t row_stride,
                  uint8_t *codes, uint16_t *sz);

/* Logical codes of one packed row, and the exact fp64 dequantization
 * x_hat = zero + code * scale. */
void hyqo_unpack_codes(const uint8_t *packed, uint8_t code[HYQO_D]);
void hyqo_dequant_row(const uint8_t *packed, const uint16_t *sz, double out[HYQO_D]);

/* ---- hybrid cache, host copy (same field meaning as the C ABI) --------- */
typedef struct {
  int32_t batch, n_q_heads, n_kv_heads, window, capacity, vl_capacity;
  const uint8_t *k_codes, *v_codes;   /* [B][Hkv][cap][64]     */
  const uint16_t *k_sz, *v_sz;        /* [B][Hkv][cap][8]      */
  const uint16_t *win_k, *win_v;      /* [B][Hkv][W][128], slot = pos % W */
  const uint16_t *vl_k, *vl_v;        /* [B][Hkv][vl_cap][128] */
  const int32_t *vl_pos;              /* [B][Hkv][vl_cap] ascending */
  const int32_t *vl_count;            /* [B][Hkv]              */
  const int32_t *seq_len;             /* [B]                   */
} hyqo_cache;

/* One decode step of GQA attention over the hybrid cache, for the listed
 * units (unit = b * Hkv + kv_head; units == NULL means all).  Key/value
 * multiset per unit: dequantized INT4 rows for p in [0, T-W) not in the VL
 * list, FP16 VL rows, FP16 window rows for p in [max(0,T-W), T).  Query head
 * h reads kv head h / G.  Scale 1/sqrt(128).  o: [B][Hq][128] fp64, lse:
 * [B][Hq] natural-log sum of exp of the scaled logits (either may be NULL).
 * Returns 0, or a negative code for an inconsistent cache. */
int hyqo_decode(const hyqo_cache *c, const uint16_t *q, const int32_t *units,
                int32_t n_units, double *o, double *lse);

/* The vertical-only ablation (AI Radio episode "HyQuant: Hybrid-Precision
 * Quantization for LLM Attention", "Paper Summary" and "Improvements and
 * Ablation Studies", Table twelve): hyqo_decode with the quantized majority
 * left out, i.e. attention over the VL rows and the window rows alone.  A
 * unit whose multiset is empty gets o = 0 and lse = -inf. */
int hyqo_decode_vl_only(const hyqo_cache *c, const uint16_t *q, const int32_t *units,
                        int32_t n_units, double *o, double *lse);

/* Prefill hybrid-precision attention (explainer "Two Operational Modes /
 * Prefill Stage"; wpnews: the bulk of query, key and value is quantized).
 * Causal attention; the pair (query row i, key j <= i) uses FP16 q, k, v
 * when j is a vertical line (vl_pos[unit][0..vl_count[unit]), NULL = none)
 * or j > i - W, and the INT4-dequantized q, k, v (the cache's quantizer)
 * otherwise.  q [B][Hq][cap][128], k/v [B][Hkv][cap][128] fp16, rows [0, T)
 * used; o [B][Hq][cap][128] fp64 and lse [B][Hq][cap] (nullable) written for
 * rows [0, T).  Returns 0, -1 (shapes), -2 (a length) or -3 (a vertical
 * line outside [0, T) or a non-finite row). */
int hyqo_prefill_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const int32_t *seq_len, int32_t B, int32_t Hq, int32_t Hkv,
                           int32_t cap, int32_t W, const int32_t *vl_pos,
                           const int32_t *vl_count, int32_t vl_stride, double *o,
                           double *lse);

/* Attention over an all-FP16 cache k, v: [B][Hkv][cap][128], T = seq_len[b]. */
int hyqo_decode_fp16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *seq_len, int32_t B, int32_t Hq, int32_t Hkv,
                     int32_t cap, const int32_t *units, int32_t n_units,
                     double *o, double *lse);

/* Vertical-line selection.  q_sel: [B][Hq][n_q][128]; query i of head h sits
 * at position T - n_q + i and sees keys p <= T - n_q + i.  Keys: k_full
 * ([B][Hkv][cap][128] fp16) when non-NULL (prefill mode), else the cache as
 * decode sees it.  For every row r = (i, h in the group): P = softmax of
 * (q . k) / sqrt(128); colsum[p] = sum over rows of P[r][p] for candidates
 * p in [0, T-W).  Top-k by (colsum desc, p asc), written ascending.
 * out_pos [B][Hkv][k]; out_colsum [B][Hkv][cap] (non-candidates 0);
 * margin [B][Hkv] = (cs_k - cs_{k+1}) / cs_k (1.0 when k == candidates).
 * Returns 0 or a negative code. */
int hyqo_select_vl(const hyqo_cache *c, const uint16_t *q_sel, int32_t n_q,
                   const uint16_t *k_full, int32_t k, const int32_t *units,
                   int32_t n_units, int32_t *out_pos, double *out_colsum,
                   double *margin);

#ifdef __cplusplus
}
#endif
#endif

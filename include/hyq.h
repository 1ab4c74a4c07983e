/*
 * hyq.h -- C ABI of libhyq.so: decode-stage attention over a hybrid
 * INT4/FP16 KV cache with fused dequantization (HyQuant), for NVIDIA B200
 * (sm_100a).
 *
 * The method ("HyQuant: Hybrid-Precision Quantization for LLM Attention",
 * arXiv 2608.27875): keys and values of most cached tokens are stored in
 * 4-bit form; a small set of vertical-line tokens (< 5% of positions, chosen
 * from column-summed attention scores of recent queries) and a local window
 * of the last 128 tokens stay in FP16; decode dequantizes on the fly inside
 * the attention kernel.  Sources: aifromscratch.in explainer, sections "How
 * It Works" (three token classes) and "Two Operational Modes / Decode Stage"
 * (fused dequantization); wpnews.pro summary (the detector keeps recent
 * queries and every 64 tokens scores them against the keys, totalling each
 * key's column); hotpaper.ai summary (selection by column totals of
 * attention, under 5% of tokens).
 *
 * Conventions for every entry point
 *   - Memory: every pointer is DEVICE memory owned by the caller, unless the
 *     argument says "host".  The library never allocates, frees or
 *     synchronizes.  Scratch space is passed in as a workspace whose size the
 *     matching *_workspace() query returns.
 *   - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  A return other than HYQ_OK means nothing was
 *     enqueued, except HYQ_ERR_CUDA, which reports a launch error.
 *   - Validation is synchronous and host-side (shapes, alignment, null
 *     pointers).  Conditions only the device can see (a sequence length out
 *     of range, a non-finite input to the quantizer, a bounded wait that ran
 *     out) are OR-ed into the optional device status word `dev_status`
 *     (uint32, HYQ_DEV_* bits) which the caller reads after synchronizing.
 *   - Alignment: every device pointer must be 16-byte aligned.
 *   - Fixed sizes: head_dim 128, quantization group 32, window 128;
 *     G = n_q_heads / n_kv_heads must be 1, 2, 4 or 8 (query head h reads
 *     KV head h / G).
 *   - Stateless and reentrant; the library caches the SM count per device.
 */
#ifndef HYQ_H
#define HYQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HYQ_OK = 0,
  HYQ_ERR_INVALID = 1,     /* bad argument: null pointer, shape, count */
  HYQ_ERR_UNSUPPORTED = 2, /* head_dim/group/window/G outside the fixed set */
  HYQ_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  HYQ_ERR_WORKSPACE = 4,   /* workspace missing or too small */
  HYQ_ERR_CUDA = 5         /* the CUDA runtime reported an error at launch */
} hyq_status;

/* device status word bits */
#define HYQ_DEV_NONFINITE 0x1u /* the quantizer saw Inf/NaN (codes undefined) */
#define HYQ_DEV_OOB 0x2u       /* an index check failed (debug build only)    */
#define HYQ_DEV_TIMEOUT 0x4u   /* a bounded wait expired; outputs undefined   */
#define HYQ_DEV_BADLEN 0x8u    /* seq_len / vl_count out of range; skipped    */

#define HYQ_HEAD_DIM 128
#define HYQ_GROUP 32
#define HYQ_WINDOW 128
#define HYQ_ROW_BYTES 64 /* packed INT4 codes per row (128 x 4 bit)        */
#define HYQ_SZ_BYTES 16  /* fp16 (scale, zero) x 4 groups per row           */

/*
 * Packed INT4 row format (64 bytes per row of 128 channels).  Channel c is in
 * group g = c / 32 at offset w = c % 32.  The row is 8 pieces of 8 bytes;
 * piece p = w / 4 holds channels 4p..4p+3 of every group.  Inside a piece,
 * byte 4*(g/2) + 2*j + (g%2), j = (w/2) % 2, holds channel w = 4p + 2j in its
 * low nibble and w = 4p + 2j + 1 in its high nibble.  (Chosen so that one
 * 16-byte load yields eight channels of every group and the nibble-to-fp16
 * conversion pairs two channels of one group per 32-bit word.)
 * Scale/zero row: fp16 {scale_0, zero_0, scale_1, zero_1, ..., zero_3}.
 *
 * Quantizer (the pages fix only the bit width, 4 bits for keys and for
 * values; this grid is fixed by the library): per group, mn/mx = min/max; scale =
 * fp16(fp32(mx - mn) / 15) with fp32 IEEE round-to-nearest-even; zero = mn
 * (a -0 minimum is stored as +0); code = 0 if scale == 0, else
 * clamp(round_half_even(fp32(x - zero) / fp32(scale)), 0, 15), computed with
 * IEEE fp32 subtraction and division (no FMA, no reciprocal).  Dequantized
 * value: zero + code * scale.
 */

/*
 * Quantized-majority blocks.  The INT4 part of a unit is stored in blocks of
 * 32 consecutive positions, each one contiguous HYQ_BLOCK_BYTES record, so a
 * decode tile is a single bulk copy:
 *   offset    0: K codes   [32][64]  (packed rows, format above)
 *   offset 2048: K scale/zero [32][8] fp16
 *   offset 2560: V codes, 2048 bytes: the packed rows of the 32 slots in
 *                position pairs.  Word h (0, 1) of piece p (0..7) of slot t
 *                (format above) has its low 16 bits at byte
 *                128 i + 16 (p xor 2 (i mod 4)) + 8 h + 2 s of this area,
 *                i = t / 2, and its high 16 bits 4 bytes further,
 *                s = (t mod 2) xor ((t / 4) mod 2):
 *                the two slots of a pair share every 32-bit word, so the
 *                decode reads the P.V operands of both with one 16-byte
 *                load.  (hyq_pack writes plain rows; only the cache's
 *                records use this order.)
 *   offset 4608: V scale/zero [32][8] fp16
 *   offset 5120: uint32 vertical-line bitmask: bit i set exactly when
 *                position 32*b + i is held in FP16 in the vertical-line rows
 *   offset 5124: 12 bytes of padding (keeps records 16-byte aligned)
 */
#define HYQ_BLOCK_TOKENS 32
#define HYQ_BLOCK_BYTES 5136
#define HYQ_BLK_KCODES 0
#define HYQ_BLK_KSZ 2048
#define HYQ_BLK_VCODES 2560
#define HYQ_BLK_VSZ 4608
#define HYQ_BLK_MASK 5120

/*
 * The hybrid cache of one layer.  All arrays are caller-owned device memory
 * and must be zero-filled before first use.  Per unit u = b * n_kv_heads + h:
 *   quantized majority  positions [0, T - window): blocks
 *                       [B][Hkv][capacity/32][HYQ_BLOCK_BYTES], position p
 *                       in block p / 32, slot p % 32;
 *   vertical-line rows  vl_k/vl_v [B][Hkv][vl_capacity][128] fp16, in the
 *                       ascending order of vl_pos [B][Hkv][vl_capacity];
 *                       vl_count [B][Hkv] rows are valid, and the block
 *                       bitmasks mark exactly these positions;
 *   local window        win_k/win_v [B][Hkv][window][128] fp16, position p
 *                       in slot p % window, positions [max(0, T-window), T);
 *   seq_len [B] int32   T, the number of positions, newest token included.
 */
typedef struct {
  int32_t batch, n_q_heads, n_kv_heads;
  int32_t head_dim;    /* must be 128 */
  int32_t group;       /* must be 32  */
  int32_t window;      /* must be 128 */
  int32_t capacity;    /* max positions per sequence, multiple of 128 */
  int32_t vl_capacity; /* max vertical-line rows per unit, >= 1 */
  uint8_t *blocks;
  void *win_k, *win_v;
  void *vl_k, *vl_v;
  int32_t *vl_pos;
  int32_t *vl_count;
  int32_t *seq_len;
  uint32_t *dev_status; /* nullable */
  /* Staged promotion (optional): the FP16 K/V rows of the stage_rows most
   * recently quantized positions [T - window - stage_rows, T - window) of
   * every unit, [B][Hkv][stage_rows][128] fp16, position p in slot
   * p % stage_rows.  hyq_prefill fills it from the prompt; hyq_append and
   * hyq_decode_step write the row leaving the window; a cache-mode
   * hyq_vl_apply promotes newly selected positions from it.  stage_rows = 0
   * turns it off (stage_k / stage_v may then be NULL). */
  void *stage_k, *stage_v;
  int32_t stage_rows; /* 0, or 1..1024 */
  /* Paged quantized majority (optional).  NULL: `blocks` holds each unit's
   * capacity/32 records contiguously (layout above).  Non-NULL: `blocks` is
   * a pool of n_pages pages of n_kv_heads records each (page g, KV head h
   * at record g * n_kv_heads + h), and sequence b's positions
   * [32 j, 32 j + 32) live in page block_table[b * (capacity/32) + j]
   * (int32 [B][capacity/32], device; pages may be shared only by sequences
   * that never write them).  An entry outside [0, n_pages) that a kernel
   * needs raises HYQ_DEV_BADLEN: reads go to page 0, writes are skipped. */
  int32_t *block_table;
  int32_t n_pages; /* >= 1 when block_table is set */
} hyq_cache;

/*
 * hyq_pack -- quantize FP16 rows to packed INT4 codes and fp16 scale/zero
 * (the KV-cache compression of the decode stage), into plain row arrays.
 * Method: aifromscratch.in explainer, "How It Works" (keys and values of the
 * long-tail tokens are kept in 4 bits) and "Two Operational Modes / Decode
 * Stage" (the cache is compressed to 4 bits as decoding proceeds); the grid
 * itself is the library's (quantizer above), since the pages fix only the
 * bit width.
 *   x          fp16 rows, row i at x + i*row_stride (elements), 128 values
 *   n_rows     >= 0 (0 enqueues nothing)
 *   row_stride >= 128, multiple of 8
 *   dst_rows   nullable int64 [n_rows]: row i goes to output row dst_rows[i]
 *              (scatter); NULL means row i -> row i
 *   codes      u8 [*][64] output; sz fp16 [*][8] output
 *   dev_status nullable; HYQ_DEV_NONFINITE is set for a row holding Inf/NaN
 */
hyq_status hyq_pack(const void *x, int64_t n_rows, int64_t row_stride,
                    const int64_t *dst_rows, uint8_t *codes, void *sz,
                    uint32_t *dev_status, void *stream);

/*
 * hyq_prefill -- build the cache from a prompt (end of prefill).  Method:
 * aifromscratch.in explainer, "How It Works" (three token classes: the
 * quantized majority, the vertical lines and the local window of the last
 * 128 tokens, kept in FP16) and "Two Operational Modes / Prefill Stage".
 * For every
 * unit with T = seq_len[b] (device): rows [0, T - window) of k_full/v_full
 * are quantized into the blocks (as hyq_pack), rows [max(0, T - window), T)
 * are copied into the window ring, and the vertical-line set is emptied
 * (vl_count = 0, every block bitmask cleared).
 *   k_full, v_full  fp16 [B][Hkv][capacity][128]
 * Sets HYQ_DEV_BADLEN (and skips the batch) when T is outside [0, capacity];
 * HYQ_DEV_NONFINITE as hyq_pack.
 */
hyq_status hyq_prefill(const hyq_cache *c, const void *k_full, const void *v_full,
                       void *stream);

/*
 * hyq_append -- add one token per sequence to the cache (decode step).
 * Method: aifromscratch.in explainer, "Two Operational Modes / Decode Stage"
 * (the token that leaves the local window is compressed to 4 bits as
 * decoding proceeds); wpnews.pro summary (the detector accumulates the
 * recent queries it scores every 64 tokens).
 * For every batch b with T = seq_len[b]: the row leaving the window
 * (position T - window, when T >= window) is packed into the codes, the new
 * K/V row takes window slot T % window, and seq_len[b] becomes T + 1.
 *   k_new, v_new  fp16 [B][Hkv][128]
 *   q_new, q_ring nullable together: q_new fp16 [B][Hq][128] is copied to
 *                 q_ring fp16 [B][Hq][n_q][128] at slot T % n_q (the ring of
 *                 recent queries the vertical-line detector accumulates)
 * Sets HYQ_DEV_BADLEN (and skips the batch) when T + 1 > capacity.
 */
hyq_status hyq_append(const hyq_cache *c, const void *k_new, const void *v_new,
                      const void *q_new, void *q_ring, int32_t n_q, void *stream);

/*
 * hyq_select_vl -- vertical-line detector.  Method: wpnews.pro summary (the
 * recent queries are kept and, every 64 tokens, multiplied against the keys,
 * after which each key's column is totalled); hotpaper.ai summary (the
 * vertical-line tokens, under 5% of positions, are those with the largest
 * column totals of attention); aifromscratch.in explainer, "What to Watch
 * For" (a top-5% cut).  For every unit, the n_q most
 * recent queries of each of its G query heads (R = n_q * G rows) are scored
 * against the keys; query i sits at position T - n_q + i and sees keys
 * p <= T - n_q + i.  Each row becomes a softmax over (q . k) / sqrt(128);
 * the probabilities are summed down each key column; the k largest column
 * sums among positions [0, T - window) are returned, ties to the lower
 * position, in ascending order.
 *   q_sel      fp16 [B][Hq][n_q][128]; q_is_ring = 0: row i at index i;
 *              q_is_ring = 1: the row of position p at index p % n_q (the
 *              layout hyq_append writes)
 *   n_q        1..64 (64 in the method)
 *   k_full     nullable fp16 [B][Hkv][capacity][128]: score these keys
 *              (prefill); NULL scores the cache as decode sees it
 *   k          number of positions to select, 0 <= k <= vl_capacity;
 *              a unit whose T - window < k sets HYQ_DEV_BADLEN
 *   out_pos    int32 [B][Hkv][k]
 *   out_colsum nullable fp32 [B][Hkv][capacity] (non-candidates 0)
 *   ws         workspace of hyq_select_vl_workspace(c, n_q) bytes
 * Requires window >= n_q.
 */
size_t hyq_select_vl_workspace(const hyq_cache *c, int32_t n_q);
hyq_status hyq_select_vl(const hyq_cache *c, const void *q_sel, int32_t n_q,
                         int32_t q_is_ring, const void *k_full, int32_t k,
                         int32_t *out_pos, float *out_colsum, void *ws,
                         size_t ws_bytes, void *stream);

/*
 * hyq_vl_apply -- make `pos` the vertical-line set.  Method: aifromscratch.in
 * explainer, "How It Works" (the vertical-line tokens keep their keys and
 * values in FP16); wpnews.pro summary (the set is re-chosen every 64 tokens).
 *   pos        int32 [B][Hkv][k], ascending, within [0, T - window)
 *   k_full/v_full  non-NULL (prefill): the FP16 rows are gathered from
 *              these [B][Hkv][capacity][128] arrays.  NULL (cache mode):
 *              positions already held in FP16 keep their rows, positions
 *              no longer selected fall back to their INT4 codes, and newly
 *              selected positions, whose FP16 copy is gone, stay INT4 and
 *              are counted in *n_unpromoted (nullable device int32,
 *              accumulated with atomicAdd; zero it first).  With staging
 *              (stage_rows > 0), a newly selected position still in the
 *              staging ring and newer than every position kept from the
 *              previous set is promoted with its staged FP16 rows (the
 *              promoted rows follow the kept rows).
 * Rows move only towards lower slots, so the update is done in place.
 */
hyq_status hyq_vl_apply(const hyq_cache *c, const int32_t *pos, int32_t k,
                        const void *k_full, const void *v_full,
                        int32_t *n_unpromoted, void *stream);

/*
 * hyq_decode -- one decode step of GQA attention over the hybrid cache.
 * Method: aifromscratch.in explainer, "Two Operational Modes / Decode Stage"
 * (the 4-bit cache is decompressed inside the attention computation, with
 * no FP16 copy written back) and "How It Works" (attention over the
 * quantized keys, the vertical lines and the window together).  INT4
 * dequantization is fused into the attention (split-KV flash decoding:
 * work is spread over n_ctas thread blocks by bytes read, per-block partial
 * (max, sum, accumulator) triples are merged by log-sum-exp in the last
 * block to finish a unit).
 *   q    fp16 [B][Hq][128]; o fp16 [B][Hq][128] output
 *   lse  nullable fp32 [B][Hq]: natural-log sum of exp of the scaled logits
 *   n_ctas  thread blocks; 0 = automatic (one per SM)
 *   ws   workspace of hyq_decode_workspace(c, n_ctas) bytes; zero-filled
 *        before the first call, every completed call leaves it reusable
 *        (re-zero it after a call that reported HYQ_DEV_TIMEOUT)
 * Scale 1/sqrt(128); all softmax arithmetic in fp32.
 * HYQ_ERR_UNSUPPORTED when batch x n_kv_heads > 4096, or when the launch's
 * work, counted as 5 per 32 capacity positions plus 4 per 8 rows of
 * vl_capacity and window, reaches 2^31 over all units.
 */
size_t hyq_decode_workspace(const hyq_cache *c, int32_t n_ctas);
hyq_status hyq_decode(const hyq_cache *c, const void *q, void *o, float *lse,
                      int32_t n_ctas, void *ws, size_t ws_bytes, void *stream);

/*
 * hyq_decode_vl_only -- the vertical-only ablation of hyq_decode: attention
 * over the cache's vertical-line rows and local window alone, with the INT4
 * majority left out (the sparse-attention variant that drops the long-tail
 * positions).  Method: AI Radio episode "HyQuant: Hybrid-Precision
 * Quantization for LLM Attention", "Paper Summary" (vertical-only variants
 * discard the long-tail positions that HyQuant keeps in low precision) and
 * "Improvements and Ablation Studies" (Table twelve compares the two).
 * Arguments, workspace (hyq_decode_workspace) and errors as hyq_decode; the
 * cache is only read.  A unit with no vertical line and an empty window
 * gets o = 0, lse = -inf.
 */
hyq_status hyq_decode_vl_only(const hyq_cache *c, const void *q, void *o, float *lse,
                              int32_t n_ctas, void *ws, size_t ws_bytes, void *stream);

/*
 * hyq_decode_step -- one whole decode step in a single launch: the append of
 * hyq_append(c, k_new, v_new, q, q_ring, n_q) fused into hyq_decode(c, q,
 * o, lse).  Results (o, lse, and the cache, ring and seq_len after the
 * call) are identical to the two calls in sequence.  Method: HyQuant,
 * "Two Operational Modes / Decode Stage" (the token leaving the local window
 * is compressed to 4 bits as decoding proceeds) and "How It Works" (the
 * decode attention over K_Q, K_VL and K_Win).
 *   q      fp16 [B][Hq][128]: the new token's queries (decoded and, when
 *          q_ring is non-NULL, stored in ring slot T % n_q)
 *   k_new, v_new  fp16 [B][Hkv][128]: the new token's key and value rows
 *   q_ring nullable fp16 [B][Hq][n_q][128]; n_q in [1, 1024] when non-NULL
 *   o, lse, n_ctas as hyq_decode
 *   ws     workspace of hyq_decode_step_workspace(c, n_ctas) bytes, zero-
 *          filled before the first call and left reusable by every
 *          completed call
 * A sequence whose length would pass capacity is not appended: its rows get
 * o = 0, lse = -inf and HYQ_DEV_BADLEN is raised (hyq_append leaves such a
 * sequence unchanged too).  Errors as hyq_decode.
 */
size_t hyq_decode_step_workspace(const hyq_cache *c, int32_t n_ctas);
hyq_status hyq_decode_step(const hyq_cache *c, const void *q, const void *k_new,
                           const void *v_new, void *q_ring, int32_t n_q, void *o,
                           float *lse, int32_t n_ctas, void *ws, size_t ws_bytes,
                           void *stream);

/*
 * hyq_decode_noalloc -- hyq_decode without a workspace argument, for callers
 * that cannot allocate device memory: for example a plugin inside a host
 * application whose own allocator owns the whole GPU memory budget and does
 * not let plugins call cudaMalloc, or a caller bound to a fixed C interface
 * with no way to carry a workspace pointer.  There is no counterpart in the
 * paper; this is a deployment convenience of the library.
 *   Arguments as hyq_decode (n_ctas is the automatic choice).
 *   Scratch: a fixed array compiled into the library (2,719,744 bytes), which
 *   every GPU that loads the library keeps until the process exits.  Limits:
 *   batch x n_kv_heads <= 4096, automatic block count <= 320, G <= 8;
 *   larger shapes return HYQ_ERR_UNSUPPORTED without enqueuing anything.
 *   The first call on a device looks up the array's device address (once
 *   per device and CUDA context, with that device current; a
 *   cudaDeviceReset makes the next call look it up again); make that first
 *   call before any stream capture.  Every call clears the array's counters
 *   (cudaMemsetAsync on `stream`) and then launches the decode.
 *   All calls share the one array: two calls whose work overlaps on the GPU
 *   (different streams, or different host threads on one device) race and
 *   give undefined results.  Serialize them on one stream.
 *   Never allocates or frees memory.
 */
hyq_status hyq_decode_noalloc(const hyq_cache *c, const void *q, void *o, float *lse,
                              void *stream);

/*
 * hyq_decode_fp16 -- the same decode kernel design over an all-FP16 cache
 * (the full-precision comparator).  Method: aifromscratch.in explainer, "Key
 * Results & Benchmarks" (HyQuant's decode kernel is measured against a
 * full-precision FlashAttention-2 baseline).
 *   q fp16 [B][Hq][128]; k, v fp16 [B][Hkv][capacity][128]; seq_len int32 [B]
 *   o fp16 [B][Hq][128]; lse nullable fp32 [B][Hq]
 *   ws   workspace of hyq_decode_fp16_workspace(B, Hq, Hkv, n_ctas) bytes,
 *        zero-filled before the first call
 * HYQ_ERR_UNSUPPORTED when batch x n_kv_heads > 4096 or when
 * batch x n_kv_heads x 4 x ceil(capacity / 8) reaches 2^31.
 */
size_t hyq_decode_fp16_workspace(int32_t batch, int32_t n_q_heads,
                                 int32_t n_kv_heads, int32_t n_ctas);
hyq_status hyq_decode_fp16(const void *q, const void *k, const void *v,
                           const int32_t *seq_len, int32_t batch,
                           int32_t n_q_heads, int32_t n_kv_heads,
                           int32_t capacity, void *o, float *lse,
                           int32_t n_ctas, void *ws, size_t ws_bytes,
                           uint32_t *dev_status, void *stream);

/*
 * hyq_prefill_attention -- the prefill-stage hybrid-precision attention
 * operator: causal GQA attention of a prompt over itself in which most
 * (query, key) pairs are computed from INT4-quantized queries, keys and
 * values while the vertical-line keys and each query's local window stay in
 * FP16, in one softmax per query row.  Method: aifromscratch.in explainer,
 * "Two Operational Modes / Prefill Stage" (a fused operator computes the
 * quantized majority and overlays the high-precision vertical lines and
 * local window into the same result); wpnews.pro summary (the bulk of the
 * query, key and value tensors is quantized, vertical-line tokens and a
 * local sliding window stay in full precision); kipquest.com abstract (the
 * prefill stage's hybrid-precision quantized attention operator).
 * Definition used (the pages give no formula): for query row i and key
 * j <= i, the pair is high precision when j is one of the unit's vertical
 * lines or j > i - window, and then uses the FP16 q_i, k_j, v_j; otherwise
 * it uses q_i, k_j, v_j quantized on the grid above and dequantized.  Scale
 * 1/sqrt(128), natural-log LSE.
 *   q       fp16 [B][Hq][capacity][128]: the prompt's queries, row p =
 *           position p
 *   k_full, v_full  fp16 [B][Hkv][capacity][128]: the prompt's keys, values
 *   o       fp32 [B][Hq][capacity][128] output (rows >= T untouched)
 *   lse     nullable fp32 [B][Hq][capacity]
 *   ws      workspace of hyq_prefill_attention_workspace(c) bytes (the
 *           dequantized operands: about (4 Hq + 8 Hkv) x capacity x 128
 *           bytes per sequence; no zeroing needed)
 * The cache supplies T = seq_len[b] and the vertical-line set (vl_pos,
 * vl_count and the block bitmasks as hyq_prefill + hyq_vl_apply leave
 * them); it is only read.  Device-side: HYQ_DEV_BADLEN for T outside
 * [0, capacity] or a bad vl_count (the sequence or its set is skipped),
 * HYQ_DEV_NONFINITE for a non-finite input row, HYQ_DEV_TIMEOUT if a wait
 * for the tensor cores runs out (outputs undefined).
 */
size_t hyq_prefill_attention_workspace(const hyq_cache *c);
hyq_status hyq_prefill_attention(const hyq_cache *c, const void *q, const void *k_full,
                                 const void *v_full, float *o, float *lse, void *ws,
                                 size_t ws_bytes, void *stream);

/*
 * hyq_copy -- copy `bytes` from src to dst on `stream` with a kernel of the
 * library: the transfer of a decode step's inputs (q, k_new, v_new) from
 * pinned host memory to the device and of its output o back, without the
 * copy engine, so the step kernel keeps its programmatic launch overlap
 * with the copy before it (not part of the method; plumbing for the
 * end-to-end loop).
 *   dst, src   device memory, or page-locked host memory mapped for the
 *              device (cudaHostAlloc / cudaMallocHost under unified
 *              addressing); 16-byte aligned
 *   bytes      a multiple of 16 (0 enqueues nothing; the pointers must
 *              still be non-null)
 * Ordered after the previous work on the stream, like cudaMemcpyAsync.
 * HYQ_ERR_INVALID (nothing enqueued) for a null pointer, a size that is
 * not a multiple of 16, or a pointer the device cannot dereference
 * (pageable host memory, page-locked memory that is not mapped);
 * HYQ_ERR_ALIGN for a misaligned pointer.
 */
hyq_status hyq_copy(void *dst, const void *src, size_t bytes, void *stream);

/* Human-readable name of a status code (static storage). */
const char *hyq_status_string(hyq_status s);

/* Number of thread blocks n_ctas = 0 selects for the decode kernels on the
 * current device (host query; needs a current CUDA device). */
int32_t hyq_decode_default_ctas(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int32_t hyq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HYQ_H */

// hyq_select.cu -- vertical-line detector: score the last n_q queries of a
// unit's G query heads against its keys, softmax each query row, sum the
// probabilities down every key column, keep the k largest column sums.
//
// Method: HyQuant.  wpnews.pro summary: the detector collects the recent
// queries and, every 64 tokens, multiplies them against the keys and adds
// up each key's column; hotpaper.ai summary: the vertical-line tokens, under
// 5% of all, are the keys with the largest column totals of attention;
// aifromscratch.in explainer, "What to Watch For": a top-5% cut.  Readings (the pages
// are silent): the scores are post-softmax probabilities with scale
// 1/sqrt(128); the column sum runs over the 64 queries and the G query heads
// that share the KV head; query i sits at position T - n_q + i and sees keys
// p <= T - n_q + i; candidates are positions older than the local window;
// ties at the k-th value go to the lower position.
//
// Kernels (one launch each, stream ordered):
//   0. rank_kernel       (cache mode only) grid (units): per bitmask word of
//      the unit, the number of vertical-line rows before it, so the scorer
//      finds the FP16 row of a vertical-line key without a search.
//   1. score_kernel<.,1> persistent, one block per SM over (unit, 512-key
//      chunk) items: S = Q K^T on the tcgen05 tensor cores (fp16 operands in
//      shared memory, fp32 accumulators in tensor memory), query rows on M;
//      per row the running max / sum of exp over the chunk's causal keys.
//   2. stats_merge_kernel grid (units): log-sum-exp merge of the chunk
//      partials in a fixed order -> (m_r, 1 / l_r).
//   3. score_kernel<.,2> the same walk with keys on M: S again for candidate
//      keys, P = exp2(S - m_r) / l_r, each thread sums one key column over
//      the rows in a fixed order (no float atomics), so equal key columns
//      give bitwise-equal sums.
//   4. topk_cluster_kernel  one cluster of 8 blocks per unit (each block a
//      slice of the positions): exact radix select on the fp32 bit patterns
//      (non-negative floats order like their bits), histograms and counts
//      combined through distributed shared memory, ties to lower positions,
//      output compacted in ascending position order; topk_kernel (one block
//      per unit) does the same when a slice would not fit shared memory.
// Keys come from k_full (prefill) or from the cache as decode sees it: FP16
// window and vertical-line rows, and INT4 rows dequantized as
// zero + code * scale in fp32 and split into two fp16 terms hi + lo (both
// multiplied on the tensor cores) so the dequantized key keeps ~22 bits.
#include <algorithm>

#include "hyq_common.cuh"

extern "C" int32_t hyq_sm_count(void);  // hyq_api.cu

namespace hyq {

static int hyq_sm_count_dev() { return hyq_sm_count(); }

constexpr int SEL_KC = 512;       // keys per work item (chunk)
constexpr int SEL_MAX_ROWS = 512; // n_q * G
constexpr int SEL_BLOCK_ROWS = SEL_MAX_ROWS;  // every query row of a unit in one block
constexpr int TOPK_THREADS = 1024;
constexpr float SEL_SCALE = 0.12751743082459868f;  // log2(e) / sqrt(128)

struct SelectArgs {
  int B, Hq, Hkv, G, n_q, q_ring, cap, W, vl_cap, U, R, k, n_chunks;
  const __half *q;       // [B][Hq][n_q][128]
  const __half *k_full;  // nullable [B][Hkv][cap][128]
  const uint8_t *blocks;  // quantized majority + bitmask, [U][cap/32][BLK_BYTES] or a page pool
  RecMap rm;              // record addresses (contiguous or through the block table)
  const __half *win_k, *vl_k;
  const int32_t *vl_pos, *vl_count;
  const int32_t *seq_len;
  float2 *stats_part;  // [U][n_chunks][SEL_MAX_ROWS]
  float2 *stats;       // [U][SEL_MAX_ROWS]  (m, 1/l)
  float *colsum_part;  // [n_rb][U][cap]  per row block
  float *colsum;       // [U][cap]  final column sums
  int n_rb;            // row blocks: ceil(R / SEL_BLOCK_ROWS)
  int32_t *rank_base;  // [U][cap/32]: vertical-line rows before each mask word
  int32_t *out_pos;    // [U][k]
  uint32_t *status;
};

__device__ __forceinline__ int sel_T(const SelectArgs &a, int u) { return a.seq_len[u / a.Hkv]; }

// ---------------------------------------------------------------- scorer
// S = Q K^T on the 5th-generation tensor cores (tcgen05, fp16 in, fp32
// accumulate in tensor memory).  One block of 16 warps per SM walks the
// (unit, 512-key chunk) items.  Per unit the R query rows sit in shared
// memory as row blocks of 128 (the MMA's M); per sub-tile of 128 keys (the
// MMA's N) the keys are written to shared memory as fp16 -- in cache mode an
// INT4 key is dequantized as zero + code * scale in fp32 and stored as
// hi + lo fp16 (both multiplied, so the key keeps ~22 bits), FP16 keys as
// they are -- and one thread issues the MMAs into the accumulators (one per
// row block, 128 columns each) and commits them to an mbarrier.  Both
// operands are K-major with the 128-byte swizzle.  The epilogue reads the
// accumulators with tcgen05.ld: warp w owns rows 32 (w % 4) .. + 31 of each
// row block and columns 64 (w / 4) .. + 63 of the sub-tile.
constexpr int TC_THREADS = 512;  // 16 warps: 4 lane quadrants x 4 column quarters
constexpr int TC_BLOCK = TC_THREADS + 32;  // and one warp that issues the MMAs
constexpr int TC_NK = 128;               // keys per sub-tile
constexpr int TC_TILE = TC_NK * 256;     // bytes of a [128][128] fp16 tile
constexpr int TC_MAX_RB = SEL_MAX_ROWS / 128;

// Byte offset of element (row r, channel k) in a [128][128] fp16 K-major tile
// with the 128-byte swizzle: channels 0-63 and 64-127 form two 16 KB halves;
// within a half, row r is 128 bytes at r * 128 and its 16-byte chunk c sits
// at position c ^ (r % 8).
__device__ __forceinline__ uint32_t sw128_off(int r, int k) {
  const int kb = k >> 6, chunk = (k & 63) >> 3;
  return kb * (TC_NK * 128) + r * 128 + ((chunk ^ (r & 7)) << 4) + (k & 7) * 2;
}
// Shared-memory matrix descriptor of k-step ks (16 channels) of such a tile:
// start address, leading offset 16 B (unused with the swizzle), stride 1024 B
// between 8-row groups, descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t tile, int ks) {
  const uint32_t start = tile + (ks >> 2) * (TC_NK * 128) + (ks & 3) * 32;
  return static_cast<uint64_t>((start >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}
// sw128_desc(tile, ks) - sw128_desc(tile, 0) in the start-address field.
__device__ __forceinline__ uint32_t sw128_koff(int ks) { return (ks >> 2) * (TC_NK * 128 / 16) + (ks & 3) * 2; }
// Instruction descriptor: fp32 accumulate, fp16 A and B, both K-major,
// N = 128, M = 128.
constexpr uint32_t TC_IDESC = (1u << 4) | ((uint32_t)(TC_NK >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t ad, uint64_t bd, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(TC_IDESC), "r"(accumulate), "r"(0u));
}
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// One quantization group (32 channels) of a key row as key_store writes it:
// FP16 (window, vertical line, prefill) as 4 x 16 B, INT4 as the packed
// row (4 x 16 B) plus the group's (scale, zero).
struct KeyRaw {
  uint4 v[4];
  uint32_t sz;
  int kind;  // 0 zero, 1 FP16, 2 INT4
};

// Two quantization groups g and g + 2 of one key row, loaded once: FP16 as
// 2 x 4 x 16 B, INT4 as the 64-byte packed row (all groups) plus the two
// groups' (scale, zero).
struct KeyRaw2 {
  uint4 v[8];
  uint32_t sz[2];
  int kind;  // 0 zero, 1 FP16, 2 INT4
};

template <bool CACHE>
__device__ __forceinline__ void key_load2(const SelectArgs &a, int u, int T, int key, int key_end, int g,
                                          KeyRaw2 &r) {
  r.kind = 0;
  if (key >= key_end) return;
  const __half *row = nullptr;
  int64_t rec = 0;
  if (!CACHE) {
    row = a.k_full + (static_cast<int64_t>(u) * a.cap + key) * D;
  } else if (key >= T - a.W) {
    row = a.win_k + (static_cast<int64_t>(u) * a.W + key % a.W) * D;
  } else {
    // a vertical line: its row is the rank of its bit among the unit's set bits
    rec = a.rm.rec_rd(u, key);
    const uint32_t w = *reinterpret_cast<const uint32_t *>(a.blocks + rec_mask(rec));
    if ((w >> (key & 31)) & 1u) {
      const int slot = a.rank_base[static_cast<int64_t>(u) * (a.cap / 32) + (key >> 5)] +
                       __popc(w & ((1u << (key & 31)) - 1u));
      row = a.vl_k + (static_cast<int64_t>(u) * a.vl_cap + slot) * D;
    }
  }
  if (row) {
    r.kind = 1;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      r.v[c] = *reinterpret_cast<const uint4 *>(row + 32 * g + 8 * c);
      r.v[4 + c] = *reinterpret_cast<const uint4 *>(row + 32 * (g + 2) + 8 * c);
    }
    return;
  }
  r.kind = 2;
  const uint4 *codes = reinterpret_cast<const uint4 *>(a.blocks + rec_kcode(rec, key));
#pragma unroll
  for (int c = 0; c < 4; ++c) r.v[c] = codes[c];
  const uint32_t *sz = reinterpret_cast<const uint32_t *>(a.blocks + rec_ksz(rec, key));
  r.sz[0] = sz[g];
  r.sz[1] = sz[g + 2];
}

// Write the thread's 4 chunks of key row kk as fp16 (hi) and, in cache mode,
// the fp16 remainder (lo).  INT4: x = zero + code * scale in fp32 (one
// rounding), hi = fp16(x), lo = fp16(x - hi).
template <bool CACHE>
__device__ __forceinline__ void key_store(const KeyRaw &r, int kk, int hf, uint8_t *hi, uint8_t *lo) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = 4 * hf + cc;  // 16-byte chunk = channels 8c .. 8c+7, group hf
    uint4 h = make_uint4(0, 0, 0, 0), l = make_uint4(0, 0, 0, 0);
    if (r.kind == 1) {
      h = r.v[cc];
    } else if (CACHE && r.kind == 2) {
      // channels 8c .. 8c+7 are group g = c / 4, pieces 2 (c % 4) and
      // 2 (c % 4) + 1, i.e. the 16 bytes at 16 (c % 4); word g / 2 of each
      // 8-byte piece, byte (g % 2) of each of its channel pairs
      const int g = c >> 2, hh = g >> 1, ii = g & 1, pc = c & 3;
      const uint4 vv = r.v[pc];
      const uint32_t wp0 = hh ? vv.y : vv.x;  // piece 2pc, word hh
      const uint32_t wp1 = hh ? vv.w : vv.z;  // piece 2pc + 1, word hh
      const __half2 sz = u2h(r.sz);  // group g == hf
      const float sc = __low2float(sz), zr = __high2float(sz);
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const uint32_t w = s2 ? wp1 : wp0;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const uint32_t byte = (w >> (8 * (2 * jj + ii))) & 0xFFu;  // channels 2jj (lo), 2jj+1 (hi)
          const float x0 = fmaf(static_cast<float>(byte & 15u), sc, zr);
          const float x1 = fmaf(static_cast<float>(byte >> 4), sc, zr);
          const __half2 hv = __floats2half2_rn(x0, x1);
          const float2 hf2 = __half22float2(hv);
          hw[2 * s2 + jj] = h2u(hv);
          lw[2 * s2 + jj] = h2u(__floats2half2_rn(x0 - hf2.x, x1 - hf2.y));
        }
      }
      h = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      l = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    const uint32_t off = sw128_off(kk, 8 * c);
    *reinterpret_cast<uint4 *>(hi + off) = h;
    if (CACHE) *reinterpret_cast<uint4 *>(lo + off) = l;
  }
}

// Write groups g and g + 2 of key row kk (key_store on each).
template <bool CACHE>
__device__ __forceinline__ void key_store2(const KeyRaw2 &r, int kk, int g, uint8_t *hi, uint8_t *lo) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    KeyRaw x;
    x.kind = r.kind;
    x.sz = r.sz[j];
#pragma unroll
    for (int c = 0; c < 4; ++c) x.v[c] = (r.kind == 1) ? r.v[4 * j + c] : r.v[c];
    key_store<CACHE>(x, kk, g + 2 * j, hi, lo);
  }
}

// One (unit, 512-key chunk) work item as both roles of the scorer see it.
struct SelItem {
  int u, T, k0, k1, nsub;  // nsub: sub-tiles of 128 keys (0: none)
  bool valid;              // the unit's length admits a selection (else reported by the top-k)
};

template <int PASS>
__device__ __forceinline__ SelItem sel_item(const SelectArgs &a, int item) {
  SelItem s;
  s.u = item / a.n_chunks;
  s.T = sel_T(a, s.u);
  s.valid = !(s.T < a.n_q || s.T > a.cap || s.T - a.W < a.k);
  const int key_end = (PASS == 1) ? s.T : s.T - a.W;
  s.k0 = (item % a.n_chunks) * SEL_KC;
  s.k1 = min(key_end, s.k0 + SEL_KC);
  s.nsub = (s.valid && s.k0 < key_end) ? (s.k1 - s.k0 + TC_NK - 1) / TC_NK : 0;
  return s;
}

// PASS 1: per-row (max, sum exp) over a chunk of keys; PASS 2: column sums.
// Block b takes a contiguous run of (unit, 512-key chunk) items, so the
// query rows are loaded once per unit.  The warps split into two roles that
// work on different sub-tiles at once and meet only through mbarriers:
//   * warps 0-7 stage key sub-tiles of 128 keys into shared memory (thread s
//     writes key row s % 128, quantization groups s / 128 and s / 128 + 2),
//     loading the next sub-tile from global memory while the current one is
//     written;
//   * warp 16 (one thread) waits until all 256 staging threads have arrived
//     on a sub-tile's barrier and the epilogue is done with the accumulator
//     set, then issues the sub-tile's MMAs and commits them, so no staging
//     warp waits for the tensor cores to accept MMAs;
//   * warps 8-15 read the accumulators the MMAs complete (lane quadrant
//     w % 4, one half of the columns of every row block) and run the exp2
//     epilogue.
// Barriers per buffer: key_full (sub-tile staged, 256 arrivals), acc_full
// (MMAs complete, one commit; it also frees the key buffer they read),
// acc_empty (epilogue done with the accumulators, 256 arrivals).  With up
// to 256 query rows key tiles and accumulators are double-buffered, so the
// staging of sub-tile g + 1 and its MMAs overlap the epilogue of g.  Every
// wait is bounded (2 s, then HYQ_DEV_TIMEOUT); after a timeout every wait
// returns at once and the loops run out without work, so the epilogue
// warps still meet at each of their named barriers.
constexpr int TC_ROLE = TC_THREADS / 2;  // threads per role

template <bool CACHE, int PASS>
__global__ void __launch_bounds__(TC_BLOCK, 1) score_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible (and its tensor memory freed)
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  __shared__ uint32_t tmem_base;
  __shared__ __align__(8) uint64_t key_full[2], acc_full[2], acc_empty[2];
  __shared__ int s_abort;
  // 128-byte swizzled tiles must start on a 1024-byte boundary
  uint8_t *sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
  const int n_rbt = (a.R + 127) / 128;
  const int nbuf = (n_rbt <= 2) ? 2 : 1;
  constexpr int KT = CACHE ? 2 * TC_TILE : TC_TILE;     // one key buffer: hi (+ lo)
  uint8_t *sQ = sm;                                      // [n_rbt][32 KB]
  uint8_t *sK = sQ + n_rbt * TC_TILE;                    // [nbuf][KT]
  float *csum = reinterpret_cast<float *>(sK + nbuf * KT);             // pass 2: [sub-tile parity][half][128]
  float2 *pst = reinterpret_cast<float2 *>(csum + 4 * TC_NK);          // pass 1: [item parity][TC_MAX_RB][128]
  float *moff = reinterpret_cast<float *>(pst + 3 * TC_MAX_RB * 128);  // pass 2: [SEL_MAX_ROWS] m_r - log2(1/l_r)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t acc_cols = static_cast<uint32_t>(n_rbt) * TC_NK;      // one accumulator set
  const uint32_t need = acc_cols * nbuf;
  const uint32_t ncols = (need <= 128) ? 128u : (need <= 256) ? 256u : 512u;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&key_full[b]), TC_ROLE);
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), TC_ROLE);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int *abort = &s_abort;
  const int n_items = a.U * a.n_chunks;
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int it0 = min(n_items, static_cast<int>(blockIdx.x) * per), it1 = min(n_items, it0 + per);
  // bounded wait for phase `parity` of barrier b (false after a timeout, here or elsewhere in the block)
  auto wait = [&](uint64_t *b, uint32_t parity) { return mbar_wait_bounded(smem_u32(b), parity, abort, a.status); };

  if (warp < TC_ROLE / 32) {
    // ---- staging: key row kk of every sub-tile, quantization groups hq and hq + 2
    const int kk = tid & 127, hq = tid >> 7;
    KeyRaw2 rk;         // the next sub-tile to stage (groups hq, hq + 2)
    bool have = false;  // rk already holds it
    int q_unit = -1, q_T = -1, gst = 0;
    for (int item = it0; item < it1; ++item) {
      const SelItem s = sel_item<PASS>(a, item);
      if (s.nsub == 0) continue;
      if (s.u != q_unit || s.T != q_T) {
        // the MMAs that read the previous unit's query rows are complete
        if (gst > 0) wait(&acc_full[(gst - 1) % nbuf], ((gst - 1) / nbuf) & 1);
        // the unit's query rows into the swizzled row blocks (zeros past R)
        const int b = s.u / a.Hkv, kvh = s.u % a.Hkv;
        for (int i = tid; i < n_rbt * 128 * 16; i += TC_ROLE) {
          const int r = i >> 4, c = i & 15;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (r < a.R) {
            const int hg = r / a.n_q, ii = r % a.n_q;
            const int slot = a.q_ring ? ((s.T - a.n_q + ii) % a.n_q + a.n_q) % a.n_q : ii;
            v = *reinterpret_cast<const uint4 *>(a.q + ((static_cast<int64_t>(b) * a.Hq + kvh * a.G + hg) * a.n_q + slot) * D +
                                                 8 * c);
          }
          *reinterpret_cast<uint4 *>(sQ + (r >> 7) * TC_TILE + sw128_off(r & 127, 8 * c)) = v;
        }
        q_unit = s.u;
        q_T = s.T;
      }
      for (int st = 0; st < s.nsub; ++st) {
        const int g = gst + st, buf = g % nbuf;
        const uint32_t ph = (g / nbuf) & 1;
        // the MMAs of sub-tile g - nbuf, the last readers of key buffer buf, are complete
        if (g >= nbuf) wait(&acc_full[buf], ph ^ 1);
        const int key0 = s.k0 + st * TC_NK;
        if (!have) key_load2<CACHE>(a, s.u, s.T, key0 + kk, s.k1, hq, rk);
        uint8_t *kb = sK + buf * KT;
        key_store2<CACHE>(rk, kk, hq, kb, kb + TC_TILE);
        // the next sub-tile (or the next item's first, same unit) loads while this one is issued
        have = false;
        if (st + 1 < s.nsub) {
          key_load2<CACHE>(a, s.u, s.T, key0 + TC_NK + kk, s.k1, hq, rk);
          have = true;
        } else if (item + 1 < it1) {
          const SelItem n = sel_item<PASS>(a, item + 1);
          if (n.nsub > 0 && n.u == s.u && n.T == s.T) {
            key_load2<CACHE>(a, n.u, n.T, n.k0 + kk, n.k1, hq, rk);
            have = true;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> the tensor core
        mbar_arrive(smem_u32(&key_full[buf]));
      }
      gst += s.nsub;
    }
  } else if (warp == TC_THREADS / 32) {
    // ---- MMA issue: sub-tile g once it is staged and accumulator set g % nbuf is free
    if (lane == 0) {
      int gst = 0;
      for (int item = it0; item < it1; ++item) {
        const SelItem s = sel_item<PASS>(a, item);
        if (s.nsub == 0) continue;
        for (int st = 0; st < s.nsub; ++st) {
          const int g = gst + st, buf = g % nbuf;
          const uint32_t ph = (g / nbuf) & 1;
          if (!wait(&key_full[buf], ph) || (g >= nbuf && !wait(&acc_empty[buf], ph ^ 1))) continue;
          uint8_t *kb = sK + buf * KT;
          // every staging thread has written sub-tile g, and the epilogue is done with accumulator set buf
          tc_fence_after();
          // descriptors of k-step 0; k-step ks adds sw128_koff(ks) to the
          // start-address field (16-byte units; tiles lie below 256 KB)
          const uint32_t kh = smem_u32(kb), kl = kh + TC_TILE;
          const uint64_t dkh = sw128_desc(kh, 0), dkl = sw128_desc(kl, 0);
          for (int rb = 0; rb < n_rbt; ++rb) {
            const uint64_t dq = sw128_desc(smem_u32(sQ) + rb * TC_TILE, 0);
            const uint32_t d = tbase + buf * acc_cols + rb * TC_NK;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t o = sw128_koff(ks);
              if (PASS == 1) {  // rows on M, keys on N
                tc_mma(d, dq + o, dkh + o, ks > 0);
                if (CACHE) tc_mma(d, dq + o, dkl + o, 1u);
              } else {          // keys on M, rows on N: each TMEM lane is one key column
                tc_mma(d, dkh + o, dq + o, ks > 0);
                if (CACHE) tc_mma(d, dkl + o, dq + o, 1u);
              }
            }
          }
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           smem_u32(&acc_full[buf]))
                       : "memory");
        }
        gst += s.nsub;
      }
    }
  } else {
    // ---- epilogue: TMEM lane quadrant qd, column half hf of every row block
    const int e = tid - TC_ROLE, ew = e >> 5, qd = ew & 3, hf = ew >> 2;
    int q_unit = -1, q_T = -1, gst = 0, ipar = 0;
    for (int item = it0; item < it1; ++item) {
      const SelItem s = sel_item<PASS>(a, item);
      if (!s.valid) continue;
      const int64_t part = (static_cast<int64_t>(s.u) * a.n_chunks + item % a.n_chunks) * SEL_MAX_ROWS;
      if (s.nsub == 0) {
        if (PASS == 1)
          for (int r = e; r < a.R; r += TC_ROLE) a.stats_part[part + r] = make_float2(-INFINITY, 0.f);
        continue;
      }
      if (PASS == 2 && (s.u != q_unit || s.T != q_T)) {
        // p = exp2(s - m_r) / l_r = exp2(s - (m_r - log2(1 / l_r))); rows
        // without keys (or past R) get +inf, i.e. p = 0
        named_bar_sync(1, TC_ROLE);  // every epilogue thread is done with the previous unit's offsets
        for (int r = e; r < n_rbt * 128; r += TC_ROLE) {
          float mo = INFINITY;
          if (r < a.R) {
            const float2 stt = a.stats[static_cast<int64_t>(s.u) * SEL_MAX_ROWS + r];
            if (stt.y > 0.f) mo = stt.x - __log2f(stt.y);
          }
          moff[r] = mo;
        }
        named_bar_sync(1, TC_ROLE);
      }
      q_unit = s.u;
      q_T = s.T;
      float rm[TC_MAX_RB], rl[TC_MAX_RB];  // pass 1: running (max, sum) of this thread's rows over its columns
#pragma unroll
      for (int rb = 0; rb < TC_MAX_RB; ++rb) {
        rm[rb] = -INFINITY;
        rl[rb] = 0.f;
      }
      for (int st = 0; st < s.nsub; ++st) {
        const int g = gst + st, buf = g % nbuf;
        const uint32_t ph = (g / nbuf) & 1;
        // the warp reads tensor memory together or not at all
        const bool ok = __all_sync(0xffffffffu, wait(&acc_full[buf], ph));
        tc_fence_after();
        const int key0 = s.k0 + st * TC_NK;
        const uint32_t tcol = tbase + (static_cast<uint32_t>(32 * qd) << 16) + buf * acc_cols + 64 * hf;
        if (PASS == 1) {
          const bool all_visible = key0 + TC_NK <= s.k1 && key0 + TC_NK - 1 <= s.T - a.n_q;
#pragma unroll
          for (int rb = 0; rb < TC_MAX_RB; ++rb) {
            if (rb >= n_rbt || !ok) break;
            const int r = 128 * rb + 32 * qd + lane;
            const bool row_ok = r < a.R;
            const int qpos = row_ok ? s.T - a.n_q + r % a.n_q : -1;  // last key this query sees
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              float v[32];
              tc_ld32(tcol + rb * TC_NK + 32 * c2, v);
              const int kb = key0 + 64 * hf + 32 * c2;  // key of v[0]
              if (!(all_visible && row_ok))
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (!(kb + j < s.k1 && kb + j <= qpos)) v[j] = -INFINITY;
              float mx = -INFINITY;
#pragma unroll
              for (int j = 0; j < 32; ++j) mx = fmaxf(mx, v[j]);
              const float mn = fmaxf(rm[rb], mx * SEL_SCALE);  // the scale is positive
              if (mn != -INFINITY) {
                float sum = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) sum += fast_exp2(fmaf(v[j], SEL_SCALE, -mn));
                rl[rb] = rl[rb] * fast_exp2(rm[rb] - mn) + sum;
                rm[rb] = mn;
              }
            }
          }
        } else {
          // this thread is key column 32 qd + lane of the sub-tile; it sums p
          // over its half of the rows (every candidate key is visible to
          // every selection query)
          float acc = 0.f;
#pragma unroll
          for (int rb = 0; rb < TC_MAX_RB; ++rb) {
            if (rb >= n_rbt || !ok) break;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              float v[32];
              tc_ld32(tcol + rb * TC_NK + 32 * c2, v);
              const float *mo = moff + rb * TC_NK + 64 * hf + 32 * c2;  // row of v[0]
#pragma unroll
              for (int j = 0; j < 32; ++j) acc += fast_exp2(fmaf(v[j], SEL_SCALE, -mo[j]));
            }
          }
          csum[((g & 1) * 2 + hf) * TC_NK + 32 * qd + lane] = acc;
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&acc_empty[buf]));  // accumulator set buf may be overwritten
        if (PASS == 2) {
          named_bar_sync(1, TC_ROLE);
          // fixed order: half 0 + half 1, the same for every key
          const int key = key0 + e;
          if (e < TC_NK && key < s.k1)
            a.colsum_part[static_cast<int64_t>(s.u) * a.cap + key] =
                csum[(g & 1) * 2 * TC_NK + e] + csum[((g & 1) * 2 + 1) * TC_NK + e];
        }
      }
      gst += s.nsub;
      if (PASS == 1) {
        // merge the two column halves of every row, then write the chunk partial
        if (hf == 1)
#pragma unroll
          for (int rb = 0; rb < TC_MAX_RB; ++rb)
            if (rb < n_rbt) pst[(ipar * TC_MAX_RB + rb) * 128 + 32 * qd + lane] = make_float2(rm[rb], rl[rb]);
        named_bar_sync(1, TC_ROLE);
        if (hf == 0)
#pragma unroll
          for (int rb = 0; rb < TC_MAX_RB; ++rb) {
            const int r = 128 * rb + 32 * qd + lane;
            if (rb >= n_rbt || r >= a.R) continue;
            const float2 o = pst[(ipar * TC_MAX_RB + rb) * 128 + 32 * qd + lane];
            const float M = fmaxf(rm[rb], o.x);
            float L = 0.f;
            if (M != -INFINITY) L = rl[rb] * fast_exp2(rm[rb] - M) + o.y * fast_exp2(o.x - M);
            a.stats_part[part + r] = make_float2(M, L);
          }
        ipar ^= 1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(ncols));
}

__global__ void __launch_bounds__(1024) rank_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  __shared__ int wsum[32];
  const int u = blockIdx.x;
  const int nw = a.cap / 32;
  int32_t *out = a.rank_base + static_cast<int64_t>(u) * nw;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  // records holding quantized positions [0, T - W); the words after them count 0
  const int T = sel_T(a, u);
  const int nq = (T >= 0 && T <= a.cap) ? (max(T - a.W, 0) + 31) / 32 : 0;
  int carry = 0;
  for (int base = 0; base < nw; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int v = (i < nq) ? __popc(*reinterpret_cast<const uint32_t *>(
                                 a.blocks + rec_mask(a.rm.rec_rd(u, static_cast<int64_t>(i) * 32))))
                           : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    int pre = 0, tot = 0;
    for (int q = 0; q < (int)(blockDim.x >> 5); ++q) {
      if (q < w) pre += wsum[q];
      tot += wsum[q];
    }
    if (i < nw) out[i] = carry + pre + x - v;
    carry += tot;
    __syncthreads();
  }
}

__global__ void stats_merge_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  const int u = blockIdx.x;
  const int T = sel_T(a, u);
  if (T < a.n_q || T > a.cap) return;
  const int nch = (T + SEL_KC - 1) / SEL_KC;
  constexpr int MB = 16;  // chunk partials loaded at once
  for (int r = threadIdx.x; r < a.R; r += blockDim.x) {
    const float2 *p = a.stats_part + static_cast<int64_t>(u) * a.n_chunks * SEL_MAX_ROWS + r;
    // log-sum-exp merge of the chunk partials in chunk order, MB loads in flight
    float M = -INFINITY, L = 0.f;
    for (int c0 = 0; c0 < nch; c0 += MB) {
      float2 v[MB];
#pragma unroll
      for (int j = 0; j < MB; ++j)
        v[j] = (c0 + j < nch) ? p[static_cast<int64_t>(c0 + j) * SEL_MAX_ROWS] : make_float2(-INFINITY, 0.f);
      float bm = M;
#pragma unroll
      for (int j = 0; j < MB; ++j) bm = fmaxf(bm, v[j].x);
      if (bm == -INFINITY) continue;
      L = (M == -INFINITY) ? 0.f : L * fast_exp2(M - bm);
#pragma unroll
      for (int j = 0; j < MB; ++j)
        if (v[j].x != -INFINITY) L += v[j].y * fast_exp2(v[j].x - bm);
      M = bm;
    }
    a.stats[static_cast<int64_t>(u) * SEL_MAX_ROWS + r] = make_float2(M, L > 0.f ? 1.f / L : 0.f);
  }
}

// Exact top-k of colsum[0, n) by (value desc, position asc), ascending output.
// One block of TOPK_THREADS per unit.  The column sums (non-negative floats,
// which order like their bit patterns) are staged in shared memory when they
// fit.  A radix select over the bit patterns, one byte per pass from the
// top, finds the k-th largest value tau and how many of the values equal to
// tau are taken (lowest positions first).  Counts go to one private 256-bin
// histogram per warp (the values crowd into a few bins, so block-wide atomics
// would serialize); after the first byte only the candidates (values whose
// top byte is the selected digit) are visited again.  Each warp then owns a
// contiguous run of positions: it counts, the counts are scanned once, and
// it writes its selected positions in order.
constexpr int TOPK_SMEM_VALS = 32768;  // values staged in shared memory (128 KB; positions fit uint16)
constexpr int TOPK_WARPS = TOPK_THREADS / 32;

__global__ void __launch_bounds__(TOPK_THREADS) topk_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  extern __shared__ uint32_t tk_smem[];  // [TOPK_SMEM_VALS] values, then [TOPK_SMEM_VALS] uint16 candidates
  __shared__ int whist[TOPK_WARPS][256];
  __shared__ int hist[256];
  __shared__ int wcnt[TOPK_WARPS][2];
  __shared__ int s_digit, s_need, s_ncand;
  const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int T = sel_T(a, u);
  const int k = a.k;
  int32_t *out = a.out_pos + static_cast<int64_t>(u) * k;
  if (T < a.n_q || T > a.cap || T - a.W < k) {
    if (tid == 0) set_status(a.status, HYQ_DEV_BADLEN);
    for (int i = tid; i < k; i += blockDim.x) out[i] = -1;
    return;
  }
  const int n = T - a.W;
  float *fin = a.colsum + static_cast<int64_t>(u) * a.cap;
  const bool reduce = a.n_rb > 1 || fin != a.colsum_part + static_cast<int64_t>(u) * a.cap;
  const bool staged = n <= TOPK_SMEM_VALS;
  // the column sums, 8 loads in flight per thread
  constexpr int LB = 8;
  for (int i0 = tid; i0 < n; i0 += LB * static_cast<int>(blockDim.x)) {
    float v[LB];
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int i = i0 + b * static_cast<int>(blockDim.x);
      v[b] = 0.f;
      if (i < n) {
        if (reduce) {
          for (int z = 0; z < a.n_rb; ++z) v[b] += __ldcg(a.colsum_part + (static_cast<int64_t>(z) * a.U + u) * a.cap + i);
        } else {
          v[b] = __ldcg(fin + i);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int i = i0 + b * static_cast<int>(blockDim.x);
      if (i < n) {
        if (reduce) fin[i] = v[b];
        if (staged) tk_smem[i] = __float_as_uint(v[b]);
      }
    }
  }
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  if (k == 0) return;
  const uint32_t *vals = staged ? tk_smem : reinterpret_cast<const uint32_t *>(fin);
  uint16_t *cand = reinterpret_cast<uint16_t *>(tk_smem + TOPK_SMEM_VALS);  // candidate positions (< 2^15)
  const bool use_cand = staged;

  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = lane; i < 256; i += 32) whist[w][i] = 0;
    __syncwarp();
    const int ncand = s_ncand;
    const bool from_cand = pass > 0 && use_cand;
    const int m = from_cand ? ncand : n;
    for (int base = 0; base < m; base += blockDim.x) {  // whole warps iterate together
      const int j = base + tid;
      uint32_t b = 0;
      bool act = false;
      if (j < m) {
        b = vals[from_cand ? cand[j] : j];
        act = (b & mask) == prefix;
      }
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t bin = (b >> shift) & 255u;
        const unsigned peers = __match_any_sync(am, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&whist[w][bin], __popc(peers));  // private to the warp: no contention
      }
    }
    __syncthreads();
    if (tid < 256) {
      int c = 0;
#pragma unroll 8
      for (int q = 0; q < TOPK_WARPS; ++q) c += whist[q][tid];
      hist[tid] = c;
    }
    __syncthreads();
    if (w == 0) {
      // suffix counts over bins 255 .. 0: lane l holds bins 255 - 8l .. 248 - 8l
      int h[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[e] = hist[255 - 8 * lane - e];
        sum += h[e];
      }
      int x = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      int run = x - sum;  // count of bins above this lane's first bin
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (run < need && run + h[e] >= need) {
          s_digit = 255 - 8 * lane - e;
          s_need = need - run;
        }
        run += h[e];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(s_digit) << shift;
    mask |= 255u << shift;
    need = s_need;
    if (pass == 0 && use_cand) {
      // candidates for the lower bytes: values whose top byte is the digit
      for (int base = 0; base < n; base += blockDim.x) {
        const int j = base + tid;
        const bool c = j < n && (vals[j] & mask) == prefix;
        const unsigned bal = __ballot_sync(0xffffffffu, c);
        int slot0 = 0;
        if (lane == 0 && bal) slot0 = atomicAdd(&s_ncand, __popc(bal));
        slot0 = __shfl_sync(0xffffffffu, slot0, 0);
        if (c) cand[slot0 + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
      }
    }
    __syncthreads();  // s_digit, s_need, s_ncand, whist and hist are reused
  }
  // tau = prefix: take every value > tau and the first `need` values == tau.
  // Warp w owns positions [w * per, (w + 1) * per).
  const uint32_t tau = prefix;
  const int per = ((n + TOPK_WARPS - 1) / TOPK_WARPS + 31) / 32 * 32;
  const int beg = min(n, w * per), end = min(n, beg + per);
  int n_gt = 0, n_eq = 0;
  for (int j = beg + lane; j < beg + per; j += 32) {  // per is a multiple of 32: whole warps iterate
    const bool in = j < end;
    const uint32_t b = in ? vals[j] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, in && b > tau));
    n_eq += __popc(__ballot_sync(0xffffffffu, in && b == tau));
  }
  if (lane == 0) {
    wcnt[w][0] = n_gt;
    wcnt[w][1] = n_eq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;
  for (int q = 0; q < w; ++q) {
    gt_before += wcnt[q][0];
    eq_before += wcnt[q][1];
  }
  const int take_eq_before = min(eq_before, need);  // equal values taken by the warps before this one
  int o = gt_before + take_eq_before, eq_seen = eq_before;
  for (int j = beg + lane; j < beg + per; j += 32) {
    const bool in = j < end;
    const uint32_t b = in ? vals[j] : 0u;
    const bool gt = in && b > tau, eq = in && b == tau;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqb & ((1u << lane) - 1u)) < need);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = o + __popc(tb & ((1u << lane) - 1u));
    if (take && pos < k) out[pos] = j;
    o += __popc(tb);
    eq_seen += __popc(eqb);
  }
}

// The same selection with the column sums of one unit spread over the TKC
// blocks of a thread-block cluster (used while every block's share fits in
// its shared memory; topk_kernel above serves longer contexts).  Block r
// stages positions [r S, r S + S), S = n / TKC rounded up to a multiple of
// 32.  In each radix pass a block counts its own values (or, after the first
// byte, its own candidates) into a 256-bin histogram; after a cluster
// barrier every block adds the TKC histograms through distributed shared
// memory and picks the same digit.  At the end each block counts its values
// above tau and equal to it, reads the counts of the blocks before it, and
// writes its selected positions at their place in the ascending output; the
// positions equal to tau are taken lowest first across the whole unit.
constexpr int TKC = 8;                // blocks per unit: one cluster (the portable maximum size)
constexpr int TKC_THREADS = 512;
constexpr int TKC_WARPS = TKC_THREADS / 32;
constexpr int TKC_MAX_VALS = 32768;   // values per block (block-local positions fit uint16)

__device__ __forceinline__ int cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return static_cast<int>(r);
}
__device__ __forceinline__ int cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return static_cast<int>(r);
}
// Every thread of every block of the cluster arrives; shared-memory writes
// before it are visible to the cluster's reads after it.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Read an int at the same shared-memory offset in block `rank` of the cluster.
__device__ __forceinline__ int ld_cluster_s32(const int *p, int rank) {
  uint32_t remote;
  int v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

__global__ void __launch_bounds__(TKC_THREADS) topk_cluster_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  extern __shared__ uint32_t tkc_smem[];  // [S] values, then [S] uint16 block-local candidate positions
  __shared__ int whist[TKC_WARPS][256];
  __shared__ int bhist[2][256];  // this block's histogram of the even / odd passes (read by the cluster)
  __shared__ int ghist[256];     // the cluster's histogram of the pass
  __shared__ int bcnt[2];        // this block's values above tau and equal to it (read by later blocks)
  __shared__ int wcnt[TKC_WARPS][2];
  __shared__ int s_digit, s_need, s_ncand, s_gt_before, s_eq_before;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int r = cluster_rank(), u = cluster_index();
  const int T = sel_T(a, u);
  const int k = a.k;
  int32_t *out = a.out_pos + static_cast<int64_t>(u) * k;
  if (T < a.n_q || T > a.cap || T - a.W < k) {  // the same decision in every block of the cluster
    if (r == 0) {
      if (tid == 0) set_status(a.status, HYQ_DEV_BADLEN);
      for (int i = tid; i < k; i += TKC_THREADS) out[i] = -1;
    }
    return;
  }
  const int n = T - a.W;
  const int S = ((n + TKC - 1) / TKC + 31) / 32 * 32;
  const int beg = min(n, r * S), m = min(n, beg + S) - beg;  // this block's positions [beg, beg + m)
  float *fin = a.colsum + static_cast<int64_t>(u) * a.cap;
  const bool reduce = a.n_rb > 1 || fin != a.colsum_part + static_cast<int64_t>(u) * a.cap;
  uint32_t *vals = tkc_smem;
  uint16_t *cand = reinterpret_cast<uint16_t *>(tkc_smem + S);
  constexpr int LB = 8;  // loads in flight per thread
  for (int i0 = tid; i0 < m; i0 += LB * TKC_THREADS) {
    float v[LB];
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int i = i0 + b * TKC_THREADS;
      v[b] = 0.f;
      if (i < m) {
        if (reduce) {
          for (int z = 0; z < a.n_rb; ++z)
            v[b] += __ldcg(a.colsum_part + (static_cast<int64_t>(z) * a.U + u) * a.cap + beg + i);
        } else {
          v[b] = __ldcg(fin + beg + i);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int i = i0 + b * TKC_THREADS;
      if (i < m) {
        if (reduce) fin[beg + i] = v[b];
        vals[i] = __float_as_uint(v[b]);
      }
    }
  }
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  if (k == 0) return;  // k is the same for every block: no block waits at a cluster barrier

  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = lane; i < 256; i += 32) whist[w][i] = 0;
    __syncwarp();
    const int mc = pass > 0 ? s_ncand : m;
    for (int base = 0; base < mc; base += TKC_THREADS) {  // whole warps iterate together
      const int j = base + tid;
      uint32_t b = 0;
      bool act = false;
      if (j < mc) {
        b = vals[pass > 0 ? cand[j] : j];
        act = (b & mask) == prefix;
      }
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t bin = (b >> shift) & 255u;
        const unsigned peers = __match_any_sync(am, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&whist[w][bin], __popc(peers));
      }
    }
    __syncthreads();
    if (tid < 256) {
      int c = 0;
#pragma unroll
      for (int q = 0; q < TKC_WARPS; ++q) c += whist[q][tid];
      bhist[pass & 1][tid] = c;
    }
    // Every block's histogram of this pass is complete.  (A block rewrites
    // bhist[pass & 1] two passes later, after the next barrier, which no
    // block reaches before it has read this pass's histograms.)
    cluster_barrier();
    if (tid < 256) {
      int c = 0;
#pragma unroll
      for (int q = 0; q < TKC; ++q) c += ld_cluster_s32(&bhist[pass & 1][tid], q);
      ghist[tid] = c;
    }
    __syncthreads();
    if (w == 0) {
      // suffix counts over bins 255 .. 0: lane l holds bins 255 - 8l .. 248 - 8l
      int h[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[e] = ghist[255 - 8 * lane - e];
        sum += h[e];
      }
      int x = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      int run = x - sum;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (run < need && run + h[e] >= need) {
          s_digit = 255 - 8 * lane - e;
          s_need = need - run;
        }
        run += h[e];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(s_digit) << shift;
    mask |= 255u << shift;
    need = s_need;
    if (pass == 0) {
      // this block's candidates for the lower bytes
      for (int base = 0; base < m; base += TKC_THREADS) {
        const int j = base + tid;
        const bool c = j < m && (vals[j] & mask) == prefix;
        const unsigned bal = __ballot_sync(0xffffffffu, c);
        int slot0 = 0;
        if (lane == 0 && bal) slot0 = atomicAdd(&s_ncand, __popc(bal));
        slot0 = __shfl_sync(0xffffffffu, slot0, 0);
        if (c) cand[slot0 + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
      }
    }
    __syncthreads();  // s_digit, s_need, s_ncand, whist and ghist are reused
  }
  // tau = prefix: take every value > tau and the first `need` values == tau
  // of the unit.  Warp w of this block owns block-local positions
  // [w * per, (w + 1) * per).
  const uint32_t tau = prefix;
  const int per = ((m + TKC_WARPS - 1) / TKC_WARPS + 31) / 32 * 32;
  const int wb = min(m, w * per), we = min(m, wb + per);
  int n_gt = 0, n_eq = 0;
  for (int j = wb + lane; j < wb + per; j += 32) {  // per is a multiple of 32: whole warps iterate
    const bool in = j < we;
    const uint32_t b = in ? vals[j] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, in && b > tau));
    n_eq += __popc(__ballot_sync(0xffffffffu, in && b == tau));
  }
  if (lane == 0) {
    wcnt[w][0] = n_gt;
    wcnt[w][1] = n_eq;
  }
  __syncthreads();
  if (tid == 0) {
    int g = 0, e = 0;
    for (int q = 0; q < TKC_WARPS; ++q) {
      g += wcnt[q][0];
      e += wcnt[q][1];
    }
    bcnt[0] = g;
    bcnt[1] = e;
  }
  cluster_barrier();  // every block's counts are complete
  if (tid == 0) {
    int g = 0, e = 0;
    for (int q = 0; q < r; ++q) {
      g += ld_cluster_s32(&bcnt[0], q);
      e += ld_cluster_s32(&bcnt[1], q);
    }
    s_gt_before = g;
    s_eq_before = e;
  }
  __syncthreads();
  int gt_before = s_gt_before, eq_before = s_eq_before;
  for (int q = 0; q < w; ++q) {
    gt_before += wcnt[q][0];
    eq_before += wcnt[q][1];
  }
  const int take_eq_before = min(eq_before, need);  // equal values taken before this warp's positions
  int o = gt_before + take_eq_before, eq_seen = eq_before;
  for (int j = wb + lane; j < wb + per; j += 32) {
    const bool in = j < we;
    const uint32_t b = in ? vals[j] : 0u;
    const bool gt = in && b > tau, eq = in && b == tau;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqb & ((1u << lane) - 1u)) < need);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = o + __popc(tb & ((1u << lane) - 1u));
    if (take && pos < k) out[pos] = beg + j;
    o += __popc(tb);
    eq_seen += __popc(eqb);
  }
  cluster_barrier();  // no block leaves while another may still read its shared memory
}

// Values per block of the cluster top-k for a cache, or 0 when topk_kernel
// (one block per unit) is used instead: when a block's share would not fit
// its shared memory, or when the clusters would fill more than two waves of
// the SMs (many units: one block per unit already spreads over the GPU, and
// measured faster at 128 units).
static int topk_cluster_vals(const SelectArgs &a, int sms) {
  const int n_max = a.cap - a.W;
  const int S = ((n_max + TKC - 1) / TKC + 31) / 32 * 32;
  if (S > TKC_MAX_VALS || static_cast<int64_t>(a.U) * TKC > 2 * static_cast<int64_t>(sms)) return 0;
  return std::max(S, 32);
}

static cudaError_t launch_topk_cluster(const SelectArgs &a, int S, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.U * TKC));
  cfg.blockDim = dim3(TKC_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(S) * (sizeof(uint32_t) + sizeof(uint16_t));
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = TKC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, a);
}

static size_t score_smem_bytes(int R, bool cache) {
  const int n_rbt = (R + 127) / 128;
  const int nbuf = (n_rbt <= 2) ? 2 : 1;
  return 1024 /* alignment */ + static_cast<size_t>(n_rbt) * TC_TILE + static_cast<size_t>(nbuf) * (cache ? 2 : 1) * TC_TILE +
         SEL_KC * 4 + 4 * TC_NK * 4 + 3 * TC_MAX_RB * 128 * 8 + SEL_MAX_ROWS * 4;
}

static cudaError_t select_launch(const SelectArgs &a, bool cache, cudaStream_t s) {
  const size_t smem = score_smem_bytes(a.R, cache);
  static int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    const int mx = static_cast<int>(std::max(score_smem_bytes(SEL_MAX_ROWS, true), score_smem_bytes(256, true)));
    cudaFuncSetAttribute(score_kernel<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    cudaFuncSetAttribute(score_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    cudaFuncSetAttribute(score_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    cudaFuncSetAttribute(score_kernel<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(TOPK_SMEM_VALS * (sizeof(uint32_t) + sizeof(uint16_t))));
    cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(TKC_MAX_VALS * (sizeof(uint32_t) + sizeof(uint16_t))));
    attr_dev = dev;
  }
  const int n_items = a.U * a.n_chunks;
  const int sms = hyq_sm_count_dev();
  const dim3 grid(n_items < sms ? n_items : sms);
  cudaError_t e;
  if (cache) {
    e = launch(rank_kernel, dim3(a.U), dim3(1024), 0, s, a);
    if (e == cudaSuccess) e = launch(score_kernel<true, 1>, grid, dim3(TC_BLOCK), smem, s, a);
  } else {
    e = launch(score_kernel<false, 1>, grid, dim3(TC_BLOCK), smem, s, a);
  }
  if (e == cudaSuccess) e = launch(stats_merge_kernel, dim3(a.U), dim3(256), 0, s, a);
  if (e == cudaSuccess) e = launch(cache ? score_kernel<true, 2> : score_kernel<false, 2>, grid, dim3(TC_BLOCK), smem, s, a);
  const int tkc_vals = topk_cluster_vals(a, sms);
  if (e == cudaSuccess)
    e = tkc_vals > 0 ? launch_topk_cluster(a, tkc_vals, s)
                     : launch(topk_kernel, dim3(a.U), dim3(TOPK_THREADS),
                              TOPK_SMEM_VALS * (sizeof(uint32_t) + sizeof(uint16_t)), s, a);
  return e;
}

}  // namespace hyq

using namespace hyq;

extern "C" hyq_status hyq_check_cache(const hyq_cache *c);

static inline bool al16s(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t a256(size_t x) { return (x + 255) / 256 * 256; }

extern "C" size_t hyq_select_vl_workspace(const hyq_cache *c, int32_t n_q) {
  if (!c || c->n_kv_heads <= 0 || c->capacity <= 0 || n_q <= 0) return 0;
  const size_t U = static_cast<size_t>(c->batch) * c->n_kv_heads;
  const size_t nch = (static_cast<size_t>(c->capacity) + SEL_KC - 1) / SEL_KC;
  const size_t n_rb = (static_cast<size_t>(n_q) * (c->n_q_heads / c->n_kv_heads) + SEL_BLOCK_ROWS - 1) / SEL_BLOCK_ROWS;
  return a256(U * nch * SEL_MAX_ROWS * 8) + a256(U * SEL_MAX_ROWS * 8) + a256(U * c->capacity * 4) * (n_rb + 1) +
         a256(U * (c->capacity / 32) * 4);
}

extern "C" hyq_status hyq_select_vl(const hyq_cache *c, const void *q_sel, int32_t n_q,
                                    int32_t q_is_ring, const void *k_full, int32_t k,
                                    int32_t *out_pos, float *out_colsum, void *ws, size_t ws_bytes,
                                    void *stream) {
  HYQ_RANGE("hyq_select_vl");
  hyq_status st = hyq_check_cache(c);
  if (st != HYQ_OK) return st;
  if (!q_sel || (k > 0 && !out_pos)) return HYQ_ERR_INVALID;
  if (n_q < 1 || n_q > 64 || n_q > c->window) return HYQ_ERR_INVALID;
  if (k < 0 || k > c->vl_capacity || k > c->capacity - c->window) return HYQ_ERR_INVALID;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (n_q * G > SEL_MAX_ROWS) return HYQ_ERR_UNSUPPORTED;
  if (!al16s(q_sel) || (k_full && !al16s(k_full)) || (out_pos && !al16s(out_pos)) ||
      (out_colsum && !al16s(out_colsum)) || !al16s(ws))
    return HYQ_ERR_ALIGN;
  if (!ws || ws_bytes < hyq_select_vl_workspace(c, n_q)) return HYQ_ERR_WORKSPACE;
  if (k == 0 && !out_colsum) return HYQ_OK;
  SelectArgs a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.G = G; a.n_q = n_q;
  a.q_ring = q_is_ring ? 1 : 0; a.cap = c->capacity; a.W = c->window; a.vl_cap = c->vl_capacity;
  a.U = c->batch * c->n_kv_heads; a.R = n_q * G; a.k = k;
  a.n_chunks = (c->capacity + SEL_KC - 1) / SEL_KC;
  a.q = static_cast<const __half *>(q_sel);
  a.k_full = static_cast<const __half *>(k_full);
  a.blocks = c->blocks;
  a.rm = RecMap{c->block_table, c->n_kv_heads, c->capacity, c->n_pages, c->dev_status};
  a.win_k = static_cast<const __half *>(c->win_k); a.vl_k = static_cast<const __half *>(c->vl_k);
  a.vl_pos = c->vl_pos; a.vl_count = c->vl_count; a.seq_len = c->seq_len;
  uint8_t *w = static_cast<uint8_t *>(ws);
  const size_t U = a.U;
  a.stats_part = reinterpret_cast<float2 *>(w);
  w += a256(U * a.n_chunks * SEL_MAX_ROWS * 8);
  a.stats = reinterpret_cast<float2 *>(w);
  w += a256(U * SEL_MAX_ROWS * 8);
  a.n_rb = (a.R + SEL_BLOCK_ROWS - 1) / SEL_BLOCK_ROWS;
  a.colsum_part = reinterpret_cast<float *>(w);
  w += a256(U * c->capacity * 4) * a.n_rb;
  a.colsum = out_colsum ? out_colsum : (a.n_rb == 1 ? a.colsum_part : reinterpret_cast<float *>(w));
  w += a256(U * c->capacity * 4);
  a.rank_base = reinterpret_cast<int32_t *>(w);
  a.out_pos = out_pos;
  a.status = c->dev_status;
  return select_launch(a, k_full == nullptr, static_cast<cudaStream_t>(stream)) == cudaSuccess ? HYQ_OK
                                                                                                : HYQ_ERR_CUDA;
}

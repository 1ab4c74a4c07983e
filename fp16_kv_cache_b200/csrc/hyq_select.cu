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
//   1. row_stats  grid (key chunks, units): S = Q K^T on the tensor cores
//      (mma.sync m16n8k16, query rows on M, keys on N, fp32 accumulate);
//      per row the running max / sum of exp over the chunk's keys.
//   2. stats_merge grid (units): log-sum-exp merge of the chunk partials in
//      a fixed order -> (m_r, 1 / l_r).
//   3. colsum     grid (key chunks, units): S again for candidate keys,
//      P = exp2(S - m_r) / l_r, column sums over the rows with a fixed
//      reduction order (no float atomics), so equal key columns give
//      bitwise-equal sums.
//   4. topk       grid (units): exact radix select on the fp32 bit patterns
//      (non-negative floats order like their bits), ties to lower positions,
//      output compacted in ascending position order.
// Keys come from k_full (prefill) or from the cache as decode sees it: FP16
// window and vertical-line rows, and INT4 rows dequantized as
// zero + code * scale in fp32 and split into two fp16 terms hi + lo (both
// multiplied on the tensor cores) so the dequantized key keeps ~22 bits.
#include "hyq_common.cuh"

extern "C" int32_t hyq_sm_count(void);  // hyq_api.cu

namespace hyq {

static int hyq_sm_count_dev() { return hyq_sm_count(); }

constexpr int SEL_SUB = 64;       // keys per shared-memory sub-tile
constexpr int SEL_KC = 512;       // keys per work item (chunk)
constexpr int SEL_MAX_ROWS = 512; // n_q * G
constexpr int SEL_BLOCK_ROWS = 256;  // query rows per block (8 warps x 32)
constexpr int TOPK_THREADS = 1024;
constexpr float SEL_SCALE = 0.12751743082459868f;  // log2(e) / sqrt(128)

struct SelectArgs {
  int B, Hq, Hkv, G, n_q, q_ring, cap, W, vl_cap, U, R, k, n_chunks;
  const __half *q;       // [B][Hq][n_q][128]
  const __half *k_full;  // nullable [B][Hkv][cap][128]
  const uint8_t *blocks;  // quantized majority + bitmask, [U][cap/32][BLK_BYTES]
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

// ldmatrix x4: four 8x8 b16 matrices, row addresses from lanes 0-7, 8-15, ...
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Swizzled offset of 16-byte chunk c (0..15) of key row p in a [64][128] fp16
// tile: chunk index XOR (p & 7) keeps ldmatrix row reads conflict free.
__device__ __forceinline__ uint32_t tile_off(int p, int c) {
  return static_cast<uint32_t>(p * 256 + ((c ^ (p & 7)) << 4));
}

__device__ __forceinline__ int sel_T(const SelectArgs &a, int u) { return a.seq_len[u / a.Hkv]; }

// One block = 256 threads; a 64-key sub-tile is 1024 items (key, 16-byte
// chunk), 4 per thread: item i = threadIdx.x + 256 j -> key i / 16, chunk i % 16.
constexpr int SEL_THREADS = 256;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Prefill mode: FP16 keys straight into the swizzled tile (zero past key_end).
__device__ __forceinline__ void issue_fp16(const SelectArgs &a, int u, int key0, int key_end, uint32_t hi) {
  const __half *base = a.k_full + static_cast<int64_t>(u) * a.cap * D;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = threadIdx.x + SEL_THREADS * j;
    const int p = i >> 4, c = i & 15;
    const int key = key0 + p;
    const bool in = key < key_end;
    cp_async16(hi + tile_off(p, c), base + static_cast<int64_t>(in ? key : 0) * D + 8 * c, in ? 16 : 0);
  }
  cp_async_commit();
}

// Cache mode: raw bytes of 4 items in registers (loaded before the current
// sub-tile is computed, converted after).
struct RawItems {
  uint4 v[4];
  uint32_t sz[4];
  int kind[4];  // -1 FP16 row (window / vertical line), -2 INT4, -3 zero
};

__device__ __forceinline__ void issue_cache(const SelectArgs &a, int u, int T, int key0, int key_end,
                                            const int *slot_of, int k0, RawItems &r) {
  const int L4 = T - a.W;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = threadIdx.x + SEL_THREADS * j;
    const int p = i >> 4, c = i & 15;
    const int key = key0 + p;
    r.v[j] = make_uint4(0, 0, 0, 0);
    r.sz[j] = 0;
    r.kind[j] = -3;
    if (key >= key_end) continue;
    if (key >= L4) {
      r.kind[j] = -1;
      r.v[j] = *reinterpret_cast<const uint4 *>(a.win_k + (static_cast<int64_t>(u) * a.W + key % a.W) * D + 8 * c);
      continue;
    }
    const int slot = slot_of[key - k0];
    if (slot >= 0) {
      r.kind[j] = -1;
      r.v[j] = *reinterpret_cast<const uint4 *>(a.vl_k + (static_cast<int64_t>(u) * a.vl_cap + slot) * D + 8 * c);
      continue;
    }
    // channels 8c..8c+7: group c / 4, pieces 2(c%4) and 2(c%4)+1
    r.kind[j] = -2;
    r.v[j] = *reinterpret_cast<const uint4 *>(a.blocks + kcode_off(u, key, a.cap) + 16 * (c & 3));
    r.sz[j] = *reinterpret_cast<const uint32_t *>(a.blocks + ksz_off(u, key, a.cap) + 4 * (c >> 2));
  }
}

// Convert the raw items into the sub-tile: every key row holds 128 fp16
// values, the INT4 codes as exact small integers (an INT4 key is zero_g +
// scale_g * code, applied after the MMA) and FP16 keys as they are.  The
// per-key tables (in the sub-tile's second 16 KB) hold scale_g as fp32
// [4][64] at byte 0 and zero_g as fp16 [64][4] at byte 1024; FP16 and
// padding keys get scale 1, zero 0.
constexpr int TAB_ZERO = 1024;
__device__ __forceinline__ void store_cache(const RawItems &r, uint8_t *hi, uint8_t *tab) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = threadIdx.x + SEL_THREADS * j;
    const int p = i >> 4, c = i & 15;
    const int g = c >> 2;
    uint4 h = r.v[j];
    __half2 sz = __floats2half2_rn(1.f, 0.f);
    if (r.kind[j] == -2) {
      const int hh = g >> 1, ii = g & 1;
      const uint32_t w0 = hh ? r.v[j].y : r.v[j].x;  // piece 2(c%4), word hh
      const uint32_t w1 = hh ? r.v[j].w : r.v[j].z;  // piece 2(c%4)+1
      uint32_t hw[4];
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const uint32_t w = s2 ? w1 : w0;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const uint32_t byte = (w >> (8 * (2 * jj + ii))) & 0xFFu;  // channels 2jj (lo), 2jj+1 (hi)
          hw[2 * s2 + jj] = h2u(__floats2half2_rn(static_cast<float>(byte & 15u), static_cast<float>(byte >> 4)));
        }
      }
      h = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      sz = u2h(r.sz[j]);
    } else if (r.kind[j] == -3) {
      h = make_uint4(0, 0, 0, 0);
    }
    *reinterpret_cast<uint4 *>(hi + tile_off(p, c)) = h;
    if ((c & 3) == 0) {
      reinterpret_cast<float *>(tab)[g * SEL_SUB + p] = __low2float(sz);
      reinterpret_cast<__half *>(tab + TAB_ZERO)[p * 4 + g] = __high2half(sz);
    }
  }
}

// Q fragments of the warp's 32 rows (2 m-tiles x 8 k-steps x 4 regs).
__device__ __forceinline__ void load_qa(const SelectArgs &a, int u, int T, int warp, int lane,
                                        uint32_t (&qa)[2][8][4], uint32_t (&qz)[2][4]) {
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  const int gid = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = 32 * warp + 16 * mt + gid + 8 * hr;
      const __half *qr = nullptr;
      if (row < a.R) {
        const int hg = row / a.n_q, i = row % a.n_q;
        int slot = i;
        if (a.q_ring) slot = ((T - a.n_q + i) % a.n_q + a.n_q) % a.n_q;
        qr = a.q + ((static_cast<int64_t>(b) * a.Hq + kvh * a.G + hg) * a.n_q + slot) * D;
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t v0 = 0, v1 = 0;
        if (qr) {
          v0 = *reinterpret_cast<const uint32_t *>(qr + 16 * ks + 2 * t4);
          v1 = *reinterpret_cast<const uint32_t *>(qr + 16 * ks + 8 + 2 * t4);
        }
        qa[mt][ks][hr] = v0;      // a0 / a1: cols 2t, 2t+1
        qa[mt][ks][2 + hr] = v1;  // a2 / a3: cols 2t+8, 2t+9
      }
    }
  // Zero-term A fragments: row r's per-group sums of q split hi + lo in
  // fp16, at k = 0,1 (hi of groups 0,1), 2,3 (lo), 8,9 (hi of 2,3), 10,11
  // (lo); lanes t = 0 and 1 carry them, lanes 2 and 3 zeros.
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float gs[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float2 f0 = __half22float2(u2h(qa[mt][2 * g + e][hr]));
          const float2 f1 = __half22float2(u2h(qa[mt][2 * g + e][2 + hr]));
          s += (f0.x + f0.y) + (f1.x + f1.y);
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        gs[g] = s;
      }
      __half hi[4], lo[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        hi[g] = __float2half_rn(gs[g]);
        lo[g] = __float2half_rn(gs[g] - __half2float(hi[g]));
      }
      qz[mt][hr] = (t4 == 0) ? h2u(__halves2half2(hi[0], hi[1])) : (t4 == 1) ? h2u(__halves2half2(lo[0], lo[1])) : 0u;
      qz[mt][2 + hr] = (t4 == 0) ? h2u(__halves2half2(hi[2], hi[3])) : (t4 == 1) ? h2u(__halves2half2(lo[2], lo[3])) : 0u;
    }
}

// S (log2 domain) for the warp's 32 rows x 64 keys of the sub-tile.
// Prefill mode: the tile holds FP16 keys, S = Q K^T.  Cache mode: per group
// g of 32 channels, S += scale_g * (Q_g . tile_g) with the scale applied in
// fp32 per key, plus sum_g zero_g * qsum_g as one more MMA per 16 rows.
template <bool CACHE>
__device__ __forceinline__ void tile_scores(uint32_t hi, uint32_t tab, const uint32_t (&qa)[2][8][4],
                                            const uint32_t (&qz)[2][4], int lane, float (&s)[2][8][4]) {
  // ldmatrix x4 row addresses: lanes 8j..8j+7 address key rows (nt*8 + lane%8)
  // at chunk (2*kp + j) for matrices j = 0..3 (two k-steps per load)
  const int kr = lane & 7, jm = lane >> 3;
  const int gid = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[mt][nt][e] = 0.f;
    if (CACHE) {
      const uint2 z = lds64(tab + TAB_ZERO + (nt * 8 + gid) * 8);  // zeros of key nt*8 + gid
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) mma16816(s[mt][nt], qz[mt][0], qz[mt][1], qz[mt][2], qz[mt][3], z.x, z.y);
    }
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {  // kp = group g: channels 32g .. 32g + 31
      const int p = nt * 8 + kr, c = 4 * kp + jm;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(hi + tile_off(p, c), b0, b1, b2, b3);
      if (CACHE) {
        float sg[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          mma16816(sg[mt], qa[mt][2 * kp][0], qa[mt][2 * kp][1], qa[mt][2 * kp][2], qa[mt][2 * kp][3], b0, b1);
          mma16816(sg[mt], qa[mt][2 * kp + 1][0], qa[mt][2 * kp + 1][1], qa[mt][2 * kp + 1][2],
                   qa[mt][2 * kp + 1][3], b2, b3);
        }
        // scales of the lane's two key columns nt*8 + 2t, nt*8 + 2t + 1
        float2 sc;
        asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(sc.x), "=f"(sc.y)
                     : "r"(tab + (kp * SEL_SUB + nt * 8 + 2 * t4) * 4));
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          s[mt][nt][0] += sc.x * sg[mt][0];
          s[mt][nt][1] += sc.y * sg[mt][1];
          s[mt][nt][2] += sc.x * sg[mt][2];
          s[mt][nt][3] += sc.y * sg[mt][3];
        }
      } else {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          mma16816(s[mt][nt], qa[mt][2 * kp][0], qa[mt][2 * kp][1], qa[mt][2 * kp][2], qa[mt][2 * kp][3], b0, b1);
          mma16816(s[mt][nt], qa[mt][2 * kp + 1][0], qa[mt][2 * kp + 1][1], qa[mt][2 * kp + 1][2],
                   qa[mt][2 * kp + 1][3], b2, b3);
        }
      }
    }
  }
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[mt][nt][e] *= SEL_SCALE;
}

// PASS 1: per-row (max, sum exp) over a chunk of keys; PASS 2: column sums.
// Persistent: block b takes work items b, b + gridDim.x, ... of the
// (unit, chunk) space; blockIdx.y is the row block (rows 256 y .. 256 y + 255).
// Shared memory: 2 x (hi, lo) 64-key tiles, slot_of[SEL_KC], cpart[8][64].
template <bool CACHE, int PASS>
__global__ void __launch_bounds__(SEL_THREADS, 1) score_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  extern __shared__ __align__(128) uint8_t sm[];
  constexpr int TILE = SEL_SUB * 256;
  uint8_t *tiles = sm;  // buf b: keys at 2b*TILE, cache-mode scale/zero tables at (2b+1)*TILE
  int *slot_of = reinterpret_cast<int *>(sm + 4 * TILE);
  float *cpart = reinterpret_cast<float *>(sm + 4 * TILE + SEL_KC * 4);
  const int rb = blockIdx.y;
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warp = wl + rb * (SEL_BLOCK_ROWS / 32);  // global warp: rows 32 warp ..
  const bool has_rows = 32 * warp < a.R;
  const int gid = lane >> 2, t4 = lane & 3;
  const int n_items = a.U * a.n_chunks;
  const uint32_t tiles_s = smem_u32(tiles);
  uint32_t qa[2][8][4], qz[2][4];
  int q_unit = -1, q_T = -1;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int u = item / a.n_chunks, chunk = item % a.n_chunks;
    const int T = sel_T(a, u);
    if (T < a.n_q || T > a.cap || T - a.W < a.k) continue;  // reported by the top-k kernel
    const int key_end = (PASS == 1) ? T : T - a.W;
    const int k0 = chunk * SEL_KC;
    if (k0 >= key_end) {
      if (PASS == 1)
        for (int r = threadIdx.x; r < SEL_BLOCK_ROWS; r += blockDim.x)
          a.stats_part[(static_cast<int64_t>(u) * a.n_chunks + chunk) * SEL_MAX_ROWS + rb * SEL_BLOCK_ROWS + r] =
              make_float2(-INFINITY, 0.f);
      continue;
    }
    const int k1 = min(key_end, k0 + SEL_KC);
    const int nsub = (k1 - k0 + SEL_SUB - 1) / SEL_SUB;
    __syncthreads();  // previous item fully done with shared memory
    RawItems raw;
    if (CACHE) {
      // vertical-line slot of every key of the chunk: rank of its mask bit
      const int32_t *rbase = a.rank_base + static_cast<int64_t>(u) * (a.cap / 32);
      for (int j = threadIdx.x; j < SEL_KC; j += blockDim.x) {
        const int key = k0 + j;
        int slot = -1;
        if (key < k1 && key < T - a.W) {
          const uint32_t w = *reinterpret_cast<const uint32_t *>(a.blocks + blk_base(u, key, a.cap) + HYQ_BLK_MASK);
          if ((w >> (key & 31)) & 1u) slot = rbase[key >> 5] + __popc(w & ((1u << (key & 31)) - 1u));
        }
        slot_of[j] = slot;
      }
      __syncthreads();
      issue_cache(a, u, T, k0, k1, slot_of, k0, raw);
    } else {
      issue_fp16(a, u, k0, k1, tiles_s);
    }
    if (u != q_unit || T != q_T) {
      load_qa(a, u, T, warp, lane, qa, qz);
      q_unit = u;
      q_T = T;
    }
    float m[2][2], l[2][2], il[2][2];
    int qpos[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = 32 * warp + 16 * mt + gid + 8 * hr;
        m[mt][hr] = -INFINITY;
        l[mt][hr] = 0.f;
        il[mt][hr] = 0.f;
        qpos[mt][hr] = (row < a.R) ? T - a.n_q + row % a.n_q : -1;  // last visible key
        if (PASS == 2 && row < a.R) {
          const float2 st = a.stats[static_cast<int64_t>(u) * SEL_MAX_ROWS + row];
          m[mt][hr] = st.x;
          il[mt][hr] = st.y;
        }
      }
    if (CACHE) store_cache(raw, tiles, tiles + TILE);
    for (int st = 0; st < nsub; ++st) {
      const int cur = st & 1;
      const int key0 = k0 + st * SEL_SUB;
      const bool more = st + 1 < nsub;
      if (more) {
        if (CACHE) issue_cache(a, u, T, key0 + SEL_SUB, k1, slot_of, k0, raw);
        else issue_fp16(a, u, key0 + SEL_SUB, k1, tiles_s + (cur ^ 1) * 2 * TILE);
      }
      if (!CACHE) {
        if (more) cp_async_wait<1>(); else cp_async_wait<0>();
      }
      __syncthreads();
      float s[2][8][4];
      if (has_rows) {
        tile_scores<CACHE>(tiles_s + cur * 2 * TILE, tiles_s + cur * 2 * TILE + TILE, qa, qz, lane, s);
        if (PASS == 1) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
              float mx = -INFINITY;
#pragma unroll
              for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int key = key0 + nt * 8 + 2 * t4 + e;
                  const bool vis = key < k1 && key <= qpos[mt][hr];
                  float &x = s[mt][nt][2 * hr + e];
                  x = vis ? x : -INFINITY;
                  mx = fmaxf(mx, x);
                }
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
              const float mn = fmaxf(m[mt][hr], mx);
              if (mn == -INFINITY) continue;
              float sum = 0.f;
#pragma unroll
              for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) sum += fast_exp2(s[mt][nt][2 * hr + e] - mn);
              l[mt][hr] = l[mt][hr] * fast_exp2(m[mt][hr] - mn) + sum;
              m[mt][hr] = mn;
            }
        } else {
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float acc = 0.f;
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr)
                  acc += (il[mt][hr] > 0.f) ? fast_exp2(s[mt][nt][2 * hr + e] - m[mt][hr]) * il[mt][hr] : 0.f;
              acc += __shfl_xor_sync(0xffffffffu, acc, 4);
              acc += __shfl_xor_sync(0xffffffffu, acc, 8);
              acc += __shfl_xor_sync(0xffffffffu, acc, 16);
              if (gid == 0) cpart[wl * SEL_SUB + nt * 8 + 2 * t4 + e] = acc;
            }
        }
      } else if (PASS == 2) {
        for (int j = lane; j < SEL_SUB; j += 32) cpart[wl * SEL_SUB + j] = 0.f;
      }
      if (CACHE && more) store_cache(raw, tiles + (cur ^ 1) * 2 * TILE, tiles + (cur ^ 1) * 2 * TILE + TILE);
      __syncthreads();
      if (PASS == 2) {
        for (int j = threadIdx.x; j < SEL_SUB; j += blockDim.x) {
          const int key = key0 + j;
          float tot = 0.f;
          for (int w = 0; w < SEL_BLOCK_ROWS / 32; ++w) tot += cpart[w * SEL_SUB + j];
          if (key < k1) a.colsum_part[(static_cast<int64_t>(rb) * a.U + u) * a.cap + key] = tot;
        }
        __syncthreads();
      }
    }
    if (PASS == 1) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          float lv = l[mt][hr];
          lv += __shfl_xor_sync(0xffffffffu, lv, 1);
          lv += __shfl_xor_sync(0xffffffffu, lv, 2);
          const int row = 32 * warp + 16 * mt + gid + 8 * hr;
          if (t4 == 0 && row < SEL_MAX_ROWS)
            a.stats_part[(static_cast<int64_t>(u) * a.n_chunks + chunk) * SEL_MAX_ROWS + row] =
                make_float2(m[mt][hr], lv);
        }
    }
  }
}

// Cache mode: rank_base[u][w] = vertical-line rows at positions < 32 w
// (exclusive prefix popcount of the unit's mask), so the slot of a position
// is one popcount away.
__global__ void __launch_bounds__(1024) rank_kernel(const SelectArgs a) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  __shared__ int wsum[32];
  const int u = blockIdx.x;
  const int nw = a.cap / 32;
  int32_t *out = a.rank_base + static_cast<int64_t>(u) * nw;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int carry = 0;
  for (int base = 0; base < nw; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int v = (i < nw) ? __popc(*reinterpret_cast<const uint32_t *>(
                                 a.blocks + blk_base(u, static_cast<int64_t>(i) * 32, a.cap) + HYQ_BLK_MASK))
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
  constexpr int MB = 8;  // chunk partials loaded at once
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
  for (int i = tid; i < n; i += blockDim.x) {
    float v;
    if (reduce) {
      v = 0.f;
      for (int z = 0; z < a.n_rb; ++z) v += a.colsum_part[(static_cast<int64_t>(z) * a.U + u) * a.cap + i];
      fin[i] = v;
    } else {
      v = fin[i];
    }
    if (staged) tk_smem[i] = __float_as_uint(v);
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

static cudaError_t select_launch(const SelectArgs &a, bool cache, cudaStream_t s) {
  const size_t smem = 4 * SEL_SUB * 256 + SEL_KC * 4 + (SEL_BLOCK_ROWS / 32) * SEL_SUB * 4;
  static int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaFuncSetAttribute(score_kernel<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(score_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(score_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(score_kernel<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(TOPK_SMEM_VALS * (sizeof(uint32_t) + sizeof(uint16_t))));
    attr_dev = dev;
  }
  const int n_items = a.U * a.n_chunks;
  const int sms = hyq_sm_count_dev();
  const dim3 grid(n_items < sms ? n_items : sms, a.n_rb);
  cudaError_t e;
  if (cache) {
    e = launch(rank_kernel, dim3(a.U), dim3(1024), 0, s, a);
    if (e == cudaSuccess) e = launch(score_kernel<true, 1>, grid, dim3(SEL_THREADS), smem, s, a);
  } else {
    e = launch(score_kernel<false, 1>, grid, dim3(SEL_THREADS), smem, s, a);
  }
  if (e == cudaSuccess) e = launch(stats_merge_kernel, dim3(a.U), dim3(256), 0, s, a);
  if (e == cudaSuccess) e = launch(cache ? score_kernel<true, 2> : score_kernel<false, 2>, grid, dim3(SEL_THREADS), smem, s, a);
  if (e == cudaSuccess) e = launch(topk_kernel, dim3(a.U), dim3(TOPK_THREADS), TOPK_SMEM_VALS * (sizeof(uint32_t) + sizeof(uint16_t)), s, a);
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

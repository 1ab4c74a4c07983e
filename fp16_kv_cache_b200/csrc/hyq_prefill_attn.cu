// hyq_prefill_attn.cu -- the prefill-stage hybrid-precision attention
// operator: causal attention over a prompt in which the quantized majority
// of (query, key) pairs is computed from INT4-dequantized queries, keys and
// values, while the vertical-line keys and each query's local window are
// computed in FP16, all in one softmax per query row.
//
// Method: HyQuant.  aifromscratch.in explainer, "Two Operational Modes /
// Prefill Stage": a fused operator computes the quantized majority and
// overlays the high-precision vertical lines and local window into the same
// result; wpnews.pro summary: the bulk of the query, key and value tensors is
// quantized to low bit widths while vertical-line tokens and a local sliding
// window stay in full precision; kipquest.com abstract: in the prefill stage
// a hybrid-precision quantized attention operator keeps vertical-line tokens
// and a local sliding window in full precision.
// Reading (the pages do not define the pairs exactly): query row i and key
// j <= i form a high-precision pair when j is a vertical line of the unit or
// lies in the query's own window (j > i - 128); it then uses the FP16 q_i,
// k_j, v_j.  Every other pair uses q_i, k_j, v_j quantized on the cache's
// INT4 grid (per token, groups of 32 channels) and dequantized.
//
// Kernels (stream ordered):
//   1. pa_rows_kernel  16 threads per row: quantizes every prompt query row
//      and key row and writes the dequantized values as fp16 hi + lo (x =
//      hi + lo to about 22 bits), zeros past the sequence end.
//   2. pa_vt_kernel    one block per (unit, 64-key tile): quantizes the value
//      rows, and writes the tile transposed ([128 channels][64 keys]) twice,
//      dequantized and in FP16, through shared memory; the same for the
//      unit's vertical-line value rows (FP16).
//   3. pa_attn_kernel  one block per (batch, query head, 128-row query
//      tile), the longest tiles first: 8 epilogue warps, in which two
//      threads own each query row, each with half of the key columns of a
//      tile and half of the output columns, and a ninth warp whose one
//      thread issues and commits every MMA, so that no epilogue warp waits
//      for the tensor cores to accept MMAs.
//      The 5th-generation tensor cores (tcgen05, fp16 operands in shared
//      memory with the 128-byte swizzle, fp32 accumulators in tensor memory)
//      compute, per 64-key tile,
//        S_lo = Q^hi K^hi^T + Q^hi K^lo^T + Q^lo K^hi^T
//                                     quantized pairs (three MMAs; fp16
//                                     operands alone miss the tolerance),
//        S_hi = Q K^T                high-precision pairs (band tiles and
//                                     vertical-line tiles only),
//      the epilogue picks each pair's score, masks, and updates the row's
//      online softmax (the running max is raised only when a tile's max
//      exceeds it by more than 8 in the exp2 domain, so the accumulator in
//      tensor memory is rescaled rarely), writes P as fp16, and the tensor
//      cores accumulate O += P_lo V^ + P_hi V.  Key tiles: the vertical-line
//      rows (FP16, pairs with j <= i - 128) and the band tiles around the
//      diagonal first (phase A, one key, value and score buffer), then the
//      off-diagonal tiles, which hold quantized pairs only (their vertical
//      lines are masked out there): in phase B the space of phase A's FP16
//      tiles double-buffers keys, values and scores, and the scores of tile
//      t + 1 and P V of tile t - 1 run on the tensor cores during tile t's
//      epilogue.
//   Output: O fp32 (the operands are already rounded to fp16 for the tensor
//   cores; an fp16 output rounding would spend the rest of the tolerance)
//   and the row's log-sum-exp.
#include <climits>

#include "hyq_common.cuh"
#include "hyq_quant.cuh"

extern "C" int32_t hyq_sm_count(void);                      // hyq_api.cu
extern "C" hyq_status hyq_check_cache(const hyq_cache *c);  // hyq_api.cu

namespace hyq {
namespace pa {

constexpr int QT = 128;      // query rows per tile (the MMA's M)
constexpr int KT = 64;       // keys per tile (N of Q K^T, K of P V)
constexpr int EPI_THREADS = 256;          // the epilogue warps: two threads per query row
constexpr int THREADS = EPI_THREADS + 32;  // and one warp that issues the MMAs
constexpr int ISSUER = EPI_THREADS;       // the thread that issues and commits every MMA
constexpr float SCALE_LOG2 = 0.12751743082459868f;  // log2(e) / sqrt(128)
constexpr float LN2 = 0.69314718055994531f;
constexpr float RAISE = 8.f;  // raise the running max only past this margin (exp2 domain)

constexpr int TILE_Q = QT * D * 2;   // [128 rows][128 ch] fp16
constexpr int TILE_K = KT * D * 2;   // [64 keys][128 ch]
constexpr int TILE_V = D * KT * 2;   // [128 ch][64 keys]
constexpr int TILE_P = QT * KT * 2;  // [128 rows][64 keys]
// shared memory: Q^hi, Q^lo, Q, K^hi, K^lo, K, V^t, Vt, P_lo, P_hi
constexpr int OFF_QH = 0, OFF_QL = OFF_QH + TILE_Q, OFF_QF = OFF_QL + TILE_Q, OFF_KH = OFF_QF + TILE_Q, OFF_KL = OFF_KH + TILE_K,
              OFF_KF = OFF_KL + TILE_K, OFF_VQ = OFF_KF + TILE_K, OFF_VF = OFF_VQ + TILE_V,
              OFF_PL = OFF_VF + TILE_V, OFF_PH = OFF_PL + TILE_P, SMEM_TILES = OFF_PH + TILE_P;
constexpr int SMEM_BYTES = SMEM_TILES + 1024;  // + alignment of the swizzled tiles to 1024 B
// tensor memory columns: S_lo [64], S_hi [64], O [128]
constexpr uint32_t TM_SLO = 0, TM_SHI = 64, TM_O = 128, TM_COLS = 256;

struct Args {
  int B, Hq, Hkv, G, cap, W, vl_cap, U;
  const __half *q, *k, *v;  // [B][Hq][cap][128], [B][Hkv][cap][128] x 2
  const uint8_t *blocks;    // the cache's block records (vertical-line bitmask)
  RecMap rm;                // record addresses (contiguous or through the block table)
  const __half *vl_k, *vl_v;
  const int32_t *vl_pos, *vl_count, *seq_len;
  __half *qh, *ql, *kh, *kl;  // workspace: dequantized rows (hi, lo)
  __half *vqt, *vft, *vlt;  // workspace: transposed value tiles [..][128][64]
  float *o, *lse;
  uint32_t *status;
};

// Byte offset of element (row r, column c) in a K-major fp16 tile of R rows
// with the 128-byte swizzle: columns 0-63 and 64-127 form two halves of
// R x 128 bytes; within a half, row r is 128 bytes at r * 128 and its 16-byte
// chunk k sits at position k ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int R, int r, int c) {
  return (c >> 6) * (R * 128) + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2;
}
// Shared-memory matrix descriptor of k-step ks (16 columns) of such a tile:
// start address, leading offset unused with the swizzle, 1024 bytes between
// 8-row groups, descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t desc(uint32_t tile, int R, int ks) {
  const uint32_t start = tile + (ks >> 2) * (R * 128) + (ks & 3) * 32;
  return static_cast<uint64_t>((start >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}
// desc(tile, R, ks) - desc(tile, R, 0), in the start-address field (16-byte
// units; tiles lie below 256 KB, so the field never carries).
__device__ __forceinline__ uint32_t koff(int R, int ks) { return (ks >> 2) * (R * 8) + (ks & 3) * 2; }
// Instruction descriptor: fp32 accumulate, fp16 A and B, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc(int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(id), "r"(accumulate), "r"(0u));
}
__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tm_ld32(uint32_t taddr, float (&v)[32]) {
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
__device__ __forceinline__ void tm_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void cp16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void st_zero16(uint32_t dst) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(dst), "r"(0u) : "memory");
}

// This thread's 8 channels of one row, quantized and dequantized: x = zero +
// code * scale in fp32 (the product is exact, one rounding in the add).
// `t` = the thread's 16-lane group index, `hmask` = the group's lanes.
__device__ __forceinline__ void dequant8(uint4 x, int t, unsigned hmask, uint32_t *status, float (&y)[8]) {
  const QuantShare q = quantize_share(x, t, hmask, status);
  // my 8 codes: channels 8t..8t+7 are pieces 2 (t % 4), 2 (t % 4) + 1 of
  // group t / 4; rebuild them from the packed words of the group's even lane
  const int g = t >> 2, sub = t & 3, h = g >> 1, odd = g & 1;
  const unsigned base = (hmask == 0xFFFFu) ? 0u : 16u;
  const int lane_even = static_cast<int>(base) + 8 * h + sub;  // the lane holding w0/w1 of my pieces
  const uint32_t w0 = __shfl_sync(hmask, q.w0, lane_even), w1 = __shfl_sync(hmask, q.w1, lane_even);
  const __half2 sz = u2h(q.sz);
  const float sc = __low2float(sz), zr = __high2float(sz);
  // word (p, h) = {g2h.j0, g2h+1.j0, g2h.j1, g2h+1.j1}: byte 2j + odd holds
  // channels 4p + 2j (low nibble) and 4p + 2j + 1 (high nibble)
#pragma unroll
  for (int pc = 0; pc < 2; ++pc) {
    const uint32_t w = pc ? w1 : w0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t byte = (w >> (8 * (2 * j + odd))) & 0xFFu;
      y[4 * pc + 2 * j] = fmaf(static_cast<float>(byte & 15u), sc, zr);
      y[4 * pc + 2 * j + 1] = fmaf(static_cast<float>(byte >> 4), sc, zr);
    }
  }
}

// Prepass 1: query rows [B][Hq][cap] then key rows [U][cap], 16 threads each.
__global__ void __launch_bounds__(256) pa_rows_kernel(const Args a, int64_t n_q_rows, int64_t n_rows) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, t = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  if (row >= n_rows) return;  // uniform over a row's 16 lanes
  const bool is_q = row < n_q_rows;
  const int64_t r = is_q ? row : row - n_q_rows;
  const int p = static_cast<int>(r % a.cap);
  const int b = static_cast<int>((r / a.cap) / (is_q ? a.Hq : a.Hkv));
  const int T = a.seq_len[b];
  uint4 hi = make_uint4(0, 0, 0, 0), lo = make_uint4(0, 0, 0, 0);
  if (T >= 0 && T <= a.cap && p < T) {
    const uint4 x = *reinterpret_cast<const uint4 *>((is_q ? a.q : a.k) + r * D + 8 * t);
    float y[8];
    dequant8(x, t, hmask, a.status, y);
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hv = __floats2half2_rn(y[2 * i], y[2 * i + 1]);
      const float2 hf = __half22float2(hv);
      hw[i] = h2u(hv);
      lw[i] = h2u(__floats2half2_rn(y[2 * i] - hf.x, y[2 * i + 1] - hf.y));
    }
    hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  if (is_q) {
    *reinterpret_cast<uint4 *>(a.qh + r * D + 8 * t) = hi;
    *reinterpret_cast<uint4 *>(a.ql + r * D + 8 * t) = lo;
  } else {
    *reinterpret_cast<uint4 *>(a.kh + r * D + 8 * t) = hi;
    *reinterpret_cast<uint4 *>(a.kl + r * D + 8 * t) = lo;
  }
}

// Prepass 2: block (unit, tile) for tile < cap / 64: the value tile
// dequantized and FP16, transposed; tile >= cap / 64: vertical-line value
// rows (FP16), transposed.  256 threads.
constexpr int VT_PAD = KT + 8;  // smem row pitch (fp16) of the transposed tiles
__global__ void __launch_bounds__(256) pa_vt_kernel(const Args a) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) __half sq[D][VT_PAD];
  __shared__ __align__(16) __half sf[D][VT_PAD];
  const int n_kt = a.cap / KT, n_vt = (a.vl_cap + KT - 1) / KT;
  const int u = blockIdx.x / (n_kt + n_vt), tile = blockIdx.x % (n_kt + n_vt);
  const bool is_vl = tile >= n_kt;
  const int b = u / a.Hkv;
  const int T = a.seq_len[b];
  const int n_valid = is_vl ? min(max(a.vl_count[u], 0), a.vl_cap) : ((T >= 0 && T <= a.cap) ? T : 0);
  const int r0 = (is_vl ? tile - n_kt : tile) * KT;
  const int lane = threadIdx.x & 31, t = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  for (int rr = threadIdx.x >> 4; rr < KT; rr += 16) {
    const int rw = r0 + rr;
    float y[8];
    uint4 x = make_uint4(0, 0, 0, 0);
    const bool ok = rw < n_valid;
    if (ok) {
      const __half *src = is_vl ? a.vl_v + (static_cast<int64_t>(u) * a.vl_cap + rw) * D
                                : a.v + (static_cast<int64_t>(u) * a.cap + rw) * D;
      x = *reinterpret_cast<const uint4 *>(src + 8 * t);
    }
    if (!is_vl && ok) {
      dequant8(x, t, hmask, a.status, y);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = 0.f;
    }
    const __half *xh = reinterpret_cast<const __half *>(&x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sq[8 * t + i][rr] = __float2half_rn(y[i]);
      sf[8 * t + i][rr] = xh[i];
    }
  }
  __syncthreads();
  // [128 ch][64 keys] = 1024 chunks of 16 bytes per tile
  const int64_t tile_idx = is_vl ? static_cast<int64_t>(u) * n_vt + (tile - n_kt) : static_cast<int64_t>(u) * n_kt + tile;
  for (int c = threadIdx.x; c < D * (KT / 8); c += blockDim.x) {
    const int ch = c >> 3, kc = c & 7;
    const uint4 vf = *reinterpret_cast<const uint4 *>(&sf[ch][8 * kc]);
    if (is_vl) {
      *reinterpret_cast<uint4 *>(a.vlt + (tile_idx * D + ch) * KT + 8 * kc) = vf;
    } else {
      *reinterpret_cast<uint4 *>(a.vft + (tile_idx * D + ch) * KT + 8 * kc) = vf;
      *reinterpret_cast<uint4 *>(a.vqt + (tile_idx * D + ch) * KT + 8 * kc) =
          *reinterpret_cast<const uint4 *>(&sq[ch][8 * kc]);
    }
  }
}

// Wait (bounded) for the MMAs committed to `bar`; on a timeout raise the
// status and the block's abort flag.
__device__ __forceinline__ void mma_wait(uint32_t bar, uint32_t parity, const Args &a, volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return;
    if (global_ns() - t0 > 2000000000ull) {
      set_status(a.status, HYQ_DEV_TIMEOUT);
      *abort = 1;
      return;
    }
  }
}

enum { JOB_VL = 0, JOB_OFF = 1, JOB_BAND = 2 };

__global__ void __launch_bounds__(THREADS, 1) pa_attn_kernel(const Args a) {
  pdl_trigger();
  pdl_wait();  // the prepass is complete (and any tensor memory of earlier kernels freed)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ uint32_t tmem_base;
  __shared__ __align__(8) uint64_t bars[1];  // phase A: each commit is P V of one job and S of the next
  __shared__ __align__(8) uint64_t bars_b[3];  // phase B: S into score buffer 0, 1; P V
  __shared__ int s_abort;
  __shared__ uint32_t s_vlmask[3][2];        // bitmask words of a 64-key tile (up to three jobs in flight)
  __shared__ int s_vlpos[2][KT];             // positions of a vertical-line tile
  __shared__ float s_red[2][QT];             // the two halves' tile max (and, at the end, row sums)
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool ep = tid < EPI_THREADS;  // an epilogue thread (else the issuer's warp)
  const int BH = a.B * a.Hq;
  const int n_qt = a.cap / QT;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / BH;  // longest tiles first
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / a.Hq, h = bh % a.Hq, u = b * a.Hkv + h / a.G;
  const int T = a.seq_len[b];
  const int q0 = qt * QT;
  if (T < 0 || T > a.cap) {
    if (tid == 0 && qt == 0 && h == 0) set_status(a.status, HYQ_DEV_BADLEN);
    return;
  }
  if (q0 >= T) return;
  int n_vl = a.vl_count[u];
  if (n_vl < 0 || n_vl > a.vl_cap) {
    if (tid == 0 && qt == 0 && h % a.G == 0) set_status(a.status, HYQ_DEV_BADLEN);
    n_vl = 0;
  }

  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t s0 = smem_u32(sm);
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                 "r"(TM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
#pragma unroll
    for (int t = 0; t < 3; ++t) mbar_init(smem_u32(&bars_b[t]), 1);
    fence_barrier_init();
    s_abort = 0;
  }
  // the query tile: Q^ (dequantized, from the prepass) and Q (FP16); rows
  // past T are zero
  {
    const __half *qh = a.qh + (static_cast<int64_t>(bh) * a.cap + q0) * D;
    const __half *ql = a.ql + (static_cast<int64_t>(bh) * a.cap + q0) * D;
    const __half *qf = a.q + (static_cast<int64_t>(bh) * a.cap + q0) * D;
    for (int c = tid; c < QT * 16; c += THREADS) {
      const int r = c >> 4, cc = c & 15;
      const uint32_t off = swz(QT, r, 8 * cc);
      if (q0 + r < T) {
        cp16(s0 + OFF_QH + off, qh + r * D + 8 * cc);
        cp16(s0 + OFF_QL + off, ql + r * D + 8 * cc);
        cp16(s0 + OFF_QF + off, qf + r * D + 8 * cc);
      } else {
        st_zero16(s0 + OFF_QH + off);
        st_zero16(s0 + OFF_QL + off);
        st_zero16(s0 + OFF_QF + off);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;
  // Thread (warp w, lane l) owns query row rr = 32 (w % 4) + l -- the tensor
  // memory lanes its warp may access -- and half hf = w / 4 of the columns:
  // key columns 32 hf .. 32 hf + 31 of each tile's scores, and output
  // columns 64 hf .. 64 hf + 63.  The two threads of a row keep the same
  // running max (the tile max is exchanged through shared memory) and their
  // own partial sums.
  const int rq = warp & 3, hf = warp >> 2, rr = 32 * rq + (tid & 31);
  const uint32_t tm_row = tm + (static_cast<uint32_t>(32 * rq) << 16);
  volatile int *abort = &s_abort;

  const int i = q0 + rr;  // this thread's query row
  float m_run = -INFINITY, l_run = 0.f;
  bool o_started = false;   // the first P V MMA overwrites O
  uint32_t ph = 0;

  // Phase A: the vertical-line tiles, then the band tiles band0 .. n_kt - 1
  // near the diagonal (the jobs with high-precision pairs).  Phase B: the
  // off-diagonal key tiles 0 .. band0 - 1 (quantized pairs only), with the
  // FP16 tiles of phase A dead, so that their space double-buffers keys,
  // values and scores.  The softmax is the same in any order of key tiles.
  const int n_vlt = (n_vl + KT - 1) / KT;
  const int last_key = min(q0 + QT, T) - 1;
  const int n_kt = last_key / KT + 1;
  const int band0 = max(0, (q0 - a.W + 1) / KT);  // first key tile holding a pair j > i - W
  const int n_jobs = n_vlt + (n_kt - band0);      // phase A
  const int n_off = band0;                        // phase B
  const __half *kbase = a.k + static_cast<int64_t>(u) * a.cap * D;
  const __half *khb = a.kh + static_cast<int64_t>(u) * a.cap * D;
  const __half *klb = a.kl + static_cast<int64_t>(u) * a.cap * D;

  // Phase A job j: the vertical-line tile j (j < n_vlt) or band key tile
  // band0 + j - n_vlt.
  auto job_kind = [&](int job, int &kt) {
    const bool is_vl = job < n_vlt;
    kt = is_vl ? job : band0 + job - n_vlt;
    return is_vl ? JOB_VL : JOB_BAND;
  };
  // Loads of a job's key rows (and the tile's vertical-line bitmask or
  // positions, into mask buffer mb) as one cp.async group, and of its value
  // tiles as another.  Rows past the end are zero-filled.  Each thread
  // copies the same four 16-byte pieces of every tile: key rows kr + 16 it,
  // piece kc (shared offset + 2048 it, global + 16 D it), value rows
  // vr + 32 it, piece vc (shared offset + 4096 it, global + 32 KT it).
  const int kr = tid >> 4, kc = tid & 15, vr = tid >> 3, vc = tid & 7;
  const uint32_t ks_off = swz(KT, kr, 8 * kc), vs_off = swz(D, vr, 8 * vc);
  const int kg_off = kr * D + 8 * kc, vg_off = vr * KT + 8 * vc;
  auto load_keys = [&](int job, int mb) {
    int kt;
    const int kind = job_kind(job, kt), j0 = kt * KT;
    if (kind == JOB_VL) {
      const __half *src = a.vl_k + (static_cast<int64_t>(u) * a.vl_cap + j0) * D + kg_off;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        if (j0 + kr + 16 * it < n_vl)
          cp16(s0 + OFF_KF + ks_off + 2048 * it, src + 16 * D * it);
        else
          st_zero16(s0 + OFF_KF + ks_off + 2048 * it);
      }
    } else {
      const int64_t ro = static_cast<int64_t>(j0) * D + kg_off;
#pragma unroll
      for (int it = 0; it < 4; ++it) {  // zeros past T (prepass)
        cp16(s0 + OFF_KH + ks_off + 2048 * it, khb + ro + 16 * D * it);
        cp16(s0 + OFF_KL + ks_off + 2048 * it, klb + ro + 16 * D * it);
      }
      if (kind == JOB_BAND) {
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          if (j0 + kr + 16 * it < T)
            cp16(s0 + OFF_KF + ks_off + 2048 * it, kbase + ro + 16 * D * it);
          else
            st_zero16(s0 + OFF_KF + ks_off + 2048 * it);
        }
      }
    }
    if (kind == JOB_VL && tid < KT) {
      if (j0 + tid < n_vl)
        cp4(smem_u32(&s_vlpos[mb][tid]), a.vl_pos + static_cast<int64_t>(u) * a.vl_cap + j0 + tid);
      else
        s_vlpos[mb][tid] = INT_MAX;
    }
    if (kind != JOB_VL && tid < 2) {
      if (j0 + 32 * tid < T)
        cp4(smem_u32(&s_vlmask[mb][tid]), a.blocks + rec_mask(a.rm.rec_rd(u, j0 + 32 * tid)));
      else
        s_vlmask[mb][tid] = 0u;
    }
    cp_commit();
  };
  auto load_values = [&](int job) {  // [128 ch][64 keys], zeros past the end (prepass)
    int kt;
    const int kind = job_kind(job, kt);
    if (kind == JOB_VL) {
      const __half *src = a.vlt + (static_cast<int64_t>(u) * ((a.vl_cap + KT - 1) / KT) + kt) * D * KT + vg_off;
#pragma unroll
      for (int it = 0; it < 4; ++it) cp16(s0 + OFF_VF + vs_off + 4096 * it, src + 32 * KT * it);
    } else {
      const int64_t tb = (static_cast<int64_t>(u) * (a.cap / KT) + kt) * D * KT + vg_off;
#pragma unroll
      for (int it = 0; it < 4; ++it) cp16(s0 + OFF_VQ + vs_off + 4096 * it, a.vqt + tb + 32 * KT * it);
      if (kind == JOB_BAND)
#pragma unroll
        for (int it = 0; it < 4; ++it) cp16(s0 + OFF_VF + vs_off + 4096 * it, a.vft + tb + 32 * KT * it);
    }
    cp_commit();
  };
  // S = Q K^T of a job: the quantized pairs from the hi/lo operands, the
  // high-precision pairs from the FP16 ones (issued by thread ISSUER).
  auto issue_s = [&](int job) {
    int kt;
    const int kind = job_kind(job, kt);
    // k-step ks of a tile = its descriptor advanced by koff(R, ks) (the
    // start-address field counts 16-byte units)
    const uint64_t dqh = desc(s0 + OFF_QH, QT, 0), dql = desc(s0 + OFF_QL, QT, 0), dqf = desc(s0 + OFF_QF, QT, 0);
    const uint64_t dkh = desc(s0 + OFF_KH, KT, 0), dkl = desc(s0 + OFF_KL, KT, 0), dkf = desc(s0 + OFF_KF, KT, 0);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t oq = koff(QT, ks), ok = koff(KT, ks);
      if (kind != JOB_VL) {
        mma(tm + TM_SLO, dqh + oq, dkh + ok, idesc(KT), ks > 0);
        mma(tm + TM_SLO, dqh + oq, dkl + ok, idesc(KT), 1u);
        mma(tm + TM_SLO, dql + oq, dkh + ok, idesc(KT), 1u);
      }
      if (kind != JOB_OFF) mma(tm + TM_SHI, dqf + oq, dkf + ok, idesc(KT), ks > 0);
    }
  };
  // Software pipeline over the single key and value buffers.  One commit
  // covers P V of job - 1 and S of job; once it completes, the keys of
  // job + 1 and the values of job load during job's epilogue, and after the
  // block barrier thread ISSUER (in a warp of its own, so the epilogue
  // warps never wait for the tensor cores to accept MMAs) issues P V of job
  // and S of job + 1 together.
  if (n_jobs > 0) {
    if (ep) {
      load_keys(0, 0);
      load_values(0);
      cp_wait_group<1>();  // the keys of job 0
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == ISSUER) {
      issue_s(0);
      commit(smem_u32(&bars[0]));
    }
  }
  for (int job = 0; job < n_jobs && !*abort; ++job) {
    int kt;
    const int kind = job_kind(job, kt), j0 = kt * KT, mb = job & 1;
    if (ep) {  // the issuer's warp skips to the barrier below
      mma_wait(smem_u32(&bars[0]), ph, a, abort);
      ph ^= 1u;
      tc_fence_after();
      // S of this job and P V of the previous one are complete: the key and
      // value buffers are free
      if (job + 1 < n_jobs) load_keys(job + 1, mb ^ 1);
      if (job > 0) load_values(job);
      // ---- epilogue: this thread's row, its 32 of the tile's 64 key columns,
      // read once from tensor memory (chunk: band and vertical-line tiles)
      auto chunk = [&](int cb, float (&x)[32], uint32_t &hmask32) {
        float lo_v[32], hi_v[32];
        if (kind != JOB_VL) tm_ld32(tm_row + TM_SLO + 32 * cb, lo_v);
        if (kind != JOB_OFF) tm_ld32(tm_row + TM_SHI + 32 * cb, hi_v);
        const uint32_t vlw = (kind != JOB_VL) ? s_vlmask[mb][cb] : 0u;
        hmask32 = 0u;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int c = 32 * cb + jj, j = j0 + c;
          float v = -INFINITY;
          if (kind == JOB_VL) {
            // vertical line j of the unit: counted here when it lies outside
            // the query's window (inside it, the band tile has it)
            if (j < n_vl && s_vlpos[mb][c] <= i - a.W) {
              v = hi_v[jj];
              hmask32 |= 1u << jj;
            }
          } else if (kind == JOB_OFF) {
            if (!((vlw >> jj) & 1u)) v = lo_v[jj];
          } else if (j <= i) {
            if (j > i - a.W) {
              v = hi_v[jj];
              hmask32 |= 1u << jj;
            } else if (!((vlw >> jj) & 1u)) {
              v = lo_v[jj];
            }
          }
          x[jj] = (v == -INFINITY) ? -INFINITY : v * SCALE_LOG2;
        }
      };
      // This thread's 32 scores of the tile, read once.  Off-diagonal tiles
      // (all pairs quantized, the only mask the tile's vertical-line bits)
      // keep the raw scores: scaling by SCALE_LOG2 > 0 is monotone, so the
      // scaled max is the max scaled, and the scale folds into the exp2
      // argument.  Band and vertical-line tiles keep x = score * SCALE_LOG2.
      const bool off = kind == JOB_OFF;
      float x[32];
      uint32_t hm = 0u;
      float mx = -INFINITY;
      if (off) {
        tm_ld32(tm_row + TM_SLO + 32 * hf, x);
        const uint32_t vlw = s_vlmask[mb][hf];
        if (vlw != 0u) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if ((vlw >> jj) & 1u) x[jj] = -INFINITY;
        }
        float m4[4] = {x[0], x[1], x[2], x[3]};  // four independent chains
#pragma unroll
        for (int jj = 4; jj < 32; ++jj) m4[jj & 3] = fmaxf(m4[jj & 3], x[jj]);
        mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * SCALE_LOG2;
      } else {
        chunk(hf, x, hm);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) mx = fmaxf(mx, x[jj]);
      }
      // the two threads of a row (warps rq and rq + 4) exchange their halves'
      // max on a 64-thread barrier of their own
      s_red[hf][rr] = mx;
      asm volatile("bar.sync %0, 64;" ::"r"(1 + rq) : "memory");
      mx = fmaxf(s_red[0][rr], s_red[1][rr]);  // the same in both threads of the row
      // raise the running max only when this tile exceeds it by more than
      // RAISE (p stays <= 2^RAISE); O and l are rescaled then
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_run + RAISE || (m_run == -INFINITY && mx != -INFINITY)) {
        const float m_new = mx;
        if (m_run != -INFINITY) {
          alpha = fast_exp2(m_run - m_new);
          rescale = o_started;
        }
        l_run *= alpha;
        m_run = m_new;
      }
      // O row *= alpha (the previous P V MMAs are complete); tensor-memory
      // loads and stores take the whole warp, so a warp with any row to
      // rescale rescales all of its rows (by 1 where nothing changed)
      if (__any_sync(0xffffffffu, rescale)) {
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {  // this thread's half of the row
          float ov[32];
          tm_ld32(tm_row + TM_O + 32 * cb, ov);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) ov[jj] *= f;
          tm_st32(tm_row + TM_O + 32 * cb, ov);
        }
      }
      // P as fp16 into P_lo / P_hi: row rr, this thread's 32 columns
      float lsum = 0.f;
      if (off) {
        // m_run is -inf only when every score so far, this tile's included,
        // is masked: then every p is exp2(-inf) = 0
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        float l4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t wl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = 8 * cc + 2 * e;
            const float p0 = fast_exp2(fmaf(x[c0], SCALE_LOG2, neg_m));
            const float p1 = fast_exp2(fmaf(x[c0 + 1], SCALE_LOG2, neg_m));
            l4[e] += p0 + p1;
            wl[e] = pack_half2(p0, p1);
          }
          const uint32_t off_p = swz(QT, rr, 32 * hf + 8 * cc);
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(s0 + OFF_PL + off_p), "r"(wl[0]), "r"(wl[1]),
                       "r"(wl[2]), "r"(wl[3]) : "memory");
        }
        lsum = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t wl[4], wh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = 8 * cc + 2 * e;
            const float p0 = (x[c0] == -INFINITY) ? 0.f : fast_exp2(x[c0] - m_run);
            const float p1 = (x[c0 + 1] == -INFINITY) ? 0.f : fast_exp2(x[c0 + 1] - m_run);
            lsum += p0 + p1;
            const uint32_t pk = pack_half2(p0, p1);
            const uint32_t keep_hi = (((hm >> c0) & 1u) ? 0x0000FFFFu : 0u) | (((hm >> (c0 + 1)) & 1u) ? 0xFFFF0000u : 0u);
            wh[e] = pk & keep_hi;
            wl[e] = pk & ~keep_hi;
          }
          const uint32_t off_p = swz(QT, rr, 32 * hf + 8 * cc);
          if (kind != JOB_VL)
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(s0 + OFF_PL + off_p), "r"(wl[0]), "r"(wl[1]),
                         "r"(wl[2]), "r"(wl[3]) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(s0 + OFF_PH + off_p), "r"(wh[0]), "r"(wh[1]),
                       "r"(wh[2]), "r"(wh[3]) : "memory");
        }
      }
      l_run += lsum;
      cp_wait_group<0>();  // this job's values and the next job's keys
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- O += P_lo V^ + P_hi V, then S of the next job
    if (tid == ISSUER) {
      uint32_t acc = o_started ? 1u : 0u;
      const uint64_t dpl = desc(s0 + OFF_PL, QT, 0), dph = desc(s0 + OFF_PH, QT, 0);
      const uint64_t dvq = desc(s0 + OFF_VQ, D, 0), dvf = desc(s0 + OFF_VF, D, 0);
#pragma unroll
      for (int ks = 0; ks < KT / 16; ++ks) {
        const uint32_t op = koff(QT, ks), ov = koff(D, ks);
        if (kind != JOB_VL) {
          mma(tm + TM_O, dpl + op, dvq + ov, idesc(D), acc);
          acc = 1u;
        }
        if (kind != JOB_OFF) {
          mma(tm + TM_O, dph + op, dvf + ov, idesc(D), acc);
          acc = 1u;
        }
      }
      if (job + 1 < n_jobs) issue_s(job + 1);
      commit(smem_u32(&bars[0]));
    }
    o_started = true;
  }
  // the last P V (nothing is in flight after an abort's timeout but what
  // the timed-out wait gave up on)
  if (ep && n_jobs > 0 && !*abort) {
    mma_wait(smem_u32(&bars[0]), ph, a, abort);
    tc_fence_after();
  }

  // ---- Phase B: off-diagonal key tile t (t < n_off) uses key buffer t & 1
  // (K^hi, K^lo at OFF_KH, OFF_KL or in the dead Q region), value buffer
  // t & 1 (OFF_VQ or the dead OFF_VF), score buffer t & 1 (tensor-memory
  // columns TM_SLO or the dead TM_SHI) and mask slot t % 3.  S of tile t + 2
  // is issued as soon as tile t's scores have been read, so the tensor cores
  // compute P V of tile t - 1 and S of tile t + 1 during tile t's epilogue.
  // P V and S are committed to barriers of their own: the epilogue waits
  // for P V of the previous tile only before it rescales O or writes P.
  auto kbuf_h = [&](int t) { return s0 + ((t & 1) ? OFF_QF : OFF_KH); };
  auto kbuf_l = [&](int t) { return s0 + ((t & 1) ? OFF_QF + TILE_K : OFF_KL); };
  auto vbuf = [&](int t) { return s0 + ((t & 1) ? OFF_VF : OFF_VQ); };
  auto load_keys_b = [&](int t) {
    const int j0 = t * KT;
    const int64_t ro = static_cast<int64_t>(j0) * D + kg_off;
    const uint32_t dh = kbuf_h(t) + ks_off, dl = kbuf_l(t) + ks_off;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      cp16(dh + 2048 * it, khb + ro + 16 * D * it);
      cp16(dl + 2048 * it, klb + ro + 16 * D * it);
    }
    if (tid < 2) {
      if (j0 + 32 * tid < T)
        cp4(smem_u32(&s_vlmask[t % 3][tid]), a.blocks + rec_mask(a.rm.rec_rd(u, j0 + 32 * tid)));
      else
        s_vlmask[t % 3][tid] = 0u;
    }
    cp_commit();
  };
  auto load_values_b = [&](int t) {
    const int64_t tb = (static_cast<int64_t>(u) * (a.cap / KT) + t) * D * KT + vg_off;
    const uint32_t dv = vbuf(t) + vs_off;
#pragma unroll
    for (int it = 0; it < 4; ++it) cp16(dv + 4096 * it, a.vqt + tb + 32 * KT * it);
    cp_commit();
  };
  auto issue_s_b = [&](int t) {  // thread ISSUER
    const uint64_t dqh = desc(s0 + OFF_QH, QT, 0), dql = desc(s0 + OFF_QL, QT, 0);
    const uint64_t dkh = desc(kbuf_h(t), KT, 0), dkl = desc(kbuf_l(t), KT, 0);
    const uint32_t d = tm + ((t & 1) ? TM_SHI : TM_SLO);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t oq = koff(QT, ks), ok = koff(KT, ks);
      mma(d, dqh + oq, dkh + ok, idesc(KT), ks > 0);
      mma(d, dqh + oq, dkl + ok, idesc(KT), 1u);
      mma(d, dql + oq, dkh + ok, idesc(KT), 1u);
    }
  };
  if (n_off > 0 && !*abort) {
    if (ep) {
      load_keys_b(0);
      load_values_b(0);
      if (n_off > 1) load_keys_b(1); else cp_commit();
      cp_wait_group<0>();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == ISSUER) {
      issue_s_b(0);
      commit(smem_u32(&bars_b[0]));
      if (n_off > 1) {
        issue_s_b(1);
        commit(smem_u32(&bars_b[1]));
      }
    }
    uint32_t ph_s0 = 0u, ph_s1 = 0u, ph_o = 0u;  // bars_b[0], [1], [2]
    for (int t = 0; t < n_off && !*abort; ++t) {
      const int sb = t & 1;
      if (ep) {  // the issuer's warp skips to the barrier below
        mma_wait(smem_u32(&bars_b[sb]), sb ? ph_s1 : ph_s0, a, abort);
        if (sb) ph_s1 ^= 1u; else ph_s0 ^= 1u;
        tc_fence_after();
        // S of tile t is complete: its key buffer takes tile t + 2
        if (t + 2 < n_off) load_keys_b(t + 2); else cp_commit();
        // the raw scores of this thread's 32 columns, masked by the tile's
        // vertical-line bits; the scale folds into the exp2 argument
        float x[32];
        tm_ld32(tm_row + (sb ? TM_SHI : TM_SLO) + 32 * hf, x);
        const uint32_t vlw = s_vlmask[t % 3][hf];
        if (vlw != 0u) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if ((vlw >> jj) & 1u) x[jj] = -INFINITY;
        }
        float mx;
        {
          float m4[4] = {x[0], x[1], x[2], x[3]};  // four independent chains
#pragma unroll
          for (int jj = 4; jj < 32; ++jj) m4[jj & 3] = fmaxf(m4[jj & 3], x[jj]);
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * SCALE_LOG2;
        }
        s_red[hf][rr] = mx;
        asm volatile("bar.sync %0, 64;" ::"r"(1 + rq) : "memory");
        mx = fmaxf(s_red[0][rr], s_red[1][rr]);
        // P V of tile t - 1 is complete: O may be rescaled, P overwritten, and
        // its value buffer takes tile t + 1
        if (t > 0) {
          mma_wait(smem_u32(&bars_b[2]), ph_o, a, abort);
          ph_o ^= 1u;
          tc_fence_after();
        }
        if (t + 1 < n_off) load_values_b(t + 1); else cp_commit();
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m_run + RAISE || (m_run == -INFINITY && mx != -INFINITY)) {
          const float m_new = mx;
          if (m_run != -INFINITY) {
            alpha = fast_exp2(m_run - m_new);
            rescale = o_started;
          }
          l_run *= alpha;
          m_run = m_new;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          const float f = rescale ? alpha : 1.f;
#pragma unroll 1
          for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
            float ov[32];
            tm_ld32(tm_row + TM_O + 32 * cb, ov);
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) ov[jj] *= f;
            tm_st32(tm_row + TM_O + 32 * cb, ov);
          }
        }
        {
          const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
          float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t wl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c0 = 8 * cc + 2 * e;
              const float p0 = fast_exp2(fmaf(x[c0], SCALE_LOG2, neg_m));
              const float p1 = fast_exp2(fmaf(x[c0 + 1], SCALE_LOG2, neg_m));
              l4[e] += p0 + p1;
              wl[e] = pack_half2(p0, p1);
            }
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(s0 + OFF_PL + swz(QT, rr, 32 * hf + 8 * cc)),
                         "r"(wl[0]), "r"(wl[1]), "r"(wl[2]), "r"(wl[3]) : "memory");
          }
          l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        }
        cp_wait_group<1>();  // this tile's values and the keys of tile t + 2
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == ISSUER) {
        uint32_t acc = o_started ? 1u : 0u;
        const uint64_t dpl = desc(s0 + OFF_PL, QT, 0), dv = desc(vbuf(t), D, 0);
#pragma unroll
        for (int ks = 0; ks < KT / 16; ++ks) {
          mma(tm + TM_O, dpl + koff(QT, ks), dv + koff(D, ks), idesc(D), acc);
          acc = 1u;
        }
        commit(smem_u32(&bars_b[2]));
        if (t + 2 < n_off) {
          issue_s_b(t + 2);
          commit(smem_u32(&bars_b[sb]));
        }
      }
      o_started = true;
    }
    if (ep && !*abort) {
      mma_wait(smem_u32(&bars_b[2]), ph_o, a, abort);
      tc_fence_after();
    }
  }
  cp_wait_group<0>();  // nothing may land in shared memory after the block exits

  // ---- O / l and the log-sum-exp of row i (the row's sum is the two halves')
  if (ep) s_red[hf][rr] = l_run;
  __syncthreads();
  if (ep) {
    l_run = s_red[0][rr] + s_red[1][rr];
    if (!*abort && o_started) {  // uniform: the tensor-memory loads take the whole warp
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      float *orow = a.o + (static_cast<int64_t>(bh) * a.cap + i) * D;
#pragma unroll
      for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
        float ov[32];
        tm_ld32(tm_row + TM_O + 32 * cb, ov);
        if (i < T)
#pragma unroll
          for (int jj = 0; jj < 32; jj += 4)
            *reinterpret_cast<float4 *>(orow + 32 * cb + jj) =
                make_float4(ov[jj] * inv, ov[jj + 1] * inv, ov[jj + 2] * inv, ov[jj + 3] * inv);
      }
      if (a.lse && i < T && hf == 0) a.lse[static_cast<int64_t>(bh) * a.cap + i] = (m_run + __log2f(l_run)) * LN2;
    } else if (o_started && i < T) {
      // a wait ran out: the row is undefined; leave a recognisable value
      if (a.lse) a.lse[static_cast<int64_t>(bh) * a.cap + i] = __int_as_float(0x7fc00000);
    } else if (!o_started && i < T) {
      if (a.lse) a.lse[static_cast<int64_t>(bh) * a.cap + i] = -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(TM_COLS));
}

// Workspace layout: Q^hi, Q^lo [B][Hq][cap][128], K^hi, K^lo [U][cap][128], V^t and
// Vt [U][cap/64][128][64], vertical-line Vt [U][ceil(vl_cap/64)][128][64]
// (fp16 each), every part 256-byte aligned.
struct WsLayout {
  size_t qh, ql, kh, kl, vqt, vft, vlt, total;
};
static WsLayout ws_layout(const hyq_cache *c) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t U = static_cast<size_t>(c->batch) * c->n_kv_heads, cap = c->capacity;
  const size_t row = D * 2;
  WsLayout w;
  w.qh = 0;
  w.ql = w.qh + up(static_cast<size_t>(c->batch) * c->n_q_heads * cap * row);
  w.kh = w.ql + up(static_cast<size_t>(c->batch) * c->n_q_heads * cap * row);
  w.kl = w.kh + up(U * cap * row);
  w.vqt = w.kl + up(U * cap * row);
  w.vft = w.vqt + up(U * cap * row);
  w.vlt = w.vft + up(U * cap * row);
  w.total = w.vlt + up(U * ((c->vl_capacity + KT - 1) / KT) * KT * row);
  return w;
}

}  // namespace pa
}  // namespace hyq

using namespace hyq;

extern "C" size_t hyq_prefill_attention_workspace(const hyq_cache *c) {
  if (hyq_check_cache(c) != HYQ_OK) return 0;
  return pa::ws_layout(c).total;
}

extern "C" hyq_status hyq_prefill_attention(const hyq_cache *c, const void *q, const void *k_full,
                                            const void *v_full, float *o, float *lse, void *ws,
                                            size_t ws_bytes, void *stream) {
  HYQ_RANGE("hyq_prefill_attention");
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!q || !k_full || !v_full || !o) return HYQ_ERR_INVALID;
  auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al16(q) || !al16(k_full) || !al16(v_full) || !al16(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      !al16(ws))
    return HYQ_ERR_ALIGN;
  const pa::WsLayout w = pa::ws_layout(c);
  if (!ws || ws_bytes < w.total) return HYQ_ERR_WORKSPACE;
  const int64_t U = static_cast<int64_t>(c->batch) * c->n_kv_heads;
  const int64_t n_bh = static_cast<int64_t>(c->batch) * c->n_q_heads;
  const int64_t n_qt = c->capacity / pa::QT;
  if (n_bh * n_qt > 0x7FFFFFFF || U * (c->capacity / pa::KT + (c->vl_capacity + pa::KT - 1) / pa::KT) > 0x7FFFFFFF)
    return HYQ_ERR_UNSUPPORTED;
  pa::Args a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.G = c->n_q_heads / c->n_kv_heads;
  a.cap = c->capacity; a.W = c->window; a.vl_cap = c->vl_capacity; a.U = static_cast<int>(U);
  a.q = static_cast<const __half *>(q);
  a.k = static_cast<const __half *>(k_full);
  a.v = static_cast<const __half *>(v_full);
  a.blocks = c->blocks;
  a.rm = RecMap{c->block_table, c->n_kv_heads, c->capacity, c->n_pages, c->dev_status};
  a.vl_k = static_cast<const __half *>(c->vl_k);
  a.vl_v = static_cast<const __half *>(c->vl_v);
  a.vl_pos = c->vl_pos; a.vl_count = c->vl_count; a.seq_len = c->seq_len;
  uint8_t *base = static_cast<uint8_t *>(ws);
  a.qh = reinterpret_cast<__half *>(base + w.qh);
  a.ql = reinterpret_cast<__half *>(base + w.ql);
  a.kh = reinterpret_cast<__half *>(base + w.kh);
  a.kl = reinterpret_cast<__half *>(base + w.kl);
  a.vqt = reinterpret_cast<__half *>(base + w.vqt);
  a.vft = reinterpret_cast<__half *>(base + w.vft);
  a.vlt = reinterpret_cast<__half *>(base + w.vlt);
  a.o = o; a.lse = lse; a.status = c->dev_status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n_q_rows = n_bh * c->capacity, n_rows = n_q_rows + U * c->capacity;
  cudaError_t e = launch(pa::pa_rows_kernel, dim3(static_cast<unsigned>((n_rows * 16 + 255) / 256)), dim3(256), 0,
                         st, a, n_q_rows, n_rows);
  if (e == cudaSuccess)
    e = launch(pa::pa_vt_kernel,
               dim3(static_cast<unsigned>(U * (c->capacity / pa::KT + (c->vl_capacity + pa::KT - 1) / pa::KT))),
               dim3(256), 0, st, a);
  if (e == cudaSuccess) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
      e = cudaFuncSetAttribute(pa::pa_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pa::SMEM_BYTES);
      if (e == cudaSuccess) configured_device = dev;
    }
  }
  if (e == cudaSuccess)
    e = launch(pa::pa_attn_kernel, dim3(static_cast<unsigned>(n_bh * n_qt)), dim3(pa::THREADS), pa::SMEM_BYTES, st,
               a);
  return e == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

// hyq_decode.cu -- one decode step of GQA attention over the hybrid INT4/FP16
// KV cache, with the INT4 dequantization fused into the attention.
//
// Method: HyQuant, aifromscratch.in explainer, "Two Operational Modes /
// Decode Stage": the cache is read in its 4-bit form and decompressed on the
// fly inside the attention computation (no FP16 copy is written back); the
// vertical-line tokens and the local window are read in FP16 ("How It
// Works", K_VL and K_Win).  The same kernel over an all-FP16 cache is the
// full-precision comparator.
//
// Design (B200, sm_100a)
//   * Work: per unit (batch, kv head) the positions are cut into tiles --
//     INT4 tiles of 32 tokens (one 5136-byte cache block record: K codes, K
//     scale/zero, V codes, V scale/zero, vertical-line bitmask) and FP16
//     tiles of 8 rows (vertical lines, then the window).  All tiles of all
//     units are concatenated and split over the launch's blocks by bytes
//     read (cost 5 per INT4 tile, 4 per FP16 tile), so any batch/length mix
//     fills every SM (split-KV, stream-K style).  With few long units the
//     split is aligned to units (whole blocks per unit).  The split is
//     planned before the wait on the previous launch and checked after it.
//   * One block per SM, 12 compute warps.  Block-local tile i belongs to
//     warp i % 12, which issues its own 1-D bulk copies (cp.async.bulk, no
//     multicast) into a private 2-slot ring with mbarrier transaction counts;
//     every wait is bounded by %globaltimer.
//   * Math: Q.K and P.V run on the tensor cores (mma.sync m16n8k16, fp16 in,
//     fp32 accumulate), tokens on the M side so a 16-token slice is one MMA
//     row block and the G <= 8 query heads of the unit fill N.  INT4 codes
//     enter the MMA as exact fp16 subnormals; the per-(token, group) scale is
//     applied in fp32 and both zero-point terms are one more MMA each:
//       s = sum_g scale_g * (q_g . code_g) + sum_g zero_g * sum(q_g)
//       o += sum_t (p_t * vscale_tg) * vcode_t + sum_t p_t * vzero_tg.
//     The softmax is fp32 online (running max / sum, exp2 domain), reduced
//     across lanes with warp shuffles; scores of skipped or padded tokens are
//     -inf.  Positions held in the vertical-line segment are skipped in the
//     INT4 sweep through the record's bitmask.
//   * Combine: the 12 warps of a block merge through shared memory; a block
//     that finishes a unit writes O directly; otherwise it writes its
//     (max, sum, acc) partial and the last block to finish the unit (atomic
//     tile counter) merges the partials by log-sum-exp.
//   * MODE_STEP (hyq_decode_step) fuses the append of the new token into the
//     same launch (see "fused step" below).
#include <cuda.h>  // driver types of the context query in hyq_decode_noalloc

#include <mutex>

#include "hyq_common.cuh"
#include "hyq_quant.cuh"

namespace hyq {

// Compute warps per block (one block per SM, each warp fed by itself): 16
// (at most 128 registers per thread) when the rings, the per-warp merge
// buffers of G heads and the per-unit tables fit in shared memory, else 12
// (168 registers).  The kernel is built for both; the host picks per launch.
constexpr int NCW_WIDE = 16, NCW_NARROW = 12;
constexpr int I4_TOK = 32;                // tokens per INT4 tile
constexpr int F16_ROWS = 8;               // rows per FP16 tile
constexpr int F16_ROW = D * 2;            // bytes of one FP16 K or V row
constexpr int SLOT_F16V = F16_ROWS * F16_ROW;  // V rows of an FP16 tile start here
// An INT4 tile is one quantized-majority block of the cache, copied whole.
constexpr int SLOT_KSZ = HYQ_BLK_KSZ;    // 2048
constexpr int SLOT_VC = HYQ_BLK_VCODES;  // 2560
constexpr int SLOT_VSZ = HYQ_BLK_VSZ;    // 4608
constexpr int SLOT_MASK = HYQ_BLK_MASK;  // 5120
constexpr int SLOT_BYTES = BLK_BYTES;    // 5136
constexpr int PART_STRIDE = 132;  // floats per (partial, head): m, l, -, -, acc[128]
constexpr float LOG2E_OVER_SQRT_D = 0.12751743082459868f;  // log2(e) / sqrt(128)
constexpr float TWO24 = 16777216.f, TWO20 = 1048576.f, TWO_M24 = 1.f / 16777216.f;
constexpr float LN2 = 0.69314718055994531f;

static_assert(2 * F16_ROWS * F16_ROW <= SLOT_MASK, "fp16 tile fits a slot");
// Split-KV balance: a block's share is measured in these tile costs (bytes
// read, in KiB: an INT4 tile moves 32 x 160 B, an FP16 tile 8 x 512 B).
constexpr int COST4 = 5, COST16 = 4;
static_assert(SLOT_BYTES % 16 == 0, "slots stay 16-byte aligned");
static_assert(I4_TOK == BLK_TOK, "an INT4 tile is one cache block");

// Ring slots per compute warp: 2 (one being read, one in flight), so one
// SM holds 24 or 32 tiles in flight (12 or 16 warps, about 120 or 160 KB),
// enough to cover the memory latency at full bandwidth while leaving shared
// memory for the merge buffers and per-unit tables (up to 4096 units with
// 12 warps).
#ifndef HYQ_DECODE_SPW
#define HYQ_DECODE_SPW 2
#endif
template <int G>
struct Ring {
  static constexpr int SPW = HYQ_DECODE_SPW;
};

// MODE_STEP: the hybrid decode with the token append of the same step fused
// in (hyq_decode_step): the cache is decoded as it is after the append.
// MODE_VLONLY: the vertical-only ablation (hyq_decode_vl_only): the same
// cache with its INT4 majority left out, i.e. attention over the vertical
// lines and the window alone.
enum { MODE_HYBRID = 0, MODE_FP16 = 1, MODE_STEP = 2, MODE_VLONLY = 3 };

// Debug builds (-DHYQ_DEBUG, built as libhyq_debug.so): the limit of the
// tile waits is a device variable the host may set (hyq_debug_set_wait), and
// a second one makes every warp's first tile wait a wait on a barrier that
// nothing completes, so that a test can make the bounded waits run out and
// check that the launch still returns, with HYQ_DEV_TIMEOUT; and the indexes
// the kernel derives (the block's share of the split, every tile's source
// rows, the partial records merged, the row leaving the window) are checked
// against the arrays they address: a failed check raises HYQ_DEV_OOB and the
// access is skipped.  Release builds compile all of it away.
#ifdef HYQ_DEBUG
__device__ unsigned long long g_debug_wait_ns = 2000000000ull;
__device__ int g_debug_stall = 0;
__device__ __forceinline__ uint64_t tile_wait_limit() {
  return *reinterpret_cast<volatile unsigned long long *>(&g_debug_wait_ns);
}
__device__ __forceinline__ bool dbg_check(bool ok, uint32_t *status) {
  if (!ok) set_status(status, HYQ_DEV_OOB);
  return ok;
}
#define DBG_OK(cond, status) dbg_check((cond), (status))
#else
__device__ __forceinline__ uint64_t tile_wait_limit() { return 2000000000ull; }
#define DBG_OK(cond, status) true
#endif

struct DecodeArgs {
  int B, Hq, Hkv, cap, W, vl_cap, U, n_ctas;
  uint8_t *blocks;        // quantized majority + bitmask, [U][cap/32][BLK_BYTES] or a page pool
  RecMap rm;              // record addresses (contiguous or through the block table)
  __half *win_k, *win_v;  // written only by the fused step
  const __half *vl_k, *vl_v;
  const int32_t *vl_count;
  int32_t *seq_len;       // written only by the fused step
  const __half *k16, *v16;  // comparator cache [B][Hkv][cap][128]
  const __half *q;
  __half *o;
  float *lse;
  float *part;        // [n_ctas][2][G][PART_STRIDE]
  int32_t *counters;  // [U]
  uint32_t *status;
  // fused step only: the new token's K/V rows [B][Hkv][128], the detector's
  // query ring [B][Hq][n_q][128] (nullable), and a block counter
  const __half *k_new, *v_new;
  __half *q_ring;
  int n_q;
  int32_t *grid_counter;
  // staging ring of the most recently quantized rows (stage_rows = 0: none)
  __half *stage_k, *stage_v;
  int stage_rows;
};

// Token order inside a 16-token MMA block: row r of the block holds token
// sig(r).  Flipping bit 0 when bit 2 is set keeps the two rows a lane pair
// reads in opposite 64-byte halves and spreads the V-code reads over banks.
__device__ __forceinline__ int sig(int r) { return r ^ ((r >> 2) & 1); }

struct UnitShape {
  int T, L4, vlc, nwin;  // positions; quantized prefix; VL rows; window rows
  int n4, nv, nw;        // tiles
};

template <int MODE>
__device__ __forceinline__ UnitShape shape_of(const DecodeArgs &a, int T, int vlc, bool &bad) {
  UnitShape s;
  s.T = T;
  bad = false;
  if (s.T < 0 || s.T > a.cap) {
    bad = true;
    s.T = 0;
  }
  if (MODE == MODE_FP16) {
    s.L4 = 0;
    s.vlc = 0;
    s.nwin = s.T;
    s.n4 = 0;
    s.nv = 0;
    s.nw = (s.T + F16_ROWS - 1) / F16_ROWS;
    return s;
  }
  s.L4 = s.T > a.W ? s.T - a.W : 0;
  s.vlc = vlc;
  if (s.vlc < 0 || s.vlc > a.vl_cap || s.vlc > s.L4) {
    bad = true;
    s.vlc = 0;
  }
  s.nwin = s.T < a.W ? s.T : a.W;
  s.n4 = (MODE == MODE_VLONLY) ? 0 : (s.L4 + I4_TOK - 1) / I4_TOK;
  s.nv = (s.vlc + F16_ROWS - 1) / F16_ROWS;
  s.nw = (s.nwin + F16_ROWS - 1) / F16_ROWS;
  return s;
}

// Shape of unit u from global state (prologue only; later reads use the
// per-unit (T, vl_count) copies kept in shared memory).
// (seq_len, vl_count) of unit u as stored.  L2-only loads: the first read
// may precede the wait on the previous launch, and no stale copy of it may
// stay in L1 for the re-read after it.
template <int MODE>
__device__ __forceinline__ int2 raw_lengths(const DecodeArgs &a, int u) {
  return make_int2(__ldcg(a.seq_len + u / a.Hkv), (MODE == MODE_FP16) ? 0 : __ldcg(a.vl_count + u));
}

template <int MODE>
__device__ __forceinline__ UnitShape shape_from_raw(const DecodeArgs &a, int2 raw, bool &bad) {
  int T = raw.x;
  if (MODE == MODE_STEP) T = (T < 0) ? -1 : T + 1;  // the length after the append
  return shape_of<MODE>(a, T, raw.y, bad);
}

template <int MODE>
__device__ __forceinline__ UnitShape unit_shape_global(const DecodeArgs &a, int u, bool &bad) {
  return shape_from_raw<MODE>(a, raw_lengths<MODE>(a, u), bad);
}

// Per-warp running state, in the accumulator layout of m16n8: lane (r, q)
// holds query heads 2q and 2q+1 of the unit (heads >= G are padding).
//
// INT4 codes enter the MMAs as fp16 subnormals (code_lo / code_hi), so
// while a warp sweeps INT4 tiles its accumulator rows carry power-of-two
// factors: rows r (elements 0, 1) hold 2^-24 O and rows r + 8 (elements 2,
// 3) hold 2^-20 O.  unscale_acc removes them before FP16 rows are added and
// before the state leaves the warp.
//
// The zero-point terms are MMAs too.  Keys: sum_g zero_g * qsum_g, with
// A = the token rows' four zeros (the same pair in every lane of a row) and
// B = qz, the per-group sums of q split into fp16 hi + lo parts (k rows 0-3
// and 8-11; the rest zero).  Values: zacc = Vzero^T P, groups on M (lane
// row r < 4 holds group r), heads on N.
struct WarpState {
  float m[2], l[2];
  float zacc[2];           // sum over tokens of p * vzero: group r, heads 2q, 2q+1
  float acc[NG][2][4];     // O^T accumulators: m-tile (group g, half j)
  uint32_t qf[NG][2][2];   // Q as the B operand: k-step (group g, piece s);
                           // piece [.][.][1] (high-nibble channels) is q / 16
  uint32_t qz[2];          // B operand of the key zero term
};

__device__ __forceinline__ void unscale_acc(WarpState &st) {
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      st.acc[g][j][0] *= TWO24;
      st.acc[g][j][1] *= TWO24;
      st.acc[g][j][2] *= TWO20;
      st.acc[g][j][3] *= TWO20;
    }
}

__device__ __forceinline__ void state_reset(WarpState &st) {
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    st.m[e] = -INFINITY;
    st.l[e] = 0.f;
    st.zacc[e] = 0.f;
  }
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[g][j][e] = 0.f;
}

// Query fragments of unit u.  Channel order inside a k-step matches the
// packed INT4 row: k-step (g, s) lane q carries channels
// 32g + 8q + 4s + {0, 2} (slots 2q, 2q+1) and {1, 3} (slots 2q+8, 2q+9).
// The odd channels meet high nibbles (16 x the code as a subnormal), so
// their q is stored divided by 16: exact for |q| >= 2^-10, and off by at
// most 2^-25 below that.
template <int G>
__device__ __forceinline__ void load_q(WarpState &st, const DecodeArgs &a, int u, int lane) {
  const int n = lane >> 2, q4 = lane & 3;
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  __half hi[NG], lo[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    uint4 x = make_uint4(0, 0, 0, 0);
    if (n < G)
      x = *reinterpret_cast<const uint4 *>(a.q + (static_cast<int64_t>(b) * a.Hq + kvh * G + n) * D +
                                           32 * g + 8 * q4);
    st.qf[g][0][0] = prmt(x.x, x.y, 0x5410u);
    st.qf[g][0][1] = prmt(x.x, x.y, 0x7632u);
    st.qf[g][1][0] = prmt(x.z, x.w, 0x5410u);
    st.qf[g][1][1] = prmt(x.z, x.w, 0x7632u);
    st.qf[g][0][1] = h2u(__hmul2(u2h(st.qf[g][0][1]), u2h(0x2C002C00u)));  // x 1/16
    st.qf[g][1][1] = h2u(__hmul2(u2h(st.qf[g][1][1]), u2h(0x2C002C00u)));
    float s = 0.f;
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __half22float2(h[i]);
      s += f.x + f.y;
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    // lanes 4n..4n+3 hold head n's group sum; keep it as hi + lo fp16
    // (relative error 2^-22)
    hi[g] = __float2half_rn(s);
    lo[g] = __float2half_rn(s - __half2float(hi[g]));
  }
  // B fragment rows k = 2q, 2q+1 (and 8 + 2q, 9 + 2q) of column n = head:
  // lane q = 0 carries the hi parts of groups (0, 1) / (2, 3), lane q = 1
  // the lo parts, lanes 2 and 3 zeros.
  st.qz[0] = (q4 == 0) ? h2u(__halves2half2(hi[0], hi[1])) : (q4 == 1) ? h2u(__halves2half2(lo[0], lo[1])) : 0u;
  st.qz[1] = (q4 == 0) ? h2u(__halves2half2(hi[2], hi[3])) : (q4 == 1) ? h2u(__halves2half2(lo[2], lo[3])) : 0u;
}

// Running-max update: when any lane sees a larger score for head 2q or
// 2q+1, the warp reduces the new maxima over its token rows and rescales the
// running sums and accumulators (exact max, so every p <= 1).
__device__ __forceinline__ void rescale_if_needed(WarpState &st, float mx0, float mx1) {
  const bool need = (mx0 > st.m[0]) || (mx1 > st.m[1]);
  if (__any_sync(0xffffffffu, need)) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float n0 = fmaxf(st.m[0], mx0), n1 = fmaxf(st.m[1], mx1);
    const float a0 = (n0 == -INFINITY) ? 1.f : fast_exp2(st.m[0] - n0);
    const float a1 = (n1 == -INFINITY) ? 1.f : fast_exp2(st.m[1] - n1);
    st.m[0] = n0;
    st.m[1] = n1;
    st.l[0] *= a0;
    st.l[1] *= a1;
    st.zacc[0] *= a0;
    st.zacc[1] *= a1;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        st.acc[g][j][0] *= a0;
        st.acc[g][j][1] *= a1;
        st.acc[g][j][2] *= a0;
        st.acc[g][j][3] *= a1;
      }
    }
  }
}

// Online softmax over the 4 scores a lane holds in one 16-token block:
// rows A (token sig(r)) and B (sig(r)+8), heads 2q and 2q+1.
__device__ __forceinline__ void softmax_step(WarpState &st, float (&S)[4], bool vA, bool vB,
                                             float (&p)[4]) {
  rescale_if_needed(st, fmaxf(S[0], S[2]), fmaxf(S[1], S[3]));
  p[0] = vA ? fast_exp2(S[0] - st.m[0]) : 0.f;
  p[1] = vA ? fast_exp2(S[1] - st.m[1]) : 0.f;
  p[2] = vB ? fast_exp2(S[2] - st.m[0]) : 0.f;
  p[3] = vB ? fast_exp2(S[3] - st.m[1]) : 0.f;
  st.l[0] += p[0] + p[2];
  st.l[1] += p[1] + p[3];
}

// One INT4 tile (up to 32 tokens) staged at `slot`, in three phases so the
// two 16-token MMA row blocks give independent work to overlap: Q.K of both
// blocks, one online-softmax update over the 32 tokens, then P.V.
// Invalid tokens (past the tile end, or held in the vertical-line segment)
// get S = -inf and p = 0.  Their codes and scale/zero rows come with the
// rest of the block record, which holds zeros or earlier quantizer output
// (the cache starts zero-filled), so p * scale and p * zero stay 0 without
// a select.
__device__ __forceinline__ void int4_tile(WarpState &st, uint32_t slot, int n_valid, uint32_t vlbits,
                                          int lane) {
  const int r = lane >> 2, q4 = lane & 3;
  const uint32_t kc = slot, ksz = slot + SLOT_KSZ, vc = slot + SLOT_VC, vsz = slot + SLOT_VSZ;
  const int s2q = sig(2 * q4), s2q1 = sig(2 * q4 + 1);
  const int nmt = (n_valid + 15) >> 4;
  constexpr int NMT = I4_TOK / 16;
  float S[NMT][4];
  bool vA[NMT], vB[NMT];

  // ---- phase 1: S = Q K^T per group on exact codes, per 16-token block
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    const int tA = 16 * mt + sig(r), tB = tA + 8;
    vA[mt] = tA < n_valid && !((vlbits >> tA) & 1u);
    vB[mt] = tB < n_valid && !((vlbits >> tB) & 1u);
#pragma unroll
    for (int e = 0; e < 4; ++e) S[mt][e] = 0.f;
    if (mt < nmt) {
      const uint4 ka = lds128(kc + tA * ROW_BYTES + 16 * q4);
      const uint4 kb = lds128(kc + tB * ROW_BYTES + 16 * q4);
      const uint4 za = lds128(ksz + tA * SZ_BYTES), zb = lds128(ksz + tB * SZ_BYTES);
      const uint32_t zaw[4] = {za.x, za.y, za.z, za.w}, zbw[4] = {zb.x, zb.y, zb.z, zb.w};
      // zero term: A row = (zero_0, zero_1 | zero_2, zero_3) of the row's token
      mma16816(S[mt], prmt(za.x, za.y, 0x7632u), prmt(zb.x, zb.y, 0x7632u), prmt(za.z, za.w, 0x7632u),
               prmt(zb.z, zb.w, 0x7632u), st.qz[0], st.qz[1]);
#pragma unroll
      for (int e = 0; e < 4; ++e) S[mt][e] *= TWO_M24;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const uint32_t w0a = (g < 2) ? ka.x : ka.y, w1a = (g < 2) ? ka.z : ka.w;
        const uint32_t w0b = (g < 2) ? kb.x : kb.y, w1b = (g < 2) ? kb.z : kb.w;
        const int sh = (g & 1) ? 8 : 0;
        float sg[4] = {0.f, 0.f, 0.f, 0.f};
        // sg = 2^-24 (q . code): low nibbles n 2^-24 against q, high
        // nibbles 16 n 2^-24 against q / 16
        mma16816(sg, code_lo(w0a >> sh), code_lo(w0b >> sh), code_hi(w0a >> sh), code_hi(w0b >> sh),
                 st.qf[g][0][0], st.qf[g][0][1]);
        mma16816(sg, code_lo(w1a >> sh), code_lo(w1b >> sh), code_hi(w1a >> sh), code_hi(w1b >> sh),
                 st.qf[g][1][0], st.qf[g][1][1]);
        const float sa = __low2float(u2h(zaw[g]));  // scales of rows A and B
        const float sb = __low2float(u2h(zbw[g]));
        S[mt][0] += sa * sg[0];
        S[mt][1] += sa * sg[1];
        S[mt][2] += sb * sg[2];
        S[mt][3] += sb * sg[3];
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) S[mt][e] *= LOG2E_OVER_SQRT_D * TWO24;
    if (!vA[mt]) S[mt][0] = S[mt][1] = -INFINITY;
    if (!vB[mt]) S[mt][2] = S[mt][3] = -INFINITY;
  }

  // ---- phase 2: one online-softmax update for the tile
  {
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt) {
      mx0 = fmaxf(mx0, fmaxf(S[mt][0], S[mt][2]));
      mx1 = fmaxf(mx1, fmaxf(S[mt][1], S[mt][3]));
    }
    rescale_if_needed(st, mx0, mx1);
  }
  float p[NMT][4];
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    p[mt][0] = vA[mt] ? fast_exp2(S[mt][0] - st.m[0]) : 0.f;
    p[mt][1] = vA[mt] ? fast_exp2(S[mt][1] - st.m[1]) : 0.f;
    p[mt][2] = vB[mt] ? fast_exp2(S[mt][2] - st.m[0]) : 0.f;
    p[mt][3] = vB[mt] ? fast_exp2(S[mt][3] - st.m[1]) : 0.f;
    st.l[0] += p[mt][0] + p[mt][2];
    st.l[1] += p[mt][1] + p[mt][3];
  }

  // ---- phase 3: O += P V, scale folded into P per group, zero separately
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    if (mt >= nmt) break;
    const int tA = 16 * mt + sig(r), tB = tA + 8;
    const uint4 wa = lds128(vsz + tA * SZ_BYTES), wb = lds128(vsz + tB * SZ_BYTES);
    const uint32_t waw[4] = {wa.x, wa.y, wa.z, wa.w}, wbw[4] = {wb.x, wb.y, wb.z, wb.w};
    // P of rows A and B as fp16 pairs (heads 2q, 2q+1), shared by the zero
    // term and, scaled per group, by the code MMAs
    const uint32_t pa2 = pack_half2(p[mt][0], p[mt][1]), pb2 = pack_half2(p[mt][2], p[mt][3]);
    {
      // zero term: A = Vzero^T (group r&3 of the tokens of k rows 2q, 2q+1,
      // 8 + 2q, 9 + 2q), B = P^T unscaled
      const uint32_t zrow = vsz + 4 * (r & 3);
      uint32_t z0, z1, z2, z3;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(z0) : "r"(zrow + (16 * mt + s2q) * SZ_BYTES));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(z1) : "r"(zrow + (16 * mt + s2q1) * SZ_BYTES));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(z2) : "r"(zrow + (16 * mt + s2q + 8) * SZ_BYTES));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(z3) : "r"(zrow + (16 * mt + s2q1 + 8) * SZ_BYTES));
      float z4[4] = {st.zacc[0], st.zacc[1], 0.f, 0.f};
      mma16816(z4, prmt(z0, z1, 0x7632u), 0u, prmt(z2, z3, 0x7632u), 0u, movmatrix_t(pa2), movmatrix_t(pb2));
      st.zacc[0] = z4[0];
      st.zacc[1] = z4[1];
    }
    // p * vscale in fp16 (one rounding of the fp16 p): the row's scale of
    // group g duplicated into both halves, one packed multiply per row
    uint32_t bq[NG][2];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const uint32_t sa2 = prmt(waw[g], 0u, 0x1010u), sb2 = prmt(wbw[g], 0u, 0x1010u);
      bq[g][0] = movmatrix_t(h2u(__hmul2(u2h(pa2), u2h(sa2))));
      bq[g][1] = movmatrix_t(h2u(__hmul2(u2h(pb2), u2h(sb2))));
    }
    // piece r of the position pairs (s2q, s2q1) and (s2q + 8, s2q1 + 8):
    // the records store each pair's words interleaved by 16 bits, so one
    // 16-byte load gives the A operands of both words (vcode_off)
    const int pr = (16 * mt + s2q) >> 1;  // pair index; the +8 pair is pr + 4 (same unit swizzle)
    const uint4 x = lds128(vc + pr * 128 + 16 * vcode_unit(pr, r));
    const uint4 y = lds128(vc + (pr + 4) * 128 + 16 * vcode_unit(pr, r));
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t xa = hh ? x.z : x.x, ya = hh ? x.w : x.y;
      const uint32_t xb = hh ? y.z : y.x, yb = hh ? y.w : y.y;
      const int g0 = 2 * hh, g1 = 2 * hh + 1;
      // rows r take low nibbles (2^-24 O), rows r + 8 high nibbles (2^-20 O)
      mma16816(st.acc[g0][0], code_lo(xa), code_hi(xa), code_lo(xb), code_hi(xb), bq[g0][0], bq[g0][1]);
      mma16816(st.acc[g0][1], code_lo(ya), code_hi(ya), code_lo(yb), code_hi(yb), bq[g0][0], bq[g0][1]);
      mma16816(st.acc[g1][0], code_lo(xa >> 8), code_hi(xa >> 8), code_lo(xb >> 8), code_hi(xb >> 8),
               bq[g1][0], bq[g1][1]);
      mma16816(st.acc[g1][1], code_lo(ya >> 8), code_hi(ya >> 8), code_lo(yb >> 8), code_hi(yb >> 8),
               bq[g1][0], bq[g1][1]);
    }
  }
}

// One FP16 tile (up to 8 rows) staged at `slot`: K rows [8][256 B], then V
// rows [8][256 B].  The MMA row block has 16 token rows; rows 8..15 are empty.
__device__ __forceinline__ void f16_tile(WarpState &st, uint32_t slot, int n_valid, int lane) {
  const int r = lane >> 2, q4 = lane & 3;
  const uint32_t kb_ = slot, vb_ = slot + SLOT_F16V;
  const int tA = sig(r);
  const bool vA = tA < n_valid;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint4 ka = lds128(kb_ + tA * F16_ROW + 64 * g + 16 * q4);
    // the odd channels' q is held divided by 16 (for the INT4 tiles)
    const uint32_t q01 = h2u(__hmul2(u2h(st.qf[g][0][1]), u2h(0x4C004C00u)));  // x 16
    const uint32_t q11 = h2u(__hmul2(u2h(st.qf[g][1][1]), u2h(0x4C004C00u)));
    mma16816(acc, prmt(ka.x, ka.y, 0x5410u), 0u, prmt(ka.x, ka.y, 0x7632u), 0u, st.qf[g][0][0], q01);
    mma16816(acc, prmt(ka.z, ka.w, 0x5410u), 0u, prmt(ka.z, ka.w, 0x7632u), 0u, st.qf[g][1][0], q11);
  }
  float S[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) S[e] = acc[e] * LOG2E_OVER_SQRT_D;
  if (!vA) S[0] = S[1] = -INFINITY;
  S[2] = S[3] = -INFINITY;
  float p[4];
  softmax_step(st, S, vA, false, p);
  const uint32_t b0 = movmatrix_t(pack_half2(p[0], p[1]));
  const int t0 = sig(2 * q4), t1 = sig(2 * q4 + 1);
  const bool v0 = t0 < n_valid, v1 = t1 < n_valid;
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint32_t off = vb_ + 64 * g + 8 * r;
    const uint2 z2 = make_uint2(0, 0);
    const uint2 A0 = v0 ? lds64(off + t0 * F16_ROW) : z2;
    const uint2 A1 = v1 ? lds64(off + t1 * F16_ROW) : z2;
    mma16816(st.acc[g][0], prmt(A0.x, A1.x, 0x5410u), prmt(A0.x, A1.x, 0x7632u), 0u, 0u, b0, 0u);
    mma16816(st.acc[g][1], prmt(A0.y, A1.y, 0x5410u), prmt(A0.y, A1.y, 0x7632u), 0u, 0u, b0, 0u);
  }
}

__host__ __device__ __forceinline__ int U_of(const DecodeArgs &a) { return a.U; }

struct Smem {
  uint32_t slots;     // shared address of slot 0: [NCW][SPW][SLOT_BYTES]
  uint64_t *full;     // [NCW][SPW] transaction barriers, one per slot
  int *abort_flag, *last_flag;
  uint64_t *never;    // a barrier nothing completes (the debug build's stall test)
  float *mm, *ml, *mo;  // merge buffers: [NCW][8], [NCW][8], [NCW][G][128]
  int *cost_start;      // [U + 1]: cost of the units before u
  int *scan;            // [NTHREADS]
  int *blk_start;       // [ALIGN_MAX_U + 1]: first block of each unit (aligned split)
  int *blk_lo;          // [ALIGN_MAX_CTAS + 1]: start cost of each block (aligned split)
  int2 *unit_tv;        // [U]: (T, vl_count) as read at launch
};

// Tiles of unit u: n4 INT4 tiles, then n16 FP16 tiles (vertical lines, window).
template <int MODE>
__device__ __forceinline__ void unit_tiles(const DecodeArgs &a, const Smem &sm, int u, int &n4, int &n16) {
  bool bad;
  const UnitShape s = shape_of<MODE>(a, sm.unit_tv[u].x, sm.unit_tv[u].y, bad);
  n4 = s.n4;
  n16 = s.nv + s.nw;
}

// First tile of a unit (cost start cs, n4 + n16 tiles) whose start cost is >= x.
// Costs are int32: the host rejects launches whose total cost reaches 2^31.
__device__ __forceinline__ int first_tile_from(int x, int cs, int n4, int n16) {
  const int rel = x - cs;
  if (rel <= 0) return 0;
  const int c4 = COST4 * n4;
  const int j = (rel <= c4) ? (rel + COST4 - 1) / COST4 : n4 + (rel - c4 + COST16 - 1) / COST16;
  return j < n4 + n16 ? j : n4 + n16;
}

// Start cost of tile j of a unit.
__device__ __forceinline__ int tile_cost(int cs, int n4, int j) {
  return j <= n4 ? cs + COST4 * j : cs + COST4 * n4 + COST16 * (j - n4);
}

// Split of the total cost over the launch's blocks.
//  * Contiguous: block c owns [lo(c), lo(c + 1)) with lo(c) = c * per +
//    min(c, rem), i.e. the first rem blocks take per + 1 and the others per;
//    a block may hold the end of one unit and the start of the next.
//  * Aligned (few long units): unit u owns the whole blocks [bs[u],
//    bs[u + 1]), bs[u] = round(n * cost_start[u] / total), and its cost is
//    spread evenly over them, so no block pays for two unit ends (two block
//    merges and two partial records).  Chosen only when every non-empty unit
//    gets a block and no block carries more than 9/8 of the mean cost; the
//    blocks' start costs are tabulated once per launch (sm.blk_lo).
constexpr int ALIGN_MAX_U = 32, ALIGN_MIN_BPU = 8, ALIGN_MAX_CTAS = 1024;
constexpr int BLK_TABLE_BYTES = ((ALIGN_MAX_U + 1) * 4 + 15) / 16 * 16 + ((ALIGN_MAX_CTAS + 1) * 4 + 15) / 16 * 16;

struct Split {
  int per, rem;
  bool aligned;
  __device__ __forceinline__ Split(int total, int n, bool al) : per(total / n), rem(total % n), aligned(al) {}
  __device__ __forceinline__ int lo(const Smem &sm, int U, int c) const {
    return aligned ? sm.blk_lo[c] : c * per + min(c, rem);
  }
  // the block whose (non-empty) range holds cost x, for 0 <= x < total
  __device__ __forceinline__ int of(const Smem &sm, int U, int x) const {
    if (!aligned) {
      const int big = rem * (per + 1);
      return x < big ? x / (per + 1) : rem + (x - big) / per;
    }
    int l = 0, h = sm.blk_start[U] - 1;  // last block c with blk_lo[c] <= x
    while (l < h) {
      const int mid = (l + h + 1) >> 1;
      if (sm.blk_lo[mid] <= x) l = mid; else h = mid - 1;
    }
    return l;
  }
};

// last unit u with cost_start[u] <= x
__device__ __forceinline__ int unit_of_cost(const int *cs, int U, int x) {
  int lo = 0, hi = U - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cs[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// A block's tiles of one unit: the segment [jb, je) of unit u, which holds
// block-local tile indices [base, base + je - jb).
struct Seg {
  int u, jb, je, base;
};

// Next non-empty segment of this block at or after unit u (u = U: none).
template <int MODE>
__device__ __forceinline__ Seg seg_from(const DecodeArgs &a, const Smem &sm, int u, int base, int lo, int hi) {
  Seg s{a.U, 0, 0, base};
  for (; u < a.U && sm.cost_start[u] < hi; ++u) {
    int n4, n16;
    unit_tiles<MODE>(a, sm, u, n4, n16);
    const int jb = first_tile_from(lo, sm.cost_start[u], n4, n16);
    const int je = first_tile_from(hi, sm.cost_start[u], n4, n16);
    if (jb < je) {
      s.u = u;
      s.jb = jb;
      s.je = je;
      return s;
    }
  }
  return s;
}

// Log-sum-exp combine of the NCW per-warp states in shared memory (sm.mm,
// sm.ml, sm.mo) for output element idx of [G][D]: returns the merged max,
// sum and unnormalized output.
template <int G, int NCW>
__device__ __forceinline__ void combine_warps(const Smem &sm, int idx, float &M, float &L, float &O) {
  const int h = idx / D, c = idx % D;
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NCW; ++w) M = fmaxf(M, sm.mm[w * 8 + h]);
  L = 0.f;
  O = 0.f;
#pragma unroll
  for (int w = 0; w < NCW; ++w) {
    const float mw = sm.mm[w * 8 + h];
    const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
    L += sm.ml[w * 8 + h] * f;
    O += sm.mo[(w * G + h) * D + c] * f;
  }
}

// Merge the partial records of unit u written by the blocks that share it
// (run by the last block to finish).  Warp w takes the records of candidate
// blocks c_lo + w, c_lo + w + NCW, ...; lane l holds channels 4l..4l+3 of
// every head.  A batch of RB records is loaded at once (one round trip to
// L2 per batch, most warps need one batch), merged online in registers, and
// the NCW warp states are then combined through shared memory like the
// warps of one block.
template <int G, int NCW>
__device__ __forceinline__ void merge_parts(const DecodeArgs &a, const Smem &sm, int u, int n4, int n16,
                                            const Split &sp, int64_t hbase, int tid) {
  constexpr int NTHREADS = NCW * 32;
  // records per batch (bounded by registers: 168 per thread at 12 warps, 128 at 16)
  constexpr int RB = (G >= 8) ? 1 : ((NCW > NCW_NARROW) ? 8 : 16) / G;
  const int warp = tid >> 5, lane = tid & 31;
  const int cs = sm.cost_start[u];
  const int c_lo = sp.of(sm, a.U, cs), c_hi = sp.of(sm, a.U, tile_cost(cs, n4, n4 + n16 - 1));
  float M[G], L[G];
  float4 acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    M[h] = -INFINITY;
    L[h] = 0.f;
    acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int c0 = c_lo + warp; c0 <= c_hi; c0 += RB * NCW) {
    float2 ml[RB][G];
    float4 x[RB][G];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      const int cc = c0 + b * NCW;
      int id = -1;  // record of block cc for unit u, if cc has tiles of u
      if (cc <= c_hi) {
        const int lo = sp.lo(sm, a.U, cc), hi = sp.lo(sm, a.U, cc + 1);
        if (first_tile_from(lo, cs, n4, n16) < first_tile_from(hi, cs, n4, n16)) id = cc * 2 + ((cs <= lo) ? 0 : 1);
        if (id >= 0 && !DBG_OK(id < 2 * a.n_ctas, lane == 0 ? a.status : nullptr)) id = -1;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        ml[b][h] = make_float2(-INFINITY, 0.f);
        x[b][h] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (id >= 0) {
          const float *pr = a.part + (static_cast<int64_t>(id) * G + h) * PART_STRIDE;
          ml[b][h] = __ldcg(reinterpret_cast<const float2 *>(pr));
          x[b][h] = __ldcg(reinterpret_cast<const float4 *>(pr + 4 + 4 * lane));
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float bm = M[h];
#pragma unroll
      for (int b = 0; b < RB; ++b) bm = fmaxf(bm, ml[b][h].x);
      if (bm == -INFINITY) continue;
      const float al = (M[h] == -INFINITY) ? 0.f : fast_exp2(M[h] - bm);
      float4 s4 = make_float4(acc[h].x * al, acc[h].y * al, acc[h].z * al, acc[h].w * al);
      float sl = L[h] * al;
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const float w = (ml[b][h].x == -INFINITY) ? 0.f : fast_exp2(ml[b][h].x - bm);
        sl += w * ml[b][h].y;
        s4.x += w * x[b][h].x;
        s4.y += w * x[b][h].y;
        s4.z += w * x[b][h].z;
        s4.w += w * x[b][h].w;
      }
      acc[h] = s4;
      M[h] = bm;
      L[h] = sl;
    }
  }
  // the block's own per-warp buffers are free again (the caller has passed
  // the barriers after its block merge)
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (lane == 0) {
      sm.mm[warp * 8 + h] = M[h];
      sm.ml[warp * 8 + h] = L[h];
    }
    *reinterpret_cast<float4 *>(sm.mo + (warp * G + h) * D + 4 * lane) = acc[h];
  }
  named_bar_sync(1, NTHREADS);
  for (int idx = tid; idx < G * D; idx += NTHREADS) {
    float Mx, Lx, Ox;
    combine_warps<G, NCW>(sm, idx, Mx, Lx, Ox);
    const int h = idx / D, c = idx % D;
    a.o[(hbase + h) * D + c] = __float2half_rn(Ox / Lx);
    if (c == 0 && a.lse) a.lse[hbase + h] = (Mx + __log2f(Lx)) * LN2;
  }
}

// ---------------------------------------------------------------- fused step
// The append of hyq_append done inside the decode of the same step, so that
// the result equals hyq_append followed by hyq_decode:
//  * the row at position T_old - W (the oldest window row, slot T_old % W)
//    is quantized by the warp that owns the unit's last INT4 tile; it
//    patches the tile in shared memory, writes the codes to the cache block
//    and then puts the new token into that window slot (every other reader
//    of the slot takes the new token from k_new / v_new);
//  * the warp that owns the window tile holding slot T_old % W patches that
//    row from k_new / v_new (and writes the slot when T_old < W, where no
//    row leaves the window);
//  * the query goes to ring slot T_old % n_q, rows spread over the blocks;
//  * seq_len = T_old + 1 is written, as it ends, by the last block to pass the prologue,
//    when every block has read the old lengths.
__device__ __forceinline__ void sts16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(static_cast<unsigned short>(v)) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Lanes 0-15 handle the K row, lanes 16-31 the V row (8 channels each).
__device__ __forceinline__ void step_exit_row(const DecodeArgs &a, int u, int T_old, uint32_t slot, int lane) {
  const int t = lane & 15;
  const bool is_v = lane >= 16;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int px = T_old - a.W;
  if (!DBG_OK(0 <= px && px < a.cap, lane == 0 ? a.status : nullptr)) return;
  __half *wrow = (is_v ? a.win_v : a.win_k) + (static_cast<int64_t>(u) * a.W + T_old % a.W) * D;
  const uint4 old = *reinterpret_cast<const uint4 *>(wrow + 8 * t);
  const QuantShare q = quantize_share(old, t, hmask, a.status);
  if (a.stage_rows > 0)  // the leaving row also enters the staging ring
    *reinterpret_cast<uint4 *>((is_v ? a.stage_v : a.stage_k) +
                               (static_cast<int64_t>(u) * a.stage_rows + px % a.stage_rows) * D + 8 * t) = old;
  const int row = px % I4_TOK;
  const uint32_t sz_s = slot + (is_v ? SLOT_VSZ : SLOT_KSZ) + row * SZ_BYTES;
  const int64_t rec = a.rm.rec(u, px);  // < 0: a bad block-table entry; the cache write is skipped
  uint32_t *sz_g = reinterpret_cast<uint32_t *>(a.blocks + (is_v ? rec_vsz(rec, px) : rec_ksz(rec, px)));
  if (q.has_codes && !is_v) {
    const uint32_t code_s = slot + row * ROW_BYTES;
    sts32(code_s + q.off0, q.w0);
    sts32(code_s + q.off1, q.w1);
    if (rec >= 0) {
      uint8_t *code_g = a.blocks + rec_kcode(rec, px);
      *reinterpret_cast<uint32_t *>(code_g + q.off0) = q.w0;
      *reinterpret_cast<uint32_t *>(code_g + q.off1) = q.w1;
    }
  }
  if (q.has_codes && is_v) {
    // V codes in position pairs: each word as its low and high 16 bits
    const int h = (q.off0 >> 2) & 1, p0 = q.off0 >> 3;
    const uint32_t oa = vcode_off(row, p0, h), ob = vcode_off(row, p0 + 1, h);
    sts16(slot + SLOT_VC + oa, q.w0 & 0xFFFFu);
    sts16(slot + SLOT_VC + oa + 4, q.w0 >> 16);
    sts16(slot + SLOT_VC + ob, q.w1 & 0xFFFFu);
    sts16(slot + SLOT_VC + ob + 4, q.w1 >> 16);
    if (rec >= 0) store_vcodes(q, a.blocks + rec_vcodes(rec), row);
  }
  if (q.has_sz) {
    sts32(sz_s + 4 * q.g, q.sz);
    if (rec >= 0) sz_g[q.g] = q.sz;
  }
  if (row == 0 && lane == 0) {
    // the first row quantized into this record: none of its positions is a
    // vertical line yet (they lie below T - W), so its bitmask starts clear
    // -- in the cache and in the staged copy of the tile -- whatever the
    // record held before
    sts32(slot + SLOT_MASK, 0u);
    if (rec >= 0) *reinterpret_cast<uint32_t *>(a.blocks + rec_mask(rec)) = 0u;
  }
  // the old row has been read (its value is consumed above): the new token
  // takes its slot
  const __half *nrow = (is_v ? a.v_new : a.k_new) + static_cast<int64_t>(u) * D;
  *reinterpret_cast<uint4 *>(wrow + 8 * t) = *reinterpret_cast<const uint4 *>(nrow + 8 * t);
  __syncwarp();
}

__device__ __forceinline__ void step_new_row(const DecodeArgs &a, int u, int s_new, int row, bool write_slot,
                                             uint32_t slot, int lane) {
  const int t = lane & 15;
  const bool is_v = lane >= 16;
  const uint4 x = *reinterpret_cast<const uint4 *>((is_v ? a.v_new : a.k_new) + static_cast<int64_t>(u) * D + 8 * t);
  sts128(slot + (is_v ? SLOT_F16V : 0) + row * F16_ROW + 16 * t, x);
  if (write_slot)
    *reinterpret_cast<uint4 *>((is_v ? a.win_v : a.win_k) + (static_cast<int64_t>(u) * a.W + s_new) * D + 8 * t) = x;
  __syncwarp();
}

// After the prologue (unit lengths in shared memory are T_old + 1).  Thread
// 0 counts the block in once every thread has read the lengths; the count
// it gets back is only looked at when the block ends (step_epilogue), so the
// round trip of the atomic overlaps the block's tiles.
template <int NTHREADS>
__device__ __forceinline__ int step_prologue(const DecodeArgs &a, const Smem &sm, int tid) {
  if (a.q_ring) {
    const int64_t items = static_cast<int64_t>(a.B) * a.Hq * 16;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * NTHREADS + tid; i < items;
         i += static_cast<int64_t>(a.n_ctas) * NTHREADS) {
      const int64_t row = i >> 4;  // b * Hq + query head
      const int part = static_cast<int>(i & 15), b = static_cast<int>(row / a.Hq);
      const int T = sm.unit_tv[b * a.Hkv].x;  // T_old + 1
      if (T < 1 || T > a.cap) continue;
      *reinterpret_cast<uint4 *>(a.q_ring + (row * a.n_q + (T - 1) % a.n_q) * D + 8 * part) =
          *reinterpret_cast<const uint4 *>(a.q + row * D + 8 * part);
    }
  }
  return (tid == 0) ? atomicAdd(a.grid_counter, 1) : -1;
}

// The block that was counted in last writes seq_len = T_old + 1: by then
// every block has read the old lengths.  (The next launch on the stream
// reads them only after this grid has completed.)
__device__ __forceinline__ void step_epilogue(const DecodeArgs &a, const Smem &sm, int tid, int arrived) {
  if (tid == 0 && arrived == a.n_ctas - 1) {
    for (int b = 0; b < a.B; ++b) {
      const int T = sm.unit_tv[b * a.Hkv].x;
      if (T >= 1 && T <= a.cap) a.seq_len[b] = T;
    }
    *a.grid_counter = 0;
  }
}

// Global source of tile j of unit u: one run (an INT4 block record) or two
// runs of `bytes` each (the K rows and the V rows of an FP16 tile).
struct TileSrc {
  const void *k, *v;
  uint32_t bytes;
};

template <int MODE>
__device__ __forceinline__ TileSrc tile_src(const DecodeArgs &a, const Smem &sm, int u, int j) {
  bool bad;
  const UnitShape us = shape_of<MODE>(a, sm.unit_tv[u].x, sm.unit_tv[u].y, bad);
  if (MODE != MODE_FP16 && j < us.n4)
    return {a.blocks + a.rm.rec_rd(u, static_cast<int64_t>(j) * I4_TOK), nullptr, BLK_BYTES};
  const __half *sk, *sv;
  int n;
  if (MODE == MODE_FP16) {
    const int r0 = j * F16_ROWS;
    n = min(F16_ROWS, us.T - r0);
    const int64_t base = (static_cast<int64_t>(u) * a.cap + r0) * D;
    sk = a.k16 + base;
    sv = a.v16 + base;
  } else if (j < us.n4 + us.nv) {
    const int r0 = (j - us.n4) * F16_ROWS;
    n = min(F16_ROWS, us.vlc - r0);
    const int64_t base = (static_cast<int64_t>(u) * a.vl_cap + r0) * D;
    sk = a.vl_k + base;
    sv = a.vl_v + base;
  } else {
    const int r0 = (j - us.n4 - us.nv) * F16_ROWS;
    n = min(F16_ROWS, us.nwin - r0);
    const int64_t base = (static_cast<int64_t>(u) * a.W + r0) * D;
    sk = a.win_k + base;
    sv = a.win_v + base;
  }
  return {sk, sv, static_cast<uint32_t>(n * F16_ROW)};
}

// Whether tile j of unit u addresses rows inside the cache's arrays: a
// quantized block below capacity, vertical-line rows below vl_capacity,
// window rows below the window, comparator rows below capacity.
template <int MODE>
__device__ __forceinline__ bool tile_in_bounds(const DecodeArgs &a, const Smem &sm, int u, int j) {
  if (u < 0 || u >= a.U || j < 0) return false;
  bool bad;
  const UnitShape us = shape_of<MODE>(a, sm.unit_tv[u].x, sm.unit_tv[u].y, bad);
  if (MODE == MODE_FP16) return j < us.nw && j * F16_ROWS < us.T && us.T <= a.cap;
  if (j < us.n4) return (j + 1) * I4_TOK <= a.cap;
  if (j < us.n4 + us.nv) {
    const int r0 = (j - us.n4) * F16_ROWS;
    return r0 < us.vlc && min(r0 + F16_ROWS, us.vlc) <= a.vl_cap;
  }
  const int r0 = (j - us.n4 - us.nv) * F16_ROWS;
  return j < us.n4 + us.nv + us.nw && r0 < us.nwin && min(r0 + F16_ROWS, us.nwin) <= a.W;
}

// Issue the bulk copies of tile j of unit u into one ring slot (lane 0 arms
// the barrier and copies; an FP16 tile is two contiguous runs of rows).
template <int MODE>
__device__ __forceinline__ void issue_tile(const DecodeArgs &a, const Smem &sm, int u, int j, uint32_t dst,
                                           uint32_t bar, int lane) {
  if (lane != 0) return;
  if (!DBG_OK(tile_in_bounds<MODE>(a, sm, u, j), a.status)) {
    mbar_arrive(bar);  // the slot's phase completes with no copy
    return;
  }
  const TileSrc t = tile_src<MODE>(a, sm, u, j);
  if (t.v == nullptr) {
    mbar_arrive_expect_tx(bar, t.bytes);
    bulk_g2s(dst, t.k, t.bytes, bar);
    return;
  }
  mbar_arrive_expect_tx(bar, 2 * t.bytes);
  bulk_g2s(dst, t.k, t.bytes, bar);
  bulk_g2s(dst + SLOT_F16V, t.v, t.bytes, bar);
}

// Read every unit's (T, vl_count) from global memory into shared memory and
// build the cost prefix sm.cost_start (and, for few units, the aligned
// split's block table).  Returns whether the split is aligned (the same in
// every thread).  Status bits for malformed lengths are raised only when
// `report` is set.
template <int MODE, int NTHREADS>
__device__ __forceinline__ bool plan_units(const DecodeArgs &a, const Smem &sm, int tid, bool report) {
  const int U = a.U, warp = tid >> 5, lane = tid & 31;
  const int per = (U + NTHREADS - 1) / NTHREADS;
  const int beg = min(U, tid * per), end = min(U, beg + per);
  int local = 0;
  for (int u = beg; u < end; ++u) {
    bool bad;
    const UnitShape s = unit_shape_global<MODE>(a, u, bad);
    sm.unit_tv[u] = make_int2(s.T, s.vlc);
    local += COST4 * s.n4 + COST16 * (s.nv + s.nw);
    if (report && bad && (u % a.n_ctas) == static_cast<int>(blockIdx.x)) set_status(a.status, HYQ_DEV_BADLEN);
  }
  int v = local;  // block exclusive scan of `local`
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += y;
  }
  if (lane == 31) sm.scan[warp] = v;
  __syncthreads();
  int wpre = 0;
  for (int w = 0; w < warp; ++w) wpre += sm.scan[w];
  int acc = wpre + v - local;
  for (int u = beg; u < end; ++u) {
    int n4, n16;
    unit_tiles<MODE>(a, sm, u, n4, n16);
    sm.cost_start[u] = acc;
    acc += COST4 * n4 + COST16 * n16;
  }
  if (tid == NTHREADS - 1) sm.cost_start[U] = acc;
  __syncthreads();
  const int n = a.n_ctas;
  if (U > ALIGN_MAX_U || U * ALIGN_MIN_BPU > n || n > ALIGN_MAX_CTAS) return false;
  const int total = sm.cost_start[U];
  if (total <= 0) return false;
  if (tid <= U)
    sm.blk_start[tid] = static_cast<int>((2 * static_cast<int64_t>(n) * sm.cost_start[tid] + total) /
                                         (2 * static_cast<int64_t>(total)));
  __syncthreads();
  int unfit = 0;
  if (tid < U) {
    const int C = sm.cost_start[tid + 1] - sm.cost_start[tid], k = sm.blk_start[tid + 1] - sm.blk_start[tid];
    unfit = C > 0 && (k == 0 || static_cast<int64_t>(C) * n * 8 > static_cast<int64_t>(total) * k * 9);
  }
  if (__syncthreads_or(unfit)) return false;
  // block c of unit u (k blocks, cost C) starts at cost_start[u] + floor(j C / k),
  // j = c - blk_start[u], evaluated exactly in 32 bits as j (C / k) + j (C % k) / k
  for (int c = tid; c <= n; c += NTHREADS) {
    int v = total;
    if (c < n) {
      int l = 0, h = U - 1;  // last unit whose first block is <= c (a non-empty one)
      while (l < h) {
        const int mid = (l + h + 1) >> 1;
        if (sm.blk_start[mid] <= c) l = mid; else h = mid - 1;
      }
      const int k = sm.blk_start[l + 1] - sm.blk_start[l], C = sm.cost_start[l + 1] - sm.cost_start[l];
      const int j = c - sm.blk_start[l];
      v = sm.cost_start[l] + j * (C / k) + j * (C % k) / k;
    }
    sm.blk_lo[c] = v;
  }
  __syncthreads();
  return true;
}

// After the wait on the previous launch: true (in every thread) when some
// unit's (T, vl_count) differs from the plan built before the wait.  Raises
// the status bits of malformed lengths.  `first` holds the raw lengths of
// the thread's first unit, read by first_lengths before the first copies
// were issued (so that read does not queue behind them).
template <int MODE, int NTHREADS>
__device__ __forceinline__ int2 first_lengths(const DecodeArgs &a, int tid) {
  const int per = (a.U + NTHREADS - 1) / NTHREADS, beg = tid * per;
  return beg < a.U ? raw_lengths<MODE>(a, beg) : make_int2(0, 0);
}

template <int MODE, int NTHREADS>
__device__ __forceinline__ bool plan_stale(const DecodeArgs &a, const Smem &sm, int tid, int2 first) {
  const int U = a.U;
  const int per = (U + NTHREADS - 1) / NTHREADS;
  const int beg = min(U, tid * per), end = min(U, beg + per);
  int changed = 0;
  for (int u = beg; u < end; ++u) {
    bool bad;
    const UnitShape s = shape_from_raw<MODE>(a, u == beg ? first : raw_lengths<MODE>(a, u), bad);
    if (s.T != sm.unit_tv[u].x || s.vlc != sm.unit_tv[u].y) changed = 1;
    if (bad && (u % a.n_ctas) == static_cast<int>(blockIdx.x)) set_status(a.status, HYQ_DEV_BADLEN);
  }
  return __syncthreads_or(changed) != 0;
}

template <int G, int MODE, int NCW>
__global__ void __launch_bounds__(NCW * 32, 1) decode_kernel(const DecodeArgs a) {
  constexpr int SPW = Ring<G>::SPW;
  constexpr int NTHREADS = NCW * 32;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Smem sm;
  {
    uint8_t *p = smem_raw;
    sm.slots = smem_u32(p);
    p += NCW * SPW * SLOT_BYTES;
    sm.full = reinterpret_cast<uint64_t *>(p);
    p += NCW * SPW * 8;
    sm.abort_flag = reinterpret_cast<int *>(p);
    sm.last_flag = sm.abort_flag + 1;
    sm.never = reinterpret_cast<uint64_t *>(sm.abort_flag + 2);  // debug builds only
    p += 16;
    sm.mm = reinterpret_cast<float *>(p);
    p += NCW * 8 * 4;
    sm.ml = reinterpret_cast<float *>(p);
    p += NCW * 8 * 4;
    sm.mo = reinterpret_cast<float *>(p);
    p += NCW * G * D * 4;
    sm.scan = reinterpret_cast<int *>(p);
    p += NTHREADS * 4;
    sm.blk_start = reinterpret_cast<int *>(p);
    sm.blk_lo = sm.blk_start + ((ALIGN_MAX_U + 1) * 4 + 15) / 16 * 4;
    p += BLK_TABLE_BYTES;
    sm.cost_start = reinterpret_cast<int *>(p);
    p += ((U_of(a) + 1) * 4 + 15) / 16 * 16;
    sm.unit_tv = reinterpret_cast<int2 *>(p);
  }
  const int U = a.U;
  pdl_trigger();  // the next kernel may be scheduled
  if (tid == 0) {
    *sm.abort_flag = 0;
    for (int s = 0; s < NCW * SPW; ++s) mbar_init(smem_u32(&sm.full[s]), 1);
#ifdef HYQ_DEBUG
    mbar_init(smem_u32(sm.never), 1);
#endif
    fence_barrier_init();
  }
  // Plan from the lengths as they stand, which the previous launch on the
  // stream may still be changing: the plan is made while that launch drains
  // and only checked after the wait.
  bool aligned = plan_units<MODE, NTHREADS>(a, sm, tid, false);
  pdl_wait();  // earlier work on the stream (an append) is complete and visible

  const int cta = blockIdx.x;
  Split sp(sm.cost_start[U], a.n_ctas, aligned);
  int lo = sp.lo(sm, U, cta), hi = sp.lo(sm, U, cta + 1);
  if (!DBG_OK(0 <= lo && lo <= hi && hi <= sm.cost_start[U], tid == 0 ? a.status : nullptr)) lo = hi = 0;
  volatile int *abort_flag = sm.abort_flag;
  int u_first = (lo < hi) ? unit_of_cost(sm.cost_start, U, lo) : U;

  // This warp's tiles are the block-local tiles warp, warp + NCW, ...; its
  // k-th tile lives in ring slot k % SPW.  The warp issues its own copies:
  // SPW tiles ahead at the start, then tile k + SPW once tile k is read.
  const uint32_t my_slots = sm.slots + warp * SPW * SLOT_BYTES;
  const uint32_t my_bars = smem_u32(&sm.full[warp * SPW]);
  int k_issued = 0, k_done = 0, first_fail = -1;
  int k_skip = 0;  // copies drained unused (a stale plan): not tiles of this plan
  Seg ic = seg_from<MODE>(a, sm, u_first, 0, lo, hi);  // issue cursor
  auto issue_next = [&]() {
    const int i = warp + NCW * (k_issued - k_skip);  // block-local tile index
    while (ic.u < U && i >= ic.base + ic.je - ic.jb)
      ic = seg_from<MODE>(a, sm, ic.u + 1, ic.base + ic.je - ic.jb, lo, hi);
    const int stop = __shfl_sync(0xffffffffu, *abort_flag, 0);  // one decision per warp
    if (ic.u >= U || stop) return;
    const int sl = k_issued % SPW;
    issue_tile<MODE>(a, sm, ic.u, ic.jb + (i - ic.base), my_slots + sl * SLOT_BYTES, my_bars + sl * 8, lane);
    __syncwarp();
    ++k_issued;
  };
  // The first copies follow the plan made before the wait; the lengths are
  // read again meanwhile (loads issued ahead of the copies).  If they changed
  // (the previous launch appended to this cache), those copies land unused
  // and the block plans again.
  const int2 first = first_lengths<MODE, NTHREADS>(a, tid);
  for (int k = 0; k < SPW; ++k) issue_next();
  if (plan_stale<MODE, NTHREADS>(a, sm, tid, first)) {
    for (; k_done < k_issued; ++k_done) {
      const bool ok = first_fail < 0 &&
                      mbar_wait_bounded(my_bars + (k_done % SPW) * 8, (k_done / SPW) & 1, abort_flag, a.status,
                                        tile_wait_limit());
      if (!__all_sync(0xffffffffu, ok) && first_fail < 0) first_fail = k_done;
    }
    aligned = plan_units<MODE, NTHREADS>(a, sm, tid, false);
    sp = Split(sm.cost_start[U], a.n_ctas, aligned);
    lo = sp.lo(sm, U, cta);
    hi = sp.lo(sm, U, cta + 1);
    if (!DBG_OK(0 <= lo && lo <= hi && hi <= sm.cost_start[U], tid == 0 ? a.status : nullptr)) lo = hi = 0;
    u_first = (lo < hi) ? unit_of_cost(sm.cost_start, U, lo) : U;
    k_skip = k_issued;
    ic = seg_from<MODE>(a, sm, u_first, 0, lo, hi);
    for (int k = 0; k < SPW; ++k) issue_next();
  }
  const int arrived = (MODE == MODE_STEP) ? step_prologue<NTHREADS>(a, sm, tid) : -1;

  WarpState st;
  for (Seg sg = seg_from<MODE>(a, sm, u_first, 0, lo, hi); sg.u < U;
       sg = seg_from<MODE>(a, sm, sg.u + 1, sg.base + sg.je - sg.jb, lo, hi)) {
    const int u = sg.u;
    bool bad;
    const UnitShape us = shape_of<MODE>(a, sm.unit_tv[u].x, sm.unit_tv[u].y, bad);
    const int n_unit = us.n4 + us.nv + us.nw;
    state_reset(st);
    load_q<G>(st, a, u, lane);
    // my tiles inside this segment: block-local i = base .. base + je - jb - 1
    int i = sg.base + (warp - sg.base % NCW + NCW) % NCW;
    bool scaled = false;  // acc holds the INT4 sweep's power-of-two factors
    for (; i < sg.base + sg.je - sg.jb; i += NCW) {
      const int kk = k_done;
      const int sl = kk % SPW;
      const uint32_t slot = my_slots + sl * SLOT_BYTES;
      ++k_done;
      uint32_t wait_bar = my_bars + sl * 8, wait_parity = (kk / SPW) & 1;
#ifdef HYQ_DEBUG
      if (kk == k_skip && *reinterpret_cast<volatile int *>(&g_debug_stall)) {
        wait_bar = smem_u32(sm.never);  // the stall test: a phase that never completes
        wait_parity = 0;
      }
#endif
      bool landed = first_fail < 0 &&
                    mbar_wait_bounded(wait_bar, wait_parity, abort_flag, a.status, tile_wait_limit());
      landed = __all_sync(0xffffffffu, landed);  // the warp computes together or not at all
      if (!landed) {
        if (first_fail < 0) first_fail = kk;
        continue;
      }
      const int j = sg.jb + (i - sg.base);
      if (MODE != MODE_FP16 && j < us.n4) {
        const int t0 = j * I4_TOK;
        const int n = min(I4_TOK, us.L4 - t0);
        // fused step: the row leaving the window is the unit's last INT4 position
        if (MODE == MODE_STEP && j == us.n4 - 1 && us.T > a.W) step_exit_row(a, u, us.T - 1, slot, lane);
        uint32_t bits;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bits) : "r"(slot + SLOT_MASK));
        int4_tile(st, slot, n, bits, lane);
        scaled = true;
      } else {
        if (scaled) unscale_acc(st);
        scaled = false;
        int n;
        if (MODE == MODE_FP16)
          n = min(F16_ROWS, us.T - j * F16_ROWS);
        else if (j < us.n4 + us.nv)
          n = min(F16_ROWS, us.vlc - (j - us.n4) * F16_ROWS);
        else
          n = min(F16_ROWS, us.nwin - (j - us.n4 - us.nv) * F16_ROWS);
        if (MODE == MODE_STEP && j >= us.n4 + us.nv) {
          // fused step: the new token's window row
          const int r0 = (j - us.n4 - us.nv) * F16_ROWS, s_new = (us.T - 1) % a.W;
          if (s_new >= r0 && s_new < r0 + n) step_new_row(a, u, s_new, s_new - r0, us.T - 1 < a.W, slot, lane);
        }
        f16_tile(st, slot, n, lane);
      }
      // the slot has been read: order those reads before the next bulk copy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      issue_next();
    }

    // ---- segment end: reduce the warp's state over token rows
    if (scaled) unscale_acc(st);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 2; ++e) st.l[e] += __shfl_xor_sync(0xffffffffu, st.l[e], off);
    }
    const int r = lane >> 2, q4 = lane & 3;
    float zs[2][NG];  // value zero term of heads 2q, 2q+1: held by lane (g, q)
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int e = 0; e < 2; ++e) zs[e][g] = __shfl_sync(0xffffffffu, st.zacc[e], 4 * g + q4);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * q4 + e;
      if (h < G) {
        if (r == 0) {
          sm.mm[warp * 8 + h] = st.m[e];
          sm.ml[warp * 8 + h] = st.l[e];
        }
        float *orow = sm.mo + (warp * G + h) * D;
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int ch = 32 * g + 4 * r + 2 * j;
            orow[ch] = st.acc[g][j][e] + zs[e][g];
            orow[ch + 1] = st.acc[g][j][2 + e] + zs[e][g];
          }
      }
    }
    named_bar_sync(1, NTHREADS);

    // ---- merge the warps of the block
    const bool complete = (sg.jb == 0) && (sg.je == n_unit);
    const int slot_id = (sm.cost_start[u] <= lo) ? 0 : 1;  // 1: the unit began after this block's start
    const int b = u / a.Hkv, kvh = u % a.Hkv;
    const int64_t hbase = static_cast<int64_t>(b) * a.Hq + kvh * G;
    for (int idx = tid; idx < G * D; idx += NTHREADS) {
      const int h = idx / D, c = idx % D;
      float M, L, O;
      combine_warps<G, NCW>(sm, idx, M, L, O);
      if (complete) {
        a.o[(hbase + h) * D + c] = __float2half_rn(O / L);
        if (c == 0 && a.lse) a.lse[hbase + h] = (M + __log2f(L)) * LN2;
      } else {
        float *pr = a.part + (static_cast<int64_t>(cta * 2 + slot_id) * G + h) * PART_STRIDE;
        if (c == 0) {
          pr[0] = M;
          pr[1] = L;
        }
        pr[4 + c] = O;
      }
    }
    if (!complete) {
      // Publish the partial: after the block barrier, one acquire-release
      // atomic by thread 0 orders the block's record writes (observed
      // through the barrier) before the count, and, in the block that
      // completes the unit, the other blocks' records before the merge
      // (the barrier after it passes the acquire on to every thread).
      named_bar_sync(1, NTHREADS);
      if (tid == 0) {
        const int mine = sg.je - sg.jb;
        int old;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
                     : "=r"(old)
                     : "l"(a.counters + u), "r"(mine)
                     : "memory");
        *sm.last_flag = (old + mine == n_unit);
      }
      named_bar_sync(1, NTHREADS);
      if (*sm.last_flag) {
        merge_parts<G, NCW>(a, sm, u, us.n4, us.nv + us.nw, sp, hbase, tid);
        if (tid == 0) a.counters[u] = 0;
      }
    }
    named_bar_sync(1, NTHREADS);
  }

  // copies still in flight (only after an abort): let them land before exit
  for (int kk = (first_fail >= 0 ? first_fail : k_done); kk < k_issued; ++kk)
    mbar_drain(my_bars + (kk % SPW) * 8, (kk / SPW) & 1, 500000000ull);
  if (MODE == MODE_STEP) step_epilogue(a, sm, tid, arrived);

  // units without any position: o = 0, lse = -inf (one block each)
  for (int u = cta; u < U; u += a.n_ctas) {
    if (sm.cost_start[u] != sm.cost_start[u + 1]) continue;
    const int b = u / a.Hkv, kvh = u % a.Hkv;
    const int64_t hbase = static_cast<int64_t>(b) * a.Hq + kvh * G;
    for (int idx = tid; idx < G * D; idx += NTHREADS) {
      a.o[(hbase + idx / D) * D + idx % D] = __float2half_rn(0.f);
      if (idx % D == 0 && a.lse) a.lse[hbase + idx / D] = -INFINITY;
    }
  }
}

// ---------------------------------------------------------------- host side
constexpr size_t DECODE_SMEM_MAX = 227 * 1024;

static size_t decode_smem_bytes(int G, int U, int ncw) {
  const int spw = Ring<1>::SPW;
  static_assert(Ring<1>::SPW == Ring<8>::SPW, "one ring depth for every G");
  return static_cast<size_t>(ncw) * spw * SLOT_BYTES + ncw * spw * 8 + 16 + ncw * 8 * 4 * 2 +
         static_cast<size_t>(ncw) * G * D * 4 + ncw * 32 * 4 + BLK_TABLE_BYTES +
         (static_cast<size_t>(U + 1) * 4 + 15) / 16 * 16 +
         static_cast<size_t>(U) * 8;
}

// 16 compute warps for launches with many tiles per block (at least
// WIDE_MIN_TILES quantized-tile slots of capacity per block: batched or long
// contexts, where the INT4 tile arithmetic sets the pace and more warps hide
// its latency), when their shared memory fits (G <= 4 and, at G = 4, up to
// about 2300 units); 12 otherwise (few tiles per warp, where the block's
// fixed costs set the pace and 168 registers per thread serve better).
constexpr int64_t WIDE_MIN_TILES = 128;
static int decode_ncw(int G, int U, int cap, int n_ctas) {
  if (G >= 8 || decode_smem_bytes(G, U, NCW_WIDE) > DECODE_SMEM_MAX) return NCW_NARROW;
  return static_cast<int64_t>(U) * (cap / I4_TOK) >= WIDE_MIN_TILES * n_ctas ? NCW_WIDE : NCW_NARROW;
}

static size_t decode_ws_bytes(int G, int U, int n_ctas) {
  const size_t cnt = (static_cast<size_t>(U) * 4 + 255) / 256 * 256;
  return cnt + static_cast<size_t>(n_ctas) * 2 * G * PART_STRIDE * 4;
}

template <int G, int MODE, int NCW>
static cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
  const size_t smem = decode_smem_bytes(G, a.U, NCW);
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<G, MODE, NCW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(DECODE_SMEM_MAX));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  return launch(decode_kernel<G, MODE, NCW>, dim3(a.n_ctas), dim3(NCW * 32), smem, s, a);
}

template <int G, int MODE>
static cudaError_t launch_decode_g(const DecodeArgs &a, cudaStream_t s) {
  if constexpr (G >= 8) {
    return launch_decode<G, MODE, NCW_NARROW>(a, s);
  } else {
    return decode_ncw(G, a.U, a.cap, a.n_ctas) == NCW_WIDE ? launch_decode<G, MODE, NCW_WIDE>(a, s)
                                                           : launch_decode<G, MODE, NCW_NARROW>(a, s);
  }
}

template <int MODE>
static cudaError_t dispatch_decode(int G, const DecodeArgs &a, cudaStream_t s) {
  switch (G) {
    case 1: return launch_decode_g<1, MODE>(a, s);
    case 2: return launch_decode_g<2, MODE>(a, s);
    case 4: return launch_decode_g<4, MODE>(a, s);
    case 8: return launch_decode_g<8, MODE>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hyq

using namespace hyq;

extern "C" hyq_status hyq_check_cache(const hyq_cache *c);  // hyq_api.cu
extern "C" int32_t hyq_sm_count(void);                      // hyq_api.cu

static inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int resolve_ctas(int32_t n_ctas) {
  if (n_ctas > 0) return n_ctas;
  return hyq_sm_count();
}

extern "C" int32_t hyq_decode_default_ctas(void) { return resolve_ctas(0); }

extern "C" size_t hyq_decode_workspace(const hyq_cache *c, int32_t n_ctas) {
  if (!c || c->n_kv_heads <= 0 || c->n_q_heads % c->n_kv_heads) return 0;
  return decode_ws_bytes(c->n_q_heads / c->n_kv_heads, c->batch * c->n_kv_heads, resolve_ctas(n_ctas));
}

extern "C" size_t hyq_decode_fp16_workspace(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                            int32_t n_ctas) {
  if (n_kv_heads <= 0 || n_q_heads % n_kv_heads) return 0;
  return decode_ws_bytes(n_q_heads / n_kv_heads, batch * n_kv_heads, resolve_ctas(n_ctas));
}

static bool g_supported(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

// The kernels split the work in int32 cost units; bound the total.
static bool cost_fits(int U, int cap, int vl_cap, int mode) {
  const int64_t per_unit = (mode == MODE_FP16)
                               ? static_cast<int64_t>(COST16) * ((cap + F16_ROWS - 1) / F16_ROWS)
                               : static_cast<int64_t>(COST4) * ((cap + I4_TOK - 1) / I4_TOK) +
                                     static_cast<int64_t>(COST16) * ((vl_cap + F16_ROWS - 1) / F16_ROWS + WIN / F16_ROWS);
  return static_cast<int64_t>(U) * per_unit < (static_cast<int64_t>(1) << 31) - 1;
}

template <int MODE>
static hyq_status decode_entry(const hyq_cache *c, const void *q, void *o, float *lse, int32_t n_ctas, void *ws,
                               size_t ws_bytes, void *stream) {
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!q || !o) return HYQ_ERR_INVALID;
  if (!al16(q) || !al16(o) || (lse && !al16(lse)) || !al16(ws)) return HYQ_ERR_ALIGN;
  if (n_ctas < 0) return HYQ_ERR_INVALID;
  const int G = c->n_q_heads / c->n_kv_heads;
  const int U = c->batch * c->n_kv_heads;
  if (U > MAX_UNITS || !cost_fits(U, c->capacity, c->vl_capacity, MODE_HYBRID)) return HYQ_ERR_UNSUPPORTED;
  const int N = resolve_ctas(n_ctas);
  if (!ws || ws_bytes < decode_ws_bytes(G, U, N)) return HYQ_ERR_WORKSPACE;
  DecodeArgs a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.cap = c->capacity;
  a.W = c->window; a.vl_cap = c->vl_capacity; a.U = U; a.n_ctas = N;
  a.blocks = c->blocks;
  a.rm = RecMap{c->block_table, c->n_kv_heads, c->capacity, c->n_pages, c->dev_status};
  a.win_k = static_cast<__half *>(c->win_k); a.win_v = static_cast<__half *>(c->win_v);
  a.vl_k = static_cast<const __half *>(c->vl_k); a.vl_v = static_cast<const __half *>(c->vl_v);
  a.vl_count = c->vl_count; a.seq_len = c->seq_len;
  a.q = static_cast<const __half *>(q); a.o = static_cast<__half *>(o); a.lse = lse;
  a.counters = static_cast<int32_t *>(ws);
  a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (static_cast<size_t>(U) * 4 + 255) / 256 * 256);
  a.status = c->dev_status;
  return dispatch_decode<MODE>(G, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

extern "C" hyq_status hyq_decode(const hyq_cache *c, const void *q, void *o, float *lse,
                                 int32_t n_ctas, void *ws, size_t ws_bytes, void *stream) {
  HYQ_RANGE("hyq_decode");
  return decode_entry<MODE_HYBRID>(c, q, o, lse, n_ctas, ws, ws_bytes, stream);
}

extern "C" hyq_status hyq_decode_vl_only(const hyq_cache *c, const void *q, void *o, float *lse,
                                         int32_t n_ctas, void *ws, size_t ws_bytes, void *stream) {
  HYQ_RANGE("hyq_decode_vl_only");
  return decode_entry<MODE_VLONLY>(c, q, o, lse, n_ctas, ws, ws_bytes, stream);
}

// Fused append + decode: the workspace of hyq_decode plus 256 bytes for the
// block counter of the seq_len update.
extern "C" size_t hyq_decode_step_workspace(const hyq_cache *c, int32_t n_ctas) {
  const size_t base = hyq_decode_workspace(c, n_ctas);
  return base ? base + 256 : 0;
}

extern "C" hyq_status hyq_decode_step(const hyq_cache *c, const void *q, const void *k_new, const void *v_new,
                                      void *q_ring, int32_t n_q, void *o, float *lse, int32_t n_ctas, void *ws,
                                      size_t ws_bytes, void *stream) {
  HYQ_RANGE("hyq_decode_step");
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!q || !o || !k_new || !v_new) return HYQ_ERR_INVALID;
  if (q_ring && (n_q < 1 || n_q > 1024)) return HYQ_ERR_INVALID;
  if (!al16(q) || !al16(o) || !al16(k_new) || !al16(v_new) || (q_ring && !al16(q_ring)) || (lse && !al16(lse)) ||
      !al16(ws))
    return HYQ_ERR_ALIGN;
  if (n_ctas < 0) return HYQ_ERR_INVALID;
  const int G = c->n_q_heads / c->n_kv_heads;
  const int U = c->batch * c->n_kv_heads;
  if (U > MAX_UNITS || !cost_fits(U, c->capacity, c->vl_capacity, MODE_STEP)) return HYQ_ERR_UNSUPPORTED;
  const int N = resolve_ctas(n_ctas);
  const size_t dws = decode_ws_bytes(G, U, N);
  if (!ws || ws_bytes < dws + 256) return HYQ_ERR_WORKSPACE;
  DecodeArgs a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.cap = c->capacity;
  a.W = c->window; a.vl_cap = c->vl_capacity; a.U = U; a.n_ctas = N;
  a.blocks = c->blocks;
  a.rm = RecMap{c->block_table, c->n_kv_heads, c->capacity, c->n_pages, c->dev_status};
  a.win_k = static_cast<__half *>(c->win_k); a.win_v = static_cast<__half *>(c->win_v);
  a.vl_k = static_cast<const __half *>(c->vl_k); a.vl_v = static_cast<const __half *>(c->vl_v);
  a.vl_count = c->vl_count; a.seq_len = c->seq_len;
  a.q = static_cast<const __half *>(q); a.o = static_cast<__half *>(o); a.lse = lse;
  a.counters = static_cast<int32_t *>(ws);
  a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (static_cast<size_t>(U) * 4 + 255) / 256 * 256);
  a.status = c->dev_status;
  a.k_new = static_cast<const __half *>(k_new); a.v_new = static_cast<const __half *>(v_new);
  a.q_ring = static_cast<__half *>(q_ring); a.n_q = n_q;
  a.stage_k = static_cast<__half *>(c->stage_k); a.stage_v = static_cast<__half *>(c->stage_v);
  a.stage_rows = c->stage_rows;
  a.grid_counter = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + dws);
  return dispatch_decode<MODE_STEP>(G, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? HYQ_OK
                                                                                            : HYQ_ERR_CUDA;
}

extern "C" hyq_status hyq_decode_fp16(const void *q, const void *k, const void *v,
                                      const int32_t *seq_len, int32_t batch, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t capacity, void *o, float *lse,
                                      int32_t n_ctas, void *ws, size_t ws_bytes,
                                      uint32_t *dev_status, void *stream) {
  HYQ_RANGE("hyq_decode_fp16");
  if (!q || !k || !v || !seq_len || !o) return HYQ_ERR_INVALID;
  if (batch <= 0 || n_kv_heads <= 0 || n_q_heads <= 0 || capacity <= 0 || n_ctas < 0)
    return HYQ_ERR_INVALID;
  if (n_q_heads % n_kv_heads || !g_supported(n_q_heads / n_kv_heads)) return HYQ_ERR_UNSUPPORTED;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || (lse && !al16(lse)) || !al16(ws) ||
      (reinterpret_cast<uintptr_t>(seq_len) & 3u))
    return HYQ_ERR_ALIGN;
  const int G = n_q_heads / n_kv_heads;
  const int U = batch * n_kv_heads;
  if (U > MAX_UNITS || !cost_fits(U, capacity, 0, MODE_FP16)) return HYQ_ERR_UNSUPPORTED;
  const int N = resolve_ctas(n_ctas);
  if (!ws || ws_bytes < decode_ws_bytes(G, U, N)) return HYQ_ERR_WORKSPACE;
  DecodeArgs a{};
  a.B = batch; a.Hq = n_q_heads; a.Hkv = n_kv_heads; a.cap = capacity; a.W = WIN; a.vl_cap = 0;
  a.U = U; a.n_ctas = N; a.seq_len = const_cast<int32_t *>(seq_len);  // read only in this mode
  a.k16 = static_cast<const __half *>(k); a.v16 = static_cast<const __half *>(v);
  a.q = static_cast<const __half *>(q); a.o = static_cast<__half *>(o); a.lse = lse;
  a.counters = static_cast<int32_t *>(ws);
  a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (static_cast<size_t>(U) * 4 + 255) / 256 * 256);
  a.status = dev_status;
  return dispatch_decode<MODE_FP16>(G, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? HYQ_OK
                                                                                            : HYQ_ERR_CUDA;
}

// ---------------------------------------------------------------- no-alloc variant
// hyq_decode_noalloc: the same decode for callers that cannot allocate
// device memory or carry a workspace pointer.  Its scratch -- the per-unit
// tile counters and the per-block partial records of the split merge -- is
// this fixed array, which every GPU that loads the library keeps until the
// process exits.  Layout as in hyq_decode: counters, then partials.
namespace {
constexpr int NOALLOC_MAX_UNITS = 4096;  // batch x kv heads
constexpr int NOALLOC_MAX_CTAS = 320;    // thread blocks of one launch
constexpr int NOALLOC_MAX_G = 8;
constexpr size_t NOALLOC_BYTES = static_cast<size_t>(NOALLOC_MAX_UNITS) * 4 +
                                 static_cast<size_t>(NOALLOC_MAX_CTAS) * 2 * NOALLOC_MAX_G * PART_STRIDE * 4;
__device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_BYTES];

// Host code cannot pass g_noalloc_scratch itself (that name is a host-side
// stand-in); its device address is looked up with cudaGetSymbolAddress, with
// the device current, once per device and CUDA context, and reused.  The
// context's unique id is part of the key: after cudaDeviceReset the runtime
// makes a new primary context and loads the module again, which may place
// the array elsewhere, so the next call looks it up again.  The driver calls
// that give the id are found through the runtime's entry-point query, so the
// library does not link the driver library itself.
struct NoallocSlot {
  unsigned long long ctx_id;
  void *addr;
};
NoallocSlot g_noalloc_slot[64] = {};
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the current context (false when none is current or the query
// is unavailable).  Called with g_noalloc_mu held.
bool current_ctx_id(unsigned long long *id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult r1 = cudaDriverEntryPointSymbolNotFound, r2 = r1;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &r1) != cudaSuccess ||
        r1 != cudaDriverEntryPointSuccess || !f1)
      return false;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &r2) != cudaSuccess ||
        r2 != cudaDriverEntryPointSuccess || !f2)
      return false;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

bool noalloc_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  NoallocSlot &slot = g_noalloc_slot[dev];
  if (have_id && slot.addr && slot.ctx_id == id) {
    *out = slot.addr;
    return true;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return false;
  // the lookup makes the device's primary context current if it was not
  if (have_id || current_ctx_id(&id)) {
    slot.ctx_id = id;
    slot.addr = p;
  }
  *out = p;
  return true;
}
}  // namespace

extern "C" hyq_status hyq_decode_noalloc(const hyq_cache *c, const void *q, void *o, float *lse,
                                         void *stream) {
  HYQ_RANGE("hyq_decode_noalloc");
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!q || !o) return HYQ_ERR_INVALID;
  if (!al16(q) || !al16(o) || (lse && !al16(lse))) return HYQ_ERR_ALIGN;
  const int G = c->n_q_heads / c->n_kv_heads;
  const int U = c->batch * c->n_kv_heads;
  const int N = resolve_ctas(0);
  if (U > NOALLOC_MAX_UNITS || N > NOALLOC_MAX_CTAS || G > NOALLOC_MAX_G) return HYQ_ERR_UNSUPPORTED;
  if (!cost_fits(U, c->capacity, c->vl_capacity, MODE_HYBRID)) return HYQ_ERR_UNSUPPORTED;
  if (decode_ws_bytes(G, U, N) > NOALLOC_BYTES) return HYQ_ERR_UNSUPPORTED;
  void *ws = nullptr;
  if (!noalloc_address(&ws)) return HYQ_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the last call's contents: the counters must start at 0
  if (cudaMemsetAsync(ws, 0, static_cast<size_t>(U) * 4, st) != cudaSuccess) return HYQ_ERR_CUDA;
  DecodeArgs a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.cap = c->capacity;
  a.W = c->window; a.vl_cap = c->vl_capacity; a.U = U; a.n_ctas = N;
  a.blocks = c->blocks;
  a.rm = RecMap{c->block_table, c->n_kv_heads, c->capacity, c->n_pages, c->dev_status};
  a.win_k = static_cast<__half *>(c->win_k); a.win_v = static_cast<__half *>(c->win_v);
  a.vl_k = static_cast<const __half *>(c->vl_k); a.vl_v = static_cast<const __half *>(c->vl_v);
  a.vl_count = c->vl_count; a.seq_len = c->seq_len;
  a.q = static_cast<const __half *>(q); a.o = static_cast<__half *>(o); a.lse = lse;
  a.counters = static_cast<int32_t *>(ws);
  a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (static_cast<size_t>(U) * 4 + 255) / 256 * 256);
  a.status = c->dev_status;
  return dispatch_decode<MODE_HYBRID>(G, a, st) == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

#ifdef HYQ_DEBUG
// Debug library only: the decode kernels' tile-wait limit and the stall
// switch on the current device.  Synchronous.
extern "C" hyq_status hyq_debug_set_wait(uint64_t limit_ns, int32_t stall_first_wait) {
  if (limit_ns < 1000 || limit_ns > 10000000000ull) return HYQ_ERR_INVALID;
  const int st = stall_first_wait ? 1 : 0;
  if (cudaMemcpyToSymbol(g_debug_wait_ns, &limit_ns, sizeof(limit_ns)) != cudaSuccess) return HYQ_ERR_CUDA;
  return cudaMemcpyToSymbol(g_debug_stall, &st, sizeof(st)) == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}
#endif

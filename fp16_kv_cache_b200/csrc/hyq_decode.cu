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
//   * Work: per unit (batch, kv head) the positions are cut into tiles -- INT4
//     tiles of 64 tokens (160 B per token: 64 B K codes, 16 B K scale/zero,
//     64 B V codes, 16 B V scale/zero) and FP16 tiles of 16 rows (512 B per
//     row).  All tiles of all units are concatenated and the launch's blocks
//     take equal contiguous runs of tiles (split-KV with the split points
//     chosen by tile count, so any batch/length mix keeps every SM busy).
//   * Pipeline: one producer warp streams tiles into an 8-slot shared-memory
//     ring with 1-D bulk copies (cp.async.bulk, no multicast) completing on
//     mbarriers; tile i is consumed by consumer warp i % 4.
//   * Math: Q.K and P.V run on the tensor cores (mma.sync m16n8k16, fp16 in,
//     fp32 accumulate), tokens on the M side so a 16-token slice is one MMA
//     row block and the G <= 8 query heads of the unit fill N.  INT4 codes
//     enter the MMA as exact small integers (nibble -> fp16 by exponent
//     bias); the per-(token, group) scale and zero are applied in fp32:
//       s = sum_g scale_g * (q_g . code_g) + zero_g * sum(q_g)
//       o += sum_t (p_t * vscale_tg) * vcode_t + sum_t p_t * vzero_tg.
//     The softmax is fp32 online (running max / sum, exp2 domain), reduced
//     across lanes with warp shuffles; scores of skipped or padded tokens are
//     -inf.  Positions held in the vertical-line segment are skipped in the
//     INT4 sweep through the cache's bitmask.
//   * Combine: a block that finishes a unit writes O directly; otherwise it
//     writes its (max, sum, acc) partial and the last block to finish the
//     unit (atomic tile counter) merges the partials by log-sum-exp.
#include "hyq_common.cuh"

namespace hyq {

constexpr int NCW = 4;                    // consumer warps
constexpr int NTHREADS = (NCW + 1) * 32;  // + 1 producer warp
constexpr int NS = 8;                     // shared-memory ring slots
constexpr int I4_TOK = 64;                // tokens per INT4 tile
constexpr int F16_ROWS = 16;              // rows per FP16 tile
constexpr int KF_STRIDE = 320;            // bytes between FP16 K rows in a slot
constexpr int VF_STRIDE = 272;            // bytes between FP16 V rows in a slot
constexpr int SLOT_KSZ = I4_TOK * ROW_BYTES;         // 4096
constexpr int SLOT_VC = SLOT_KSZ + I4_TOK * SZ_BYTES;  // 5120
constexpr int SLOT_VSZ = SLOT_VC + I4_TOK * ROW_BYTES;  // 9216
constexpr int SLOT_MASK = SLOT_VSZ + I4_TOK * SZ_BYTES;  // 10240
constexpr int SLOT_BYTES = SLOT_MASK + 64;                // 10304
constexpr int PART_STRIDE = 132;  // floats per (partial, head): m, l, -, -, acc[128]
constexpr float LOG2E_OVER_SQRT_D = 0.12751743082459868f;  // log2(e) / sqrt(128)
constexpr float LN2 = 0.69314718055994531f;

static_assert(F16_ROWS * (KF_STRIDE + VF_STRIDE) <= SLOT_MASK, "fp16 tile fits a slot");

enum { MODE_HYBRID = 0, MODE_FP16 = 1 };

struct DecodeArgs {
  int B, Hq, Hkv, cap, W, vl_cap, U, n_ctas;
  const uint8_t *k_codes, *v_codes, *k_sz, *v_sz;
  const __half *win_k, *win_v, *vl_k, *vl_v;
  const int32_t *vl_count;
  const uint32_t *vl_mask;
  const int32_t *seq_len;
  const __half *k16, *v16;  // comparator cache [B][Hkv][cap][128]
  const __half *q;
  __half *o;
  float *lse;
  float *part;        // [n_ctas][2][G][PART_STRIDE]
  int32_t *counters;  // [U]
  uint32_t *status;
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
__device__ __forceinline__ UnitShape unit_shape(const DecodeArgs &a, int u, bool &bad) {
  UnitShape s;
  const int b = u / a.Hkv;
  s.T = a.seq_len[b];
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
  s.vlc = a.vl_count[u];
  if (s.vlc < 0 || s.vlc > a.vl_cap || s.vlc > s.L4) {
    bad = true;
    s.vlc = 0;
  }
  s.nwin = s.T < a.W ? s.T : a.W;
  s.n4 = (s.L4 + I4_TOK - 1) / I4_TOK;
  s.nv = (s.vlc + F16_ROWS - 1) / F16_ROWS;
  s.nw = (s.nwin + F16_ROWS - 1) / F16_ROWS;
  return s;
}

// Per-warp running state, in the accumulator layout of m16n8: lane (r, q)
// holds query heads 2q and 2q+1 of the unit (heads >= G are padding).
struct WarpState {
  float m[2], l[2];
  float zs[2][NG];         // sum over tokens of p * vzero, per (head, group)
  float acc[NG][2][4];     // O^T accumulators: m-tile (group g, half j)
  uint32_t qf[NG][2][2];   // Q as the B operand: k-step (group g, piece s)
  float qs[2][NG];         // log2(e)/sqrt(d) * sum of q over each group
};

__device__ __forceinline__ void state_reset(WarpState &st) {
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    st.m[e] = -INFINITY;
    st.l[e] = 0.f;
#pragma unroll
    for (int g = 0; g < NG; ++g) st.zs[e][g] = 0.f;
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
template <int G>
__device__ __forceinline__ void load_q(WarpState &st, const DecodeArgs &a, int u, int lane) {
  const int n = lane >> 2, q4 = lane & 3;
  const int b = u / a.Hkv, kvh = u % a.Hkv;
  float part[NG];
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
    float s = 0.f;
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __half22float2(h[i]);
      s += f.x + f.y;
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    part[g] = s * LOG2E_OVER_SQRT_D;  // lanes 4n..4n+3 hold head n
  }
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    st.qs[0][g] = __shfl_sync(0xffffffffu, part[g], (2 * q4) * 4);
    st.qs[1][g] = __shfl_sync(0xffffffffu, part[g], (2 * q4 + 1) * 4);
  }
}

// Online softmax over the 4 scores a lane holds: rows A (token sig(r)) and
// B (sig(r)+8), heads 2q and 2q+1.  Returns the probabilities relative to the
// running max; rescales the running state when the max grows.
__device__ __forceinline__ void softmax_step(WarpState &st, float (&S)[4], bool vA, bool vB,
                                             float (&p)[4]) {
  float mx0 = fmaxf(S[0], S[2]), mx1 = fmaxf(S[1], S[3]);
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
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      st.zs[0][g] *= a0;
      st.zs[1][g] *= a1;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        st.acc[g][j][0] *= a0;
        st.acc[g][j][1] *= a1;
        st.acc[g][j][2] *= a0;
        st.acc[g][j][3] *= a1;
      }
    }
  }
  p[0] = vA ? fast_exp2(S[0] - st.m[0]) : 0.f;
  p[1] = vA ? fast_exp2(S[1] - st.m[1]) : 0.f;
  p[2] = vB ? fast_exp2(S[2] - st.m[0]) : 0.f;
  p[3] = vB ? fast_exp2(S[3] - st.m[1]) : 0.f;
  st.l[0] += p[0] + p[2];
  st.l[1] += p[1] + p[3];
}

// One INT4 tile (up to 64 tokens) staged at `slot`.
__device__ __forceinline__ void int4_tile(WarpState &st, uint32_t slot, int n_valid, uint64_t vlbits,
                                          int lane) {
  const int r = lane >> 2, q4 = lane & 3;
  const uint32_t kc = slot, ksz = slot + SLOT_KSZ, vc = slot + SLOT_VC, vsz = slot + SLOT_VSZ;
  const int s2q = sig(2 * q4), s2q1 = sig(2 * q4 + 1);
#pragma unroll 1
  for (int mt = 0; mt < I4_TOK / 16; ++mt) {
    if (16 * mt >= n_valid) break;
    const int tA = 16 * mt + sig(r), tB = tA + 8;
    const bool vA = tA < n_valid && !((vlbits >> tA) & 1ull);
    const bool vB = tB < n_valid && !((vlbits >> tB) & 1ull);

    // ---- S = Q K^T per group on exact codes
    const uint4 ka = lds128(kc + tA * ROW_BYTES + 16 * q4);
    const uint4 kb = lds128(kc + tB * ROW_BYTES + 16 * q4);
    float sg[NG][4];
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) sg[g][e] = 0.f;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const uint32_t wa0 = s ? ka.z : ka.x, wa1 = s ? ka.w : ka.y;
      const uint32_t wb0 = s ? kb.z : kb.x, wb1 = s ? kb.w : kb.y;
      mma16816(sg[0], nib_lo(wa0), nib_lo(wb0), nib_hi(wa0), nib_hi(wb0), st.qf[0][s][0], st.qf[0][s][1]);
      mma16816(sg[1], nib_lo(wa0 >> 8), nib_lo(wb0 >> 8), nib_hi(wa0 >> 8), nib_hi(wb0 >> 8),
               st.qf[1][s][0], st.qf[1][s][1]);
      mma16816(sg[2], nib_lo(wa1), nib_lo(wb1), nib_hi(wa1), nib_hi(wb1), st.qf[2][s][0], st.qf[2][s][1]);
      mma16816(sg[3], nib_lo(wa1 >> 8), nib_lo(wb1 >> 8), nib_hi(wa1 >> 8), nib_hi(wb1 >> 8),
               st.qf[3][s][0], st.qf[3][s][1]);
    }
    const uint4 za = lds128(ksz + tA * SZ_BYTES), zb = lds128(ksz + tB * SZ_BYTES);
    const uint32_t zaw[4] = {za.x, za.y, za.z, za.w}, zbw[4] = {zb.x, zb.y, zb.z, zb.w};
    float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float2 fa = __half22float2(u2h(zaw[g]));  // (scale, zero) of row A
      const float2 fb = __half22float2(u2h(zbw[g]));
      const float ca = fa.x * LOG2E_OVER_SQRT_D, cb = fb.x * LOG2E_OVER_SQRT_D;
      S[0] += ca * sg[g][0] + fa.y * st.qs[0][g];
      S[1] += ca * sg[g][1] + fa.y * st.qs[1][g];
      S[2] += cb * sg[g][2] + fb.y * st.qs[0][g];
      S[3] += cb * sg[g][3] + fb.y * st.qs[1][g];
    }
    if (!vA) S[0] = S[1] = -INFINITY;
    if (!vB) S[2] = S[3] = -INFINITY;
    float p[4];
    softmax_step(st, S, vA, vB, p);

    // ---- O += P V: scale folded into P per group, zero added separately
    const uint4 wa = lds128(vsz + tA * SZ_BYTES), wb = lds128(vsz + tB * SZ_BYTES);
    const uint32_t waw[4] = {wa.x, wa.y, wa.z, wa.w}, wbw[4] = {wb.x, wb.y, wb.z, wb.w};
    uint32_t bq[NG][2];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float2 fa = __half22float2(u2h(waw[g]));
      const float2 fb = __half22float2(u2h(wbw[g]));
      const float sa = vA ? fa.x : 0.f, sb = vB ? fb.x : 0.f;
      const float za_ = vA ? fa.y : 0.f, zb_ = vB ? fb.y : 0.f;
      st.zs[0][g] += p[0] * za_ + p[2] * zb_;
      st.zs[1][g] += p[1] * za_ + p[3] * zb_;
      bq[g][0] = movmatrix_t(pack_half2(p[0] * sa, p[1] * sa));
      bq[g][1] = movmatrix_t(pack_half2(p[2] * sb, p[3] * sb));
    }
    const uint32_t vrow = vc + 8 * r;
    const uint2 x0 = lds64(vrow + (16 * mt + s2q) * ROW_BYTES);
    const uint2 x1 = lds64(vrow + (16 * mt + s2q1) * ROW_BYTES);
    const uint2 y0 = lds64(vrow + (16 * mt + s2q + 8) * ROW_BYTES);
    const uint2 y1 = lds64(vrow + (16 * mt + s2q1 + 8) * ROW_BYTES);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t A0 = hh ? x0.y : x0.x, A1 = hh ? x1.y : x1.x;
      const uint32_t B0 = hh ? y0.y : y0.x, B1 = hh ? y1.y : y1.x;
      const uint32_t xa = prmt(A0, A1, 0x5410u), ya = prmt(A0, A1, 0x7632u);
      const uint32_t xb = prmt(B0, B1, 0x5410u), yb = prmt(B0, B1, 0x7632u);
      const int g0 = 2 * hh, g1 = 2 * hh + 1;
      mma16816(st.acc[g0][0], nib_lo(xa), nib_hi(xa), nib_lo(xb), nib_hi(xb), bq[g0][0], bq[g0][1]);
      mma16816(st.acc[g0][1], nib_lo(ya), nib_hi(ya), nib_lo(yb), nib_hi(yb), bq[g0][0], bq[g0][1]);
      mma16816(st.acc[g1][0], nib_lo(xa >> 8), nib_hi(xa >> 8), nib_lo(xb >> 8), nib_hi(xb >> 8),
               bq[g1][0], bq[g1][1]);
      mma16816(st.acc[g1][1], nib_lo(ya >> 8), nib_hi(ya >> 8), nib_lo(yb >> 8), nib_hi(yb >> 8),
               bq[g1][0], bq[g1][1]);
    }
  }
}

// One FP16 tile (up to 16 rows) staged at `slot` (K rows at KF_STRIDE, V rows
// at VF_STRIDE).
__device__ __forceinline__ void f16_tile(WarpState &st, uint32_t slot, int n_valid, int lane) {
  const int r = lane >> 2, q4 = lane & 3;
  const uint32_t kb_ = slot, vb_ = slot + F16_ROWS * KF_STRIDE;
  const int tA = sig(r), tB = tA + 8;
  const bool vA = tA < n_valid, vB = tB < n_valid;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint4 ka = lds128(kb_ + tA * KF_STRIDE + 64 * g + 16 * q4);
    const uint4 kb = lds128(kb_ + tB * KF_STRIDE + 64 * g + 16 * q4);
    mma16816(acc, prmt(ka.x, ka.y, 0x5410u), prmt(kb.x, kb.y, 0x5410u), prmt(ka.x, ka.y, 0x7632u),
             prmt(kb.x, kb.y, 0x7632u), st.qf[g][0][0], st.qf[g][0][1]);
    mma16816(acc, prmt(ka.z, ka.w, 0x5410u), prmt(kb.z, kb.w, 0x5410u), prmt(ka.z, ka.w, 0x7632u),
             prmt(kb.z, kb.w, 0x7632u), st.qf[g][1][0], st.qf[g][1][1]);
  }
  float S[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) S[e] = acc[e] * LOG2E_OVER_SQRT_D;
  if (!vA) S[0] = S[1] = -INFINITY;
  if (!vB) S[2] = S[3] = -INFINITY;
  float p[4];
  softmax_step(st, S, vA, vB, p);
  const uint32_t b0 = movmatrix_t(pack_half2(p[0], p[1]));
  const uint32_t b1 = movmatrix_t(pack_half2(p[2], p[3]));
  const int t0 = sig(2 * q4), t1 = sig(2 * q4 + 1);
  const bool v0 = t0 < n_valid, v1 = t1 < n_valid, v2 = t0 + 8 < n_valid, v3 = t1 + 8 < n_valid;
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint32_t off = vb_ + 64 * g + 8 * r;
    const uint2 z2 = make_uint2(0, 0);
    const uint2 A0 = v0 ? lds64(off + t0 * VF_STRIDE) : z2;
    const uint2 A1 = v1 ? lds64(off + t1 * VF_STRIDE) : z2;
    const uint2 B0 = v2 ? lds64(off + (t0 + 8) * VF_STRIDE) : z2;
    const uint2 B1 = v3 ? lds64(off + (t1 + 8) * VF_STRIDE) : z2;
    mma16816(st.acc[g][0], prmt(A0.x, A1.x, 0x5410u), prmt(A0.x, A1.x, 0x7632u), prmt(B0.x, B1.x, 0x5410u),
             prmt(B0.x, B1.x, 0x7632u), b0, b1);
    mma16816(st.acc[g][1], prmt(A0.y, A1.y, 0x5410u), prmt(A0.y, A1.y, 0x7632u), prmt(B0.y, B1.y, 0x5410u),
             prmt(B0.y, B1.y, 0x7632u), b0, b1);
  }
}

struct Smem {
  uint32_t slots;     // shared address of slot 0
  uint64_t *full, *empty;
  int *abort_flag, *last_flag;
  float *mm, *ml, *mo;  // merge buffers: [NCW][8], [NCW][8], [NCW][G][128]
  int *tile_start;      // [U + 1]
  int *scan;            // [NTHREADS]
};

__device__ __forceinline__ int64_t cta_first_tile(int64_t c, int64_t n_tiles, int64_t n_ctas) {
  return c * n_tiles / n_ctas;
}
// CTA that owns global tile t: the largest c with first_tile(c) <= t.
__device__ __forceinline__ int cta_of_tile(int64_t t, int64_t n_tiles, int64_t n_ctas) {
  return static_cast<int>(((t + 1) * n_ctas - 1) / n_tiles);
}

// last unit u with tile_start[u] <= t < tile_start[u+1]
__device__ __forceinline__ int unit_of_tile(const int *ts, int U, int t) {
  int lo = 0, hi = U - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ts[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Merge the partials of unit u written by the blocks that share it (run by
// the last one to finish; 128 consumer threads).  Parts are taken in chunks
// of MERGE_CHUNK: their (max, sum) pairs are loaded in parallel, per-head
// weights 2^(m_p - M) live in shared memory, and every thread accumulates
// float4 slices of the output with many loads in flight.
constexpr int MERGE_CHUNK = 128;

template <int G>
__device__ __forceinline__ void merge_parts(const DecodeArgs &a, const Smem &sm, int u, int u0, int u1,
                                            int64_t n_tiles, int64_t N, int64_t hbase, int tid) {
  float *pw = sm.mo;                       // [MERGE_CHUNK][G] weights
  float *pl = sm.mo + MERGE_CHUNK * G;     // [MERGE_CHUNK][G] sums
  int *pid = sm.scan;                      // [MERGE_CHUNK] partial record index or -1
  float *runM = sm.mm, *runL = sm.ml, *alpha = sm.mm + 8;
  const int c_lo = cta_of_tile(u0, n_tiles, N), c_hi = cta_of_tile(u1 - 1, n_tiles, N);
  constexpr int NV = (G * D / 4 + NCW * 32 - 1) / (NCW * 32);  // float4 outputs per thread
  float4 acc[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid < G) {
    runM[tid] = -INFINITY;
    runL[tid] = 0.f;
  }
  for (int base = c_lo; base <= c_hi; base += MERGE_CHUNK) {
    const int n = min(MERGE_CHUNK, c_hi - base + 1);
    named_bar_sync(1, NCW * 32);
    for (int j = tid; j < n; j += NCW * 32) {
      const int64_t cc = base + j;
      const int64_t f0 = cta_first_tile(cc, n_tiles, N), f1 = cta_first_tile(cc + 1, n_tiles, N);
      pid[j] = (f0 == f1) ? -1 : static_cast<int>(cc * 2 + ((u0 >= f0) ? 0 : 1));
    }
    named_bar_sync(1, NCW * 32);
    for (int e = tid; e < n * G; e += NCW * 32) {
      const int j = e / G, h = e % G;
      float m = -INFINITY, l = 0.f;
      if (pid[j] >= 0) {
        const float *pr = a.part + (static_cast<int64_t>(pid[j]) * G + h) * PART_STRIDE;
        m = __ldcg(pr);
        l = __ldcg(pr + 1);
      }
      pw[e] = m;
      pl[e] = l;
    }
    named_bar_sync(1, NCW * 32);
    if (tid < G) {
      const int h = tid;
      float cm = -INFINITY;
      for (int j = 0; j < n; ++j) cm = fmaxf(cm, pw[j * G + h]);
      const float M = fmaxf(runM[h], cm);
      const float al = (runM[h] == -INFINITY) ? 0.f : fast_exp2(runM[h] - M);
      float L = runL[h] * al;
      for (int j = 0; j < n; ++j) {
        const float m = pw[j * G + h];
        const float w = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
        pw[j * G + h] = w;
        L += pl[j * G + h] * w;
      }
      runM[h] = M;
      runL[h] = L;
      alpha[h] = al;
    }
    named_bar_sync(1, NCW * 32);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int o4 = tid + v * NCW * 32;  // float4 index over [G][32]
      if (o4 < G * D / 4) {
        const int h = o4 / (D / 4), c4 = o4 % (D / 4);
        const float al = alpha[h];
        float4 s = make_float4(acc[v].x * al, acc[v].y * al, acc[v].z * al, acc[v].w * al);
#pragma unroll 16
        for (int j = 0; j < n; ++j) {
          const int id = pid[j];
          if (id < 0) continue;
          const float w = pw[j * G + h];
          const float4 x = __ldcg(reinterpret_cast<const float4 *>(
              a.part + (static_cast<int64_t>(id) * G + h) * PART_STRIDE + 4 + 4 * c4));
          s.x += w * x.x;
          s.y += w * x.y;
          s.z += w * x.z;
          s.w += w * x.w;
        }
        acc[v] = s;
      }
    }
  }
  named_bar_sync(1, NCW * 32);
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int o4 = tid + v * NCW * 32;
    if (o4 < G * D / 4) {
      const int h = o4 / (D / 4), c4 = o4 % (D / 4);
      const float inv = 1.f / runL[h];
      __half2 lo = __floats2half2_rn(acc[v].x * inv, acc[v].y * inv);
      __half2 hi = __floats2half2_rn(acc[v].z * inv, acc[v].w * inv);
      uint2 pk = make_uint2(h2u(lo), h2u(hi));
      *reinterpret_cast<uint2 *>(a.o + (hbase + h) * D + 4 * c4) = pk;
      if (c4 == 0 && a.lse) a.lse[hbase + h] = (runM[h] + __log2f(runL[h])) * LN2;
    }
  }
}

template <int G, int MODE>
__global__ void __launch_bounds__(NTHREADS, 2) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Smem sm;
  {
    uint8_t *p = smem_raw;
    sm.slots = smem_u32(p);
    p += NS * SLOT_BYTES;
    sm.full = reinterpret_cast<uint64_t *>(p);
    p += NS * 8;
    sm.empty = reinterpret_cast<uint64_t *>(p);
    p += NS * 8;
    sm.abort_flag = reinterpret_cast<int *>(p);
    sm.last_flag = sm.abort_flag + 1;
    p += 16;
    sm.mm = reinterpret_cast<float *>(p);
    p += NCW * 8 * 4;
    sm.ml = reinterpret_cast<float *>(p);
    p += NCW * 8 * 4;
    sm.mo = reinterpret_cast<float *>(p);
    p += NCW * G * D * 4;
    sm.scan = reinterpret_cast<int *>(p);
    p += NTHREADS * 4;
    sm.tile_start = reinterpret_cast<int *>(p);
  }
  const int U = a.U;

  // ---- schedule: tile_start[u] = tiles of units before u
  {
    const int per = (U + NTHREADS - 1) / NTHREADS;
    const int beg = min(U, tid * per), end = min(U, beg + per);
    int local = 0;
    for (int u = beg; u < end; ++u) {
      bool bad;
      const UnitShape s = unit_shape<MODE>(a, u, bad);
      local += s.n4 + s.nv + s.nw;
    }
    // block exclusive scan of `local`
    int v = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    if (lane == 31) sm.scan[warp] = v;
    if (tid == 0) {
      *sm.abort_flag = 0;
      for (int s = 0; s < NS; ++s) {
        mbar_init(smem_u32(&sm.full[s]), 1);
        mbar_init(smem_u32(&sm.empty[s]), 1);
      }
      fence_barrier_init();
    }
    __syncthreads();
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += sm.scan[w];
    int acc = wpre + v - local;
    for (int u = beg; u < end; ++u) {
      bool bad;
      const UnitShape s = unit_shape<MODE>(a, u, bad);
      sm.tile_start[u] = acc;
      acc += s.n4 + s.nv + s.nw;
      if (bad && (u % a.n_ctas) == static_cast<int>(blockIdx.x)) set_status(a.status, HYQ_DEV_BADLEN);
    }
    if (tid == NTHREADS - 1) sm.tile_start[U] = acc;
    __syncthreads();
  }
  const int64_t n_tiles = sm.tile_start[U];
  const int64_t N = a.n_ctas;
  const int cta = blockIdx.x;
  const int t_begin = static_cast<int>(cta_first_tile(cta, n_tiles, N));
  const int t_end = static_cast<int>(cta_first_tile(cta + 1, n_tiles, N));
  volatile int *abort_flag = sm.abort_flag;

  if (warp == NCW) {
    // ================= producer
    int i = 0;
    bool ok = true;
    for (int t = t_begin; t < t_end && ok;) {
      const int u = unit_of_tile(sm.tile_start, U, t);
      const int u0 = sm.tile_start[u], u1 = sm.tile_start[u + 1];
      const int seg_end = min(t_end, u1);
      bool bad;
      const UnitShape us = unit_shape<MODE>(a, u, bad);
      for (; t < seg_end; ++t, ++i) {
        const int s = i % NS;
        const uint32_t ph = (i / NS) & 1;
        if (i >= NS && !mbar_wait_bounded(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag, a.status)) {
          ok = false;
          break;
        }
        const uint32_t dst = sm.slots + s * SLOT_BYTES;
        const uint32_t bar = smem_u32(&sm.full[s]);
        const int j = t - u0;
        if (MODE == MODE_HYBRID && j < us.n4) {
          const int t0 = j * I4_TOK;
          const int n = min(I4_TOK, us.L4 - t0);
          if (lane == 0) {
            const int64_t row = static_cast<int64_t>(u) * a.cap + t0;
            mbar_arrive_expect_tx(bar, n * 160 + 16);
            bulk_g2s(dst, a.k_codes + row * ROW_BYTES, n * ROW_BYTES, bar);
            bulk_g2s(dst + SLOT_KSZ, a.k_sz + row * SZ_BYTES, n * SZ_BYTES, bar);
            bulk_g2s(dst + SLOT_VC, a.v_codes + row * ROW_BYTES, n * ROW_BYTES, bar);
            bulk_g2s(dst + SLOT_VSZ, a.v_sz + row * SZ_BYTES, n * SZ_BYTES, bar);
            const uint32_t *mrow = a.vl_mask + static_cast<int64_t>(u) * (a.cap / 32);
            bulk_g2s(dst + SLOT_MASK, mrow + ((t0 / 32) & ~3), 16, bar);
          }
        } else {
          const __half *sk, *sv;
          int r0, n;
          if (MODE == MODE_FP16) {
            r0 = j * F16_ROWS;
            n = min(F16_ROWS, us.T - r0);
            const int64_t base = (static_cast<int64_t>(u) * a.cap + r0) * D;
            sk = a.k16 + base;
            sv = a.v16 + base;
          } else if (j < us.n4 + us.nv) {
            r0 = (j - us.n4) * F16_ROWS;
            n = min(F16_ROWS, us.vlc - r0);
            const int64_t base = (static_cast<int64_t>(u) * a.vl_cap + r0) * D;
            sk = a.vl_k + base;
            sv = a.vl_v + base;
          } else {
            r0 = (j - us.n4 - us.nv) * F16_ROWS;
            n = min(F16_ROWS, us.nwin - r0);
            const int64_t base = (static_cast<int64_t>(u) * a.W + r0) * D;
            sk = a.win_k + base;
            sv = a.win_v + base;
          }
          if (lane == 0) mbar_arrive_expect_tx(bar, n * 2 * D * 2);
          __syncwarp();
          if (lane < n) {
            bulk_g2s(dst + lane * KF_STRIDE, sk + lane * D, D * 2, bar);
            bulk_g2s(dst + F16_ROWS * KF_STRIDE + lane * VF_STRIDE, sv + lane * D, D * 2, bar);
          }
        }
        __syncwarp();
      }
      (void)u1;
    }
    if (!ok) {
      // let copies already issued land before the block can exit
      for (int k = (i > NS ? i - NS : 0); k < i; ++k)
        mbar_wait_bounded(smem_u32(&sm.full[k % NS]), (k / NS) & 1, abort_flag, a.status, 500000000ull);
    }
    return;
  }

  // ================= consumers
  WarpState st;
  int i = 0;
  for (int t = t_begin; t < t_end;) {
    const int u = unit_of_tile(sm.tile_start, U, t);
    const int u0 = sm.tile_start[u], u1 = sm.tile_start[u + 1];
    const int seg_beg = t, seg_end = min(t_end, u1);
    bool bad;
    const UnitShape us = unit_shape<MODE>(a, u, bad);
    state_reset(st);
    load_q<G>(st, a, u, lane);
    for (; t < seg_end; ++t, ++i) {
      if (i % NCW != warp) continue;
      const int s = i % NS;
      const uint32_t ph = (i / NS) & 1;
      if (!mbar_wait_bounded(smem_u32(&sm.full[s]), ph, abort_flag, a.status)) continue;
      const uint32_t slot = sm.slots + s * SLOT_BYTES;
      const int j = t - u0;
      if (MODE == MODE_HYBRID && j < us.n4) {
        const int t0 = j * I4_TOK;
        const int n = min(I4_TOK, us.L4 - t0);
        const uint4 mw = lds128(slot + SLOT_MASK);
        const int wsel = (t0 / 32) & 3;  // 0 or 2
        const uint32_t lo = wsel ? mw.z : mw.x, hi = wsel ? mw.w : mw.y;
        int4_tile(st, slot, n, (static_cast<uint64_t>(hi) << 32) | lo, lane);
      } else {
        int n;
        if (MODE == MODE_FP16)
          n = min(F16_ROWS, us.T - j * F16_ROWS);
        else if (j < us.n4 + us.nv)
          n = min(F16_ROWS, us.vlc - (j - us.n4) * F16_ROWS);
        else
          n = min(F16_ROWS, us.nwin - (j - us.n4 - us.nv) * F16_ROWS);
        f16_tile(st, slot, n, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
    }

    // ---- segment end: reduce the warp's state over token rows
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        st.l[e] += __shfl_xor_sync(0xffffffffu, st.l[e], off);
#pragma unroll
        for (int g = 0; g < NG; ++g) st.zs[e][g] += __shfl_xor_sync(0xffffffffu, st.zs[e][g], off);
      }
    }
    const int r = lane >> 2, q4 = lane & 3;
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
            orow[ch] = st.acc[g][j][e] + st.zs[e][g];
            orow[ch + 1] = st.acc[g][j][2 + e] + st.zs[e][g];
          }
      }
    }
    named_bar_sync(1, NCW * 32);

    // ---- merge the consumer warps
    const bool complete = (seg_beg == u0) && (seg_end == u1);
    const int slot_id = (u0 >= t_begin) ? 0 : 1;  // 1: the unit began in an earlier block
    const int b = u / a.Hkv, kvh = u % a.Hkv;
    const int64_t hbase = static_cast<int64_t>(b) * a.Hq + kvh * G;
    for (int idx = tid; idx < G * D; idx += NCW * 32) {
      const int h = idx / D, c = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, sm.mm[w * 8 + h]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = sm.mm[w * 8 + h];
        const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
        L += sm.ml[w * 8 + h] * f;
        O += sm.mo[(w * G + h) * D + c] * f;
      }
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
      __threadfence();
      named_bar_sync(1, NCW * 32);
      if (tid == 0) {
        const int mine = seg_end - seg_beg;
        const int old = atomicAdd(&a.counters[u], mine);
        *sm.last_flag = (old + mine == u1 - u0);
      }
      named_bar_sync(1, NCW * 32);
      if (*sm.last_flag) {
        __threadfence();
        merge_parts<G>(a, sm, u, u0, u1, n_tiles, N, hbase, tid);
        if (tid == 0) a.counters[u] = 0;
      }
    }
    named_bar_sync(1, NCW * 32);
    t = seg_end;
  }

  // units without any position: o = 0, lse = -inf (one block each)
  for (int u = cta; u < U; u += a.n_ctas) {
    if (sm.tile_start[u] != sm.tile_start[u + 1]) continue;
    const int b = u / a.Hkv, kvh = u % a.Hkv;
    const int64_t hbase = static_cast<int64_t>(b) * a.Hq + kvh * G;
    for (int idx = tid; idx < G * D; idx += NCW * 32) {
      a.o[(hbase + idx / D) * D + idx % D] = __float2half_rn(0.f);
      if (idx % D == 0 && a.lse) a.lse[hbase + idx / D] = -INFINITY;
    }
  }
}

// ---------------------------------------------------------------- host side
static size_t decode_smem_bytes(int G, int U) {
  return static_cast<size_t>(NS) * SLOT_BYTES + NS * 16 + 16 + NCW * 8 * 4 * 2 +
         static_cast<size_t>(NCW) * G * D * 4 + NTHREADS * 4 + static_cast<size_t>(U + 1) * 4;
}

static size_t decode_ws_bytes(int G, int U, int n_ctas) {
  const size_t cnt = (static_cast<size_t>(U) * 4 + 255) / 256 * 256;
  return cnt + static_cast<size_t>(n_ctas) * 2 * G * PART_STRIDE * 4;
}

template <int G, int MODE>
static cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
  const size_t smem = decode_smem_bytes(G, a.U);
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<G, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  decode_kernel<G, MODE><<<a.n_ctas, NTHREADS, smem, s>>>(a);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t dispatch_decode(int G, const DecodeArgs &a, cudaStream_t s) {
  switch (G) {
    case 1: return launch_decode<1, MODE>(a, s);
    case 2: return launch_decode<2, MODE>(a, s);
    case 4: return launch_decode<4, MODE>(a, s);
    case 8: return launch_decode<8, MODE>(a, s);
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
  return 2 * hyq_sm_count();
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

extern "C" hyq_status hyq_decode(const hyq_cache *c, const void *q, void *o, float *lse,
                                 int32_t n_ctas, void *ws, size_t ws_bytes, void *stream) {
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!q || !o) return HYQ_ERR_INVALID;
  if (!al16(q) || !al16(o) || (lse && !al16(lse)) || !al16(ws)) return HYQ_ERR_ALIGN;
  if (n_ctas < 0) return HYQ_ERR_INVALID;
  const int G = c->n_q_heads / c->n_kv_heads;
  const int U = c->batch * c->n_kv_heads;
  if (U > MAX_UNITS) return HYQ_ERR_UNSUPPORTED;
  const int N = resolve_ctas(n_ctas);
  if (!ws || ws_bytes < decode_ws_bytes(G, U, N)) return HYQ_ERR_WORKSPACE;
  DecodeArgs a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.cap = c->capacity;
  a.W = c->window; a.vl_cap = c->vl_capacity; a.U = U; a.n_ctas = N;
  a.k_codes = c->k_codes; a.v_codes = c->v_codes;
  a.k_sz = static_cast<const uint8_t *>(c->k_sz); a.v_sz = static_cast<const uint8_t *>(c->v_sz);
  a.win_k = static_cast<const __half *>(c->win_k); a.win_v = static_cast<const __half *>(c->win_v);
  a.vl_k = static_cast<const __half *>(c->vl_k); a.vl_v = static_cast<const __half *>(c->vl_v);
  a.vl_count = c->vl_count; a.vl_mask = c->vl_mask; a.seq_len = c->seq_len;
  a.q = static_cast<const __half *>(q); a.o = static_cast<__half *>(o); a.lse = lse;
  a.counters = static_cast<int32_t *>(ws);
  a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (static_cast<size_t>(U) * 4 + 255) / 256 * 256);
  a.status = c->dev_status;
  return dispatch_decode<MODE_HYBRID>(G, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? HYQ_OK
                                                                                              : HYQ_ERR_CUDA;
}

extern "C" hyq_status hyq_decode_fp16(const void *q, const void *k, const void *v,
                                      const int32_t *seq_len, int32_t batch, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t capacity, void *o, float *lse,
                                      int32_t n_ctas, void *ws, size_t ws_bytes,
                                      uint32_t *dev_status, void *stream) {
  if (!q || !k || !v || !seq_len || !o) return HYQ_ERR_INVALID;
  if (batch <= 0 || n_kv_heads <= 0 || n_q_heads <= 0 || capacity <= 0 || n_ctas < 0)
    return HYQ_ERR_INVALID;
  if (n_q_heads % n_kv_heads || !g_supported(n_q_heads / n_kv_heads)) return HYQ_ERR_UNSUPPORTED;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || (lse && !al16(lse)) || !al16(ws) ||
      (reinterpret_cast<uintptr_t>(seq_len) & 3u))
    return HYQ_ERR_ALIGN;
  const int G = n_q_heads / n_kv_heads;
  const int U = batch * n_kv_heads;
  if (U > MAX_UNITS) return HYQ_ERR_UNSUPPORTED;
  const int N = resolve_ctas(n_ctas);
  if (!ws || ws_bytes < decode_ws_bytes(G, U, N)) return HYQ_ERR_WORKSPACE;
  DecodeArgs a{};
  a.B = batch; a.Hq = n_q_heads; a.Hkv = n_kv_heads; a.cap = capacity; a.W = WIN; a.vl_cap = 0;
  a.U = U; a.n_ctas = N; a.seq_len = seq_len;
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
void *g_noalloc_addr[64] = {nullptr};  // device address of the array, per device

// Host code cannot pass g_noalloc_scratch itself (that name is a host-side
// stand-in); look its device address up once per device, with the device
// current, and reuse it.
bool noalloc_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!g_noalloc_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return false;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return true;
}
}  // namespace

extern "C" hyq_status hyq_decode_noalloc(const hyq_cache *c, const void *q, void *o, float *lse,
                                         void *stream) {
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!q || !o) return HYQ_ERR_INVALID;
  if (!al16(q) || !al16(o) || (lse && !al16(lse))) return HYQ_ERR_ALIGN;
  const int G = c->n_q_heads / c->n_kv_heads;
  const int U = c->batch * c->n_kv_heads;
  const int N = resolve_ctas(0);
  if (U > NOALLOC_MAX_UNITS || N > NOALLOC_MAX_CTAS || G > NOALLOC_MAX_G) return HYQ_ERR_UNSUPPORTED;
  if (decode_ws_bytes(G, U, N) > NOALLOC_BYTES) return HYQ_ERR_UNSUPPORTED;
  void *ws = nullptr;
  if (!noalloc_address(&ws)) return HYQ_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the last call's contents: the counters must start at 0
  if (cudaMemsetAsync(ws, 0, static_cast<size_t>(U) * 4, st) != cudaSuccess) return HYQ_ERR_CUDA;
  DecodeArgs a{};
  a.B = c->batch; a.Hq = c->n_q_heads; a.Hkv = c->n_kv_heads; a.cap = c->capacity;
  a.W = c->window; a.vl_cap = c->vl_capacity; a.U = U; a.n_ctas = N;
  a.k_codes = c->k_codes; a.v_codes = c->v_codes;
  a.k_sz = static_cast<const uint8_t *>(c->k_sz); a.v_sz = static_cast<const uint8_t *>(c->v_sz);
  a.win_k = static_cast<const __half *>(c->win_k); a.win_v = static_cast<const __half *>(c->win_v);
  a.vl_k = static_cast<const __half *>(c->vl_k); a.vl_v = static_cast<const __half *>(c->vl_v);
  a.vl_count = c->vl_count; a.vl_mask = c->vl_mask; a.seq_len = c->seq_len;
  a.q = static_cast<const __half *>(q); a.o = static_cast<__half *>(o); a.lse = lse;
  a.counters = static_cast<int32_t *>(ws);
  a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (static_cast<size_t>(U) * 4 + 255) / 256 * 256);
  a.status = c->dev_status;
  return dispatch_decode<MODE_HYBRID>(G, a, st) == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

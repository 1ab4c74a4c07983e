// hyq_quant.cuh -- the library's INT4 quantizer for one 128-channel row,
// shared by the compression kernels (pack, prefill, append) and the fused
// append + decode step.
//
// Grid (fixed by the library, the pages give none; see include/hyq.h):
// asymmetric INT4 over groups of 32 channels, scale = fp16((max - min) / 15),
// zero = min (-0 stored as +0), code = clamp(rne((x - zero) / scale), 0, 15)
// with IEEE fp32 subtraction and division and no contraction into FMA.
//
// One row is handled by 16 threads; thread t owns channels 8t..8t+7, i.e.
// group g = t/4, pieces 2(t%4) and 2(t%4)+1 of the packed format.  The group
// min/max is a 4-lane shuffle reduction.
#pragma once

#include "hyq_common.cuh"

namespace hyq {

// This thread's share of one packed row: up to two 32-bit code words (at
// byte offsets off0 / off1 of the 64-byte code row) and the group's
// (scale, zero) half2 (at word g of the 16-byte scale/zero row).
struct QuantShare {
  uint32_t w0, w1, sz;
  int off0, off1, g;
  bool has_codes, has_sz;
};

// Quantize this thread's 8 channels (x = 16 bytes of fp16).  `hmask` = the
// 16 lanes that own this row.
__device__ __forceinline__ QuantShare quantize_share(uint4 x, int t, unsigned hmask, uint32_t *status) {
  float v[8];
  const __half2 *hx = reinterpret_cast<const __half2 *>(&x);
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(hx[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
  float mn = v[0], mx = v[0];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    finite = finite && isfinite(v[i]);
    mn = fminf(mn, v[i]);
    mx = fmaxf(mx, v[i]);
  }
  mn = fminf(mn, __shfl_xor_sync(hmask, mn, 1));
  mx = fmaxf(mx, __shfl_xor_sync(hmask, mx, 1));
  mn = fminf(mn, __shfl_xor_sync(hmask, mn, 2));
  mx = fmaxf(mx, __shfl_xor_sync(hmask, mx, 2));
  if (!finite) set_status(status, HYQ_DEV_NONFINITE);

  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  const __half sh = __float2half_rn(s32);
  __half zh = __float2half_rn(mn);  // exact: mn is an fp16 value
  if (mn == 0.0f) zh = __ushort_as_half(0);
  const float sf = __half2float(sh);
  const float zf = __half2float(zh);

  // code = rne(fl(d / s)), d = fl(x - zero) >= 0, clamped to [0, 15].  Only
  // the integer is needed: y = d * rcp(s) (rcp.approx, at most 1 ulp off,
  // one more rounding in the product) is within 2^-18 of fl(d / s) for
  // quotients below 16, so both round to the same integer unless y lies
  // within 2^-16 of a half-integer; there (exact ties included) the IEEE
  // quotient decides.  Quotients of 16 and more clamp to 15 either way.
  uint32_t c[8];
  float rs = 0.f;
  if (sf != 0.0f) asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rs) : "f"(sf));
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int q = 0;
    if (sf != 0.0f) {
      const float d = __fsub_rn(v[i], zf);
      float y = __fmul_rn(d, rs);
      if (fabsf(y - floorf(y) - 0.5f) <= 0x1p-16f) y = __fdiv_rn(d, sf);  // near a half-integer
      q = __float2int_rn(y);  // ties to even
      q = min(max(q, 0), 15);
    }
    c[i] = static_cast<uint32_t>(q);
  }
  // my bytes: piece p0 = 2(t%4): (j0, j1), piece p1 = p0 + 1: (j0, j1)
  const uint32_t mine = (c[0] | (c[1] << 4)) | ((c[2] | (c[3] << 4)) << 8) |
                        ((c[4] | (c[5] << 4)) << 16) | ((c[6] | (c[7] << 4)) << 24);
  // the odd group of the pair (g = 2h+1) sits 4 lanes above the even one
  const uint32_t other = __shfl_down_sync(hmask, mine, 4);
  QuantShare r;
  r.g = t >> 2;
  const int sub = t & 3;
  // word (p, h) = {g2h.j0, g2h+1.j0, g2h.j1, g2h+1.j1}
  r.has_codes = (r.g & 1) == 0;
  const int h = r.g >> 1, p0 = 2 * sub;
  r.w0 = prmt(mine, other, 0x5140u);
  r.w1 = prmt(mine, other, 0x7362u);
  r.off0 = 8 * p0 + 4 * h;
  r.off1 = 8 * (p0 + 1) + 4 * h;
  r.has_sz = sub == 0;
  r.sz = h2u(__halves2half2(sh, zh));
  return r;
}

// Quantize and store into a packed code row and its scale/zero row.
__device__ __forceinline__ void quantize_part(uint4 x, int t, unsigned hmask, uint8_t *codes_row,
                                              uint32_t *sz_row, uint32_t *status) {
  const QuantShare q = quantize_share(x, t, hmask, status);
  if (q.has_codes) {
    *reinterpret_cast<uint32_t *>(codes_row + q.off0) = q.w0;
    *reinterpret_cast<uint32_t *>(codes_row + q.off1) = q.w1;
  }
  if (q.has_sz) sz_row[q.g] = q.sz;
}

// Store this thread's code words of slot `slot` into a block record's V code
// area `vcodes` (position pairs, vcode_off): each 32-bit word goes out as its
// low and high 16 bits.
__device__ __forceinline__ void store_vcodes(const QuantShare &q, uint8_t *vcodes, int slot) {
  if (!q.has_codes) return;
  const int h = (q.off0 >> 2) & 1, p0 = q.off0 >> 3;
  uint8_t *a = vcodes + vcode_off(slot, p0, h), *b = vcodes + vcode_off(slot, p0 + 1, h);
  *reinterpret_cast<uint16_t *>(a) = static_cast<uint16_t>(q.w0);
  *reinterpret_cast<uint16_t *>(a + 4) = static_cast<uint16_t>(q.w0 >> 16);
  *reinterpret_cast<uint16_t *>(b) = static_cast<uint16_t>(q.w1);
  *reinterpret_cast<uint16_t *>(b + 4) = static_cast<uint16_t>(q.w1 >> 16);
}

// Quantize a V row into slot `slot` of a block record (codes in position
// pairs) and its scale/zero row.
__device__ __forceinline__ void quantize_part_v(uint4 x, int t, unsigned hmask, uint8_t *vcodes, int slot,
                                                uint32_t *sz_row, uint32_t *status) {
  const QuantShare q = quantize_share(x, t, hmask, status);
  store_vcodes(q, vcodes, slot);
  if (q.has_sz) sz_row[q.g] = q.sz;
}

}  // namespace hyq

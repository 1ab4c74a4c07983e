// hyq_pack.cu -- KV-cache compression kernels: hyq_pack (FP16 rows -> packed
// INT4 codes + fp16 scale/zero), hyq_append (one decode step's new token:
// the row leaving the local window is packed, the new row enters the ring)
// and hyq_vl_apply (install a vertical-line set).
//
// Method: HyQuant ("HyQuant: Hybrid-Precision Quantization for LLM
// Attention"), aifromscratch.in explainer, "How It Works" (quantized majority
// K_Q at 4 bits for keys and values, local window K_Win of the last 128
// tokens, vertical-line tokens K_VL in full precision) and "Two Operational
// Modes / Decode Stage" (the KV cache is compressed to 4 bits).  The
// quantization grid is the library's (see include/hyq.h): the pages do not
// give one.
//
// One row of 128 channels is handled by 16 threads (hyq_quant.cuh).
#include "hyq_common.cuh"
#include "hyq_quant.cuh"

namespace hyq {

__device__ __forceinline__ RecMap recmap(const hyq_cache &c) {
  return RecMap{c.block_table, c.n_kv_heads, c.capacity, c.n_pages, c.dev_status};
}
// The bitmask word of the record holding position p (nullptr: a bad
// block-table entry, already reported).
__device__ __forceinline__ uint32_t *mask_of(const hyq_cache &c, int64_t u, int64_t p) {
  const int64_t r = recmap(c).rec(u, p);
  return r < 0 ? nullptr : reinterpret_cast<uint32_t *>(c.blocks + rec_mask(r));
}

__global__ void __launch_bounds__(256) pack_kernel(const __half *__restrict__ x, int64_t n_rows,
                                                   int64_t stride,
                                                   const int64_t *__restrict__ dst_rows,
                                                   uint8_t *__restrict__ codes,
                                                   uint32_t *__restrict__ sz, uint32_t *status) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  const int lane = threadIdx.x & 31;
  const int t = lane & 15;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  if (row >= n_rows) return;  // both halves of a warp exit or stay together per row
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const uint4 xv = *reinterpret_cast<const uint4 *>(x + row * stride + 8 * t);
  const int64_t dst = dst_rows ? dst_rows[row] : row;
  quantize_part(xv, t, hmask, codes + dst * ROW_BYTES, sz + dst * (SZ_BYTES / 4), status);
}

// Prefill: one 16-thread group per (unit, position, K|V) row of the prompt.
// The rows of a pair of positions (2i, 2i + 1) come as a quad K(2i),
// K(2i + 1), V(2i), V(2i + 1), so the two V rows of a pair meet in one warp:
// each half quantizes its row, the halves swap their code words, and the
// record's paired V words (include/hyq.h) are written whole.
// Six blocks per SM (40 registers, a few bytes of spill): the kernel is
// bound by memory latency, and more rows in flight outweigh the spills
// (32K prompt, 8 KV heads: 137 -> 128 us).
__global__ void __launch_bounds__(256, 6) prefill_kernel(hyq_cache c, const __half *__restrict__ k_full,
                                                      const __half *__restrict__ v_full,
                                                      int64_t n_rows) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  const int lane = threadIdx.x & 31;
  const int t = lane & 15;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  if (row >= n_rows) return;  // n_rows is a multiple of 4: a warp's halves leave together
  const int sub = static_cast<int>(row & 3);
  const bool is_v = sub >= 2;
  const int64_t up = ((row >> 2) << 1) | (sub & 1);  // unit * capacity + position
  const int p = static_cast<int>(up % c.capacity);
  const int64_t u = up / c.capacity;
  const int b = static_cast<int>(u / c.n_kv_heads);
  const int T = c.seq_len[b];
  if (T < 0 || T > c.capacity) {  // the same for both halves (one unit)
    if (p == 0 && t == 0 && !is_v && (u % c.n_kv_heads) == 0) set_status(c.dev_status, HYQ_DEV_BADLEN);
    return;
  }
  const int W = c.window;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  if (!is_v) {
    // clear this unit's vertical-line set (the bitmask words of the records
    // holding its positions, and the count)
    if (t == 0 && p == 0) c.vl_count[u] = 0;
    if (p >= T) return;
    if (t == 0 && (p % BLK_TOK) == 0) {
      uint32_t *m = mask_of(c, u, p);
      if (m) *m = 0u;
    }
    const uint4 xv = *reinterpret_cast<const uint4 *>(k_full + up * D + 8 * t);
    if (p < T - W) {
      const int64_t rec = recmap(c).rec(u, p);
      if (rec >= 0)  // uniform over the row's 16 lanes
        quantize_part(xv, t, hmask, c.blocks + rec_kcode(rec, p),
                      reinterpret_cast<uint32_t *>(c.blocks + rec_ksz(rec, p)), c.dev_status);
      if (c.stage_rows > 0 && p >= T - W - c.stage_rows)  // staging ring: the most recent quantized rows
        *reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(c.stage_k) + (u * c.stage_rows + p % c.stage_rows) * D +
                                   8 * t) = xv;
    } else {
      *reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(c.win_k) + (u * W + p % W) * D + 8 * t) = xv;
    }
    return;
  }
  // V rows: both halves of the warp reach the exchanges below
  const bool valid = p < T, quant = p < T - W;
  const bool partner_quant = __shfl_xor_sync(0xffffffffu, quant ? 1 : 0, 16) != 0;
  // the pair's record, looked up at its even position (below T whenever a
  // member is quantized); < 0: a bad block-table entry, the writes are skipped
  const int64_t rec = (quant || partner_quant) ? recmap(c).rec(u, p & ~1) : -1;
  uint4 xv = make_uint4(0, 0, 0, 0);
  if (valid) xv = *reinterpret_cast<const uint4 *>(v_full + up * D + 8 * t);
  uint32_t w0 = 0, w1 = 0;
  if (quant) {
    const QuantShare q = quantize_share(xv, t, hmask, c.dev_status);
    w0 = q.w0;
    w1 = q.w1;
    if (rec >= 0 && q.has_sz) reinterpret_cast<uint32_t *>(c.blocks + rec_vsz(rec, p))[q.g] = q.sz;
    if (c.stage_rows > 0 && p >= T - W - c.stage_rows)  // staging ring: the most recent quantized rows
      *reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(c.stage_v) + (u * c.stage_rows + p % c.stage_rows) * D +
                                 8 * t) = xv;
  } else if (valid) {
    *reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(c.win_v) + (u * W + p % W) * D + 8 * t) = xv;
  }
  const uint32_t o0 = __shfl_xor_sync(0xffffffffu, w0, 16), o1 = __shfl_xor_sync(0xffffffffu, w1, 16);
  // Threads of the even groups hold code words (quantize_share): pieces
  // 2 (t % 4) and 2 (t % 4) + 1, word t / 8.  The pair's first member writes
  // the words of low halves, the second the words of high halves; a member
  // that is not quantized (in the window, or past T) contributes zeros.
  if (rec >= 0 && ((t >> 2) & 1) == 0) {
    const int slot = p % BLK_TOK, pair = slot >> 1, h = t >> 3, p0 = 2 * (t & 3);
    const bool first = ((slot & 1) ^ ((slot >> 2) & 1)) == 0;
    uint8_t *vc = c.blocks + rec_vcodes(rec) + pair * 128 + 8 * h + (first ? 0 : 4);
    const uint32_t a0 = first ? (w0 & 0xFFFFu) | (o0 << 16) : (o0 >> 16) | (w0 & 0xFFFF0000u);
    const uint32_t a1 = first ? (w1 & 0xFFFFu) | (o1 << 16) : (o1 >> 16) | (w1 & 0xFFFF0000u);
    *reinterpret_cast<uint32_t *>(vc + 16 * vcode_unit(pair, p0)) = a0;
    *reinterpret_cast<uint32_t *>(vc + 16 * vcode_unit(pair, p0 + 1)) = a1;
  }
}

// One block per batch b; 16 threads per (kv head, K|V) row, then the query
// copy into the detector's ring.
__global__ void append_kernel(hyq_cache c, const __half *__restrict__ k_new,
                              const __half *__restrict__ v_new, const __half *__restrict__ q_new,
                              __half *__restrict__ q_ring, int n_q) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  const int b = blockIdx.x;
  const int T = c.seq_len[b];
  __syncthreads();  // every thread has read seq_len[b] before it changes
  if (T < 0 || T + 1 > c.capacity) {
    if (threadIdx.x == 0) set_status(c.dev_status, HYQ_DEV_BADLEN);
    return;
  }
  const int W = c.window;
  const int slot = T % W;
  const int n_rows = 2 * c.n_kv_heads;
  const int row = threadIdx.x >> 4, t = threadIdx.x & 15;
  const int lane = threadIdx.x & 31;
  if (row < n_rows) {
    const int h = row >> 1;
    const bool is_v = row & 1;
    const int64_t u = static_cast<int64_t>(b) * c.n_kv_heads + h;
    __half *win = reinterpret_cast<__half *>(is_v ? c.win_v : c.win_k) + (u * W + slot) * D;
    if (T >= W) {
      const unsigned hmask = 0xFFFFu << (lane & 16);
      const uint4 old = *reinterpret_cast<const uint4 *>(win + 8 * t);
      const int64_t p = T - W;
      const int64_t rec = recmap(c).rec(u, p);
      if (rec >= 0) {  // uniform over the row's 16 lanes
        if (is_v)
          quantize_part_v(old, t, hmask, c.blocks + rec_vcodes(rec), static_cast<int>(p % BLK_TOK),
                          reinterpret_cast<uint32_t *>(c.blocks + rec_vsz(rec, p)), c.dev_status);
        else
          quantize_part(old, t, hmask, c.blocks + rec_kcode(rec, p),
                        reinterpret_cast<uint32_t *>(c.blocks + rec_ksz(rec, p)), c.dev_status);
        // the first row quantized into a record: no position of it is a
        // vertical line yet (they lie below T - W), so its bitmask starts
        // clear, whatever the record held before
        if (!is_v && t == 0 && (p % BLK_TOK) == 0) *reinterpret_cast<uint32_t *>(c.blocks + rec_mask(rec)) = 0u;
      }
      if (c.stage_rows > 0) {  // the leaving row also enters the staging ring
        __half *st = reinterpret_cast<__half *>(is_v ? c.stage_v : c.stage_k) +
                     (u * c.stage_rows + p % c.stage_rows) * D;
        *reinterpret_cast<uint4 *>(st + 8 * t) = old;
      }
    }
    const __half *src = (is_v ? v_new : k_new) + u * D;
    *reinterpret_cast<uint4 *>(win + 8 * t) = *reinterpret_cast<const uint4 *>(src + 8 * t);
  }
  if (q_new && q_ring) {
    const int qs = T % n_q;
    for (int i = threadIdx.x; i < c.n_q_heads * 16; i += blockDim.x) {
      const int64_t hq = static_cast<int64_t>(b) * c.n_q_heads + (i >> 4);
      const int part = i & 15;
      *reinterpret_cast<uint4 *>(q_ring + (hq * n_q + qs) * D + 8 * part) =
          *reinterpret_cast<const uint4 *>(q_new + hq * D + 8 * part);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) c.seq_len[b] = T + 1;
}

// ---------------------------------------------------------------- VL apply
// One block per unit.  Shared memory: int32 [2][vl_capacity] (cache mode:
// old slot and position of every kept row, in new-slot order).
__device__ __forceinline__ int find_sorted(const int32_t *a, int n, int32_t key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (a[mid] < key) lo = mid + 1; else hi = mid;
  }
  return (lo < n && a[lo] == key) ? lo : -1;
}

// Prefill mode, step 1 (one block per unit): validate the new list, clear
// the unit's bitmask, publish the count (0 when the list is invalid, which
// turns step 2 into a no-op for the unit).
__global__ void __launch_bounds__(256) vl_reset_kernel(hyq_cache c, const int32_t *__restrict__ pos, int k) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  __shared__ int s_bad;
  const int u = blockIdx.x;
  const int T = c.seq_len[u / c.n_kv_heads];
  const int L4 = T - c.window;
  const int32_t *np = pos + static_cast<int64_t>(u) * k;
  if (threadIdx.x == 0) s_bad = (T < 0 || T > c.capacity);
  __syncthreads();
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const int p = np[i];
    if (p < 0 || p >= L4 || (i > 0 && np[i - 1] >= p)) s_bad = 1;
  }
  // the bitmask words of the records holding quantized positions [0, L4)
  for (int w = threadIdx.x; w < (max(L4, 0) + BLK_TOK - 1) / BLK_TOK; w += blockDim.x) {
    uint32_t *m = mask_of(c, u, static_cast<int64_t>(w) * BLK_TOK);
    if (m) *m = 0u;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (s_bad) set_status(c.dev_status, HYQ_DEV_BADLEN);
    c.vl_count[u] = s_bad ? 0 : k;
  }
}

// Prefill mode, step 2 (blocks of 32 rows x 16 lanes): gather the FP16 rows,
// write the position list, set the bits.
__global__ void __launch_bounds__(512) vl_gather_kernel(hyq_cache c, const int32_t *__restrict__ pos, int k,
                                                        const __half *__restrict__ k_full,
                                                        const __half *__restrict__ v_full) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  const int u = blockIdx.y;
  if (c.vl_count[u] != k) return;  // invalid list: left empty by step 1
  const int r = blockIdx.x * 32 + (threadIdx.x >> 4), part = threadIdx.x & 15;
  if (r >= k) return;
  const int p = pos[static_cast<int64_t>(u) * k + r];
  const int64_t so = (static_cast<int64_t>(u) * c.capacity + p) * D + 8 * part;
  const int64_t d = (static_cast<int64_t>(u) * c.vl_capacity + r) * D + 8 * part;
  *reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(c.vl_k) + d) = *reinterpret_cast<const uint4 *>(k_full + so);
  *reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(c.vl_v) + d) = *reinterpret_cast<const uint4 *>(v_full + so);
  if (part == 0) {
    uint32_t *m = mask_of(c, u, p);
    if (m) atomicOr(m, 1u << (p & 31));
    c.vl_pos[static_cast<int64_t>(u) * c.vl_capacity + r] = p;
  }
}

// Cache mode (one block of 1024 threads per unit): kept = new ∩ old in
// ascending order; kslot[r] = old slot of the r-th kept position, kpos[r] =
// that position.  Rows only move to lower slots (r <= kslot[r]), so the move
// is done in place, 64 rows per chunk, each chunk reading all its sources
// before writing.
__global__ void __launch_bounds__(1024) vl_recompact_kernel(hyq_cache c, const int32_t *__restrict__ pos, int k,
                                                            int32_t *n_unpromoted) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // earlier work on the stream is complete and visible
  extern __shared__ int32_t vl_list[];  // [2][vl_capacity]
  __shared__ int red[32];
  __shared__ int s_bad, s_prom;
  const int u = blockIdx.x;
  const int T = c.seq_len[u / c.n_kv_heads];
  const int L4 = T - c.window;
  const int32_t *np = pos + static_cast<int64_t>(u) * k;
  int32_t *old = c.vl_pos + static_cast<int64_t>(u) * c.vl_capacity;
  const int old_n = c.vl_count[u];
  if (threadIdx.x == 0) s_bad = (old_n < 0 || old_n > c.vl_capacity);
  __syncthreads();
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const int p = np[i];
    if (p < 0 || p >= L4 || (i > 0 && np[i - 1] >= p)) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) set_status(c.dev_status, HYQ_DEV_BADLEN);
    return;
  }
  __half *vk = reinterpret_cast<__half *>(c.vl_k);
  __half *vv = reinterpret_cast<__half *>(c.vl_v);
  const int64_t row_base = static_cast<int64_t>(u) * c.vl_capacity;
  int32_t *kslot = vl_list;
  int32_t *kpos = vl_list + c.vl_capacity;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int n_kept = 0;
  for (int base = 0; base < k; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int j = (i < k) ? find_sorted(old, old_n, np[i]) : -1;
    const bool kept = j >= 0;
    const unsigned bal = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) red[w] = __popc(bal);
    __syncthreads();
    int pre = 0, tot = 0;
    for (int q = 0; q < nw; ++q) {
      if (q < w) pre += red[q];
      tot += red[q];
    }
    pre += __popc(bal & ((1u << lane) - 1u));
    if (kept) {
      kslot[n_kept + pre] = j;
      kpos[n_kept + pre] = np[i];
    }
    n_kept += tot;
    __syncthreads();
  }
  // dropped old positions fall back to their codes
  for (int j = threadIdx.x; j < old_n; j += blockDim.x) {
    const int p = old[j];
    if (p >= 0 && p < c.capacity && find_sorted(np, k, p) < 0)
      if (uint32_t *m = mask_of(c, u, p)) atomicAnd(m, ~(1u << (p & 31)));
  }
  __syncthreads();
  // Kept rows move down to their new slots (a destination is never above its
  // source): each pass loads RM rows per 16-thread group, and all its loads
  // complete (barrier) before any of its stores, so no row is overwritten
  // before it is read.
  constexpr int RM = 2;
  const int rows = blockDim.x / 16;
  for (int base = 0; base < n_kept; base += RM * rows) {
    const int part = threadIdx.x & 15;
    uint4 rk[RM], rv[RM];
    bool act[RM];
#pragma unroll
    for (int q = 0; q < RM; ++q) {
      const int r = base + q * rows + (threadIdx.x >> 4);
      act[q] = r < n_kept && kslot[r] != r;
      rk[q] = rv[q] = make_uint4(0, 0, 0, 0);
      if (act[q]) {
        const int64_t so = (row_base + kslot[r]) * D + 8 * part;
        rk[q] = *reinterpret_cast<const uint4 *>(vk + so);
        rv[q] = *reinterpret_cast<const uint4 *>(vv + so);
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < RM; ++q) {
      if (!act[q]) continue;
      const int64_t d = (row_base + base + q * rows + (threadIdx.x >> 4)) * D + 8 * part;
      *reinterpret_cast<uint4 *>(vk + d) = rk[q];
      *reinterpret_cast<uint4 *>(vv + d) = rv[q];
    }
    __syncthreads();
  }
  // Staged promotion: the new positions newer than every kept one and still
  // in the staging ring, [T - window - stage_rows, T - window), take their
  // rows from the ring.  They are a suffix of the ascending list and go
  // after the kept rows (whose moves above are complete).
  int n_prom = 0;
  if (c.stage_rows > 0) {
    const int last_kept = (n_kept > 0) ? kpos[n_kept - 1] : -1;
    const int thr = max(last_kept + 1, L4 - c.stage_rows);
    if (threadIdx.x == 0) s_prom = 0;
    __syncthreads();
    int cnt = 0;
    for (int i = threadIdx.x; i < k; i += blockDim.x) cnt += (np[i] >= thr);
    if (cnt) atomicAdd(&s_prom, cnt);
    __syncthreads();
    n_prom = s_prom;
    const int first = k - n_prom;
    const __half *sk = reinterpret_cast<const __half *>(c.stage_k);
    const __half *sv = reinterpret_cast<const __half *>(c.stage_v);
    for (int base = 0; base < n_prom; base += rows) {
      const int r = base + (threadIdx.x >> 4), part = threadIdx.x & 15;
      if (r < n_prom) {
        const int p = np[first + r];
        const int64_t so = (static_cast<int64_t>(u) * c.stage_rows + p % c.stage_rows) * D + 8 * part;
        const int64_t d = (row_base + n_kept + r) * D + 8 * part;
        *reinterpret_cast<uint4 *>(vk + d) = *reinterpret_cast<const uint4 *>(sk + so);
        *reinterpret_cast<uint4 *>(vv + d) = *reinterpret_cast<const uint4 *>(sv + so);
        if (part == 0) {
          if (uint32_t *m = mask_of(c, u, p)) atomicOr(m, 1u << (p & 31));
          kpos[n_kept + r] = p;
        }
      }
    }
    __syncthreads();
  }
  const int n_new = n_kept + n_prom;
  for (int r = threadIdx.x; r < old_n || r < n_new; r += blockDim.x)
    old[r] = (r < n_new) ? kpos[r] : -1;
  if (threadIdx.x == 0) {
    c.vl_count[u] = n_new;
    if (n_unpromoted) atomicAdd(n_unpromoted, k - n_new);
  }
}

}  // namespace hyq

using namespace hyq;

static inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

extern "C" hyq_status hyq_check_cache(const hyq_cache *c);  // hyq_api.cu

extern "C" hyq_status hyq_pack(const void *x, int64_t n_rows, int64_t row_stride,
                               const int64_t *dst_rows, uint8_t *codes, void *sz,
                               uint32_t *dev_status, void *stream) {
  HYQ_RANGE("hyq_pack");
  if (n_rows < 0 || row_stride < D || (row_stride % 8) != 0) return HYQ_ERR_INVALID;
  if (n_rows == 0) return HYQ_OK;
  if (!x || !codes || !sz) return HYQ_ERR_INVALID;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sz) || (dst_rows && !aligned16(dst_rows)))
    return HYQ_ERR_ALIGN;
  const int64_t threads = n_rows * 16;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFll) return HYQ_ERR_INVALID;
  const cudaError_t e = launch(pack_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                                static_cast<cudaStream_t>(stream), static_cast<const __half *>(x), n_rows,
                                row_stride, dst_rows, codes, static_cast<uint32_t *>(sz), dev_status);
  return e == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

extern "C" hyq_status hyq_prefill(const hyq_cache *c, const void *k_full, const void *v_full,
                                  void *stream) {
  HYQ_RANGE("hyq_prefill");
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!k_full || !v_full) return HYQ_ERR_INVALID;
  if (!aligned16(k_full) || !aligned16(v_full)) return HYQ_ERR_ALIGN;
  const int64_t n_rows = static_cast<int64_t>(c->batch) * c->n_kv_heads * c->capacity * 2;
  const int64_t blocks = (n_rows * 16 + 255) / 256;
  if (blocks > 0x7FFFFFFFll) return HYQ_ERR_INVALID;
  const cudaError_t e = launch(prefill_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                                static_cast<cudaStream_t>(stream), *c, static_cast<const __half *>(k_full),
                                static_cast<const __half *>(v_full), n_rows);
  return e == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

extern "C" hyq_status hyq_append(const hyq_cache *c, const void *k_new, const void *v_new,
                                 const void *q_new, void *q_ring, int32_t n_q, void *stream) {
  HYQ_RANGE("hyq_append");
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (!k_new || !v_new) return HYQ_ERR_INVALID;
  if ((q_new == nullptr) != (q_ring == nullptr)) return HYQ_ERR_INVALID;
  if (q_new && (n_q < 1 || n_q > 1024)) return HYQ_ERR_INVALID;
  if (!aligned16(k_new) || !aligned16(v_new) || (q_new && (!aligned16(q_new) || !aligned16(q_ring))))
    return HYQ_ERR_ALIGN;
  if (c->n_kv_heads > 32) return HYQ_ERR_UNSUPPORTED;  // 2 rows x 16 threads per kv head
  const int threads = 32 * c->n_kv_heads < 128 ? 128 : 32 * c->n_kv_heads;
  const cudaError_t e = launch(append_kernel, dim3(c->batch), dim3(threads), 0, static_cast<cudaStream_t>(stream),
                                *c, static_cast<const __half *>(k_new), static_cast<const __half *>(v_new),
                                static_cast<const __half *>(q_new), static_cast<__half *>(q_ring), n_q);
  return e == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

extern "C" hyq_status hyq_vl_apply(const hyq_cache *c, const int32_t *pos, int32_t k,
                                   const void *k_full, const void *v_full,
                                   int32_t *n_unpromoted, void *stream) {
  HYQ_RANGE("hyq_vl_apply");
  hyq_status s = hyq_check_cache(c);
  if (s != HYQ_OK) return s;
  if (k < 0 || k > c->vl_capacity) return HYQ_ERR_INVALID;
  if (k > 0 && !pos) return HYQ_ERR_INVALID;
  if ((k_full == nullptr) != (v_full == nullptr)) return HYQ_ERR_INVALID;
  if ((pos && !aligned16(pos)) || (k_full && (!aligned16(k_full) || !aligned16(v_full))))
    return HYQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int U = c->batch * c->n_kv_heads;
  cudaError_t e = cudaSuccess;
  if (k_full) {
    e = launch(vl_reset_kernel, dim3(U), dim3(256), 0, st, *c, pos, k);
    if (e == cudaSuccess && k > 0)
      e = launch(vl_gather_kernel, dim3((k + 31) / 32, U), dim3(512), 0, st, *c, pos, k,
                 static_cast<const __half *>(k_full), static_cast<const __half *>(v_full));
  } else {
    const size_t smem = 2 * sizeof(int32_t) * static_cast<size_t>(c->vl_capacity);
    if (smem > 200 * 1024) return HYQ_ERR_UNSUPPORTED;
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
      cudaFuncSetAttribute(vl_recompact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      attr_dev = dev;
    }
    e = launch(vl_recompact_kernel, dim3(U), dim3(1024), smem, st, *c, pos, k, n_unpromoted);
  }
  return e == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

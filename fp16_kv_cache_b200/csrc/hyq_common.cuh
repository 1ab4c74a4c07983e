// hyq_common.cuh -- device helpers shared by the libhyq kernels (sm_100a).
//
// Inline PTX wrappers for the asynchronous bulk-copy engine (cp.async.bulk +
// mbarrier transaction counts), warp-level tensor-core MMA, the 8x8 b16
// register transpose, and the nibble -> fp16 subnormal view used to feed
// packed INT4 codes to the tensor cores.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <utility>

#include "../../include/hyq.h"

namespace hyq {

// Host-side NVTX range named after the entry point, open for the whole call
// (argument checks, launches).  NVTX is header-only: without a tool attached
// to the process the push and pop return at once.
struct CallRange {
  explicit CallRange(const char *name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange &) = delete;
  CallRange &operator=(const CallRange &) = delete;
};
#define HYQ_RANGE(name) const ::hyq::CallRange hyq_call_range_(name)

constexpr int D = 128;
constexpr int GROUP = 32;
constexpr int NG = 4;
constexpr int WIN = 128;
constexpr int ROW_BYTES = 64;
constexpr int SZ_BYTES = 16;
constexpr int MAX_UNITS = 4096;  // units (batch x kv heads) one launch schedules
constexpr int BLK_TOK = HYQ_BLOCK_TOKENS;
constexpr int BLK_BYTES = HYQ_BLOCK_BYTES;

// ---------------------------------------------------------------- status
__device__ __forceinline__ void set_status(uint32_t *st, uint32_t bits) {
  if (st) atomicOr(st, bits);
}

// Quantized-majority block of position p of unit u, and the byte offsets of
// that position's K/V codes and scale/zero rows inside the cache's blocks
// (contiguous layout: each unit owns capacity / 32 consecutive records).
__host__ __device__ __forceinline__ int64_t blk_base(int64_t u, int64_t p, int cap) {
  return (u * (cap / BLK_TOK) + p / BLK_TOK) * BLK_BYTES;
}

// Where the record of (unit u, position p) lives.  Contiguous layout (no
// block table): blk_base.  Paged layout: sequence b = u / Hkv maps its
// logical block p / 32 to page table[b * (cap / 32) + p / 32] of a pool of
// n_pages pages, and a page holds the records of the Hkv KV heads in order,
// so the record is page * Hkv + u % Hkv.  A table entry outside [0,
// n_pages) raises HYQ_DEV_BADLEN; reads then go to page 0 (in bounds) and
// writers skip the access (rec() < 0).
struct RecMap {
  const int32_t *table;  // nullable
  int Hkv, cap, n_pages;
  uint32_t *status;
  __device__ __forceinline__ int64_t rec(int64_t u, int64_t p) const {
    if (!table) return blk_base(u, p, cap);
    const int64_t pg = table[(u / Hkv) * (cap / BLK_TOK) + p / BLK_TOK];
    if (pg < 0 || pg >= n_pages) {
      set_status(status, HYQ_DEV_BADLEN);
      return -1;
    }
    return (pg * Hkv + u % Hkv) * BLK_BYTES;
  }
  // for reads: an invalid entry reads page 0
  __device__ __forceinline__ int64_t rec_rd(int64_t u, int64_t p) const {
    const int64_t r = rec(u, p);
    return r < 0 ? 0 : r;
  }
};
__host__ __device__ __forceinline__ int64_t rec_kcode(int64_t rec, int64_t p) { return rec + HYQ_BLK_KCODES + (p % BLK_TOK) * ROW_BYTES; }
__host__ __device__ __forceinline__ int64_t rec_ksz(int64_t rec, int64_t p) { return rec + HYQ_BLK_KSZ + (p % BLK_TOK) * SZ_BYTES; }
__host__ __device__ __forceinline__ int64_t rec_vcodes(int64_t rec) { return rec + HYQ_BLK_VCODES; }
// V codes are stored in position pairs (include/hyq.h): the byte offset,
// inside a record's V code area, of the low 16 bits of word h of piece
// `piece` of slot t; the high 16 bits are 4 bytes further.  The pair
// {2i, 2i + 1} shares each 32-bit word, in the order the decode's P.V
// operand wants: (2i, 2i + 1) when i % 4 < 2, else (2i + 1, 2i).  Pair i
// keeps piece p in its 16-byte unit p xor 2 (i mod 4), so the 8 lanes of a
// 16-byte shared-memory load phase (pieces r, r + 1 of four pairs) fall in
// 8 different bank groups.
__host__ __device__ __forceinline__ int vcode_unit(int pair, int piece) { return piece ^ ((pair & 3) << 1); }
__host__ __device__ __forceinline__ int vcode_off(int t, int piece, int h) {
  return (t >> 1) * 128 + vcode_unit(t >> 1, piece) * 16 + h * 8 + (((t & 1) ^ ((t >> 2) & 1)) << 1);
}
__host__ __device__ __forceinline__ int64_t rec_vsz(int64_t rec, int64_t p) { return rec + HYQ_BLK_VSZ + (p % BLK_TOK) * SZ_BYTES; }
__host__ __device__ __forceinline__ int64_t rec_mask(int64_t rec) { return rec + HYQ_BLK_MASK; }

// ---------------------------------------------------------------- smem
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Complete the current phase of a barrier armed for one arrival without
// waiting for any bytes (a copy that is not issued).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(bar) : "memory");
}

// Bounded wait on an mbarrier phase.  Gives up after `limit_ns` of wall time
// (or as soon as *abort is raised by another warp), raising *abort and
// HYQ_DEV_TIMEOUT in the status word.  Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int *abort, uint32_t *status,
                                                  uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((it & 15u) == 15u && global_ns() - t0 > limit_ns) {
      *abort = 1;
      set_status(status, HYQ_DEV_TIMEOUT);
      return false;
    }
  }
}

// Wait (bounded by time only) for copies already issued to land, used when a
// block gives up: shared memory must not be released with copies in flight.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return;
  }
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// 1-D bulk copy global -> shared, completing `bytes` on the mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// ---------------------------------------------------------------- tensor core
// D = A(16x16, row) * B(16x8, col) + D; fp16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 matrix of 16-bit elements held one row per 4 lanes.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// ---------------------------------------------------------------- bit tricks
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// Nibbles in bits 0-3 / 4-7 and 16-19 / 20-23 of w as a half2 of fp16
// subnormals, one AND each: a half whose exponent field is zero and whose
// fraction is f has the value f * 2^-24 exactly (IEEE 754 binary16), so
// bits 0-3 give n * 2^-24 and bits 4-7 give 16 n * 2^-24.  The tensor core
// multiplies these exactly; the caller undoes the power-of-two factors in
// fp32.
__device__ __forceinline__ uint32_t code_lo(uint32_t w) { return w & 0x000F000Fu; }
__device__ __forceinline__ uint32_t code_hi(uint32_t w) { return w & 0x00F000F0u; }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  return h2u(__floats2half2_rn(lo, hi));
}

// ---------------------------------------------------------------- launches
// Programmatic dependent launch: every library kernel is launched with
// programmatic stream serialization, so it may be scheduled while the
// previous kernel on the stream is still running.  Each kernel calls
// pdl_trigger() early (the next kernel may then be scheduled once every
// block of this one has started) and pdl_wait() before it touches global
// memory: the wait returns when the previous grid has completed and its
// writes are visible, so stream order is kept.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
static inline cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace hyq

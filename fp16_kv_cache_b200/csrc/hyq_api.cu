// hyq_api.cu -- host-side helpers of the libhyq C ABI: descriptor
// validation, status strings, version, cached SM count, and the copy of a
// step's inputs and outputs between pinned host memory and the device.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/hyq.h"
#include "hyq_common.cuh"

static inline bool al16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

extern "C" hyq_status hyq_check_cache(const hyq_cache *c) {
  if (!c) return HYQ_ERR_INVALID;
  if (c->head_dim != HYQ_HEAD_DIM || c->group != HYQ_GROUP || c->window != HYQ_WINDOW)
    return HYQ_ERR_UNSUPPORTED;
  if (c->batch <= 0 || c->n_kv_heads <= 0 || c->n_q_heads <= 0) return HYQ_ERR_INVALID;
  if (c->n_q_heads % c->n_kv_heads) return HYQ_ERR_INVALID;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return HYQ_ERR_UNSUPPORTED;
  if (c->capacity <= 0 || (c->capacity % 128) != 0) return HYQ_ERR_INVALID;
  if (c->vl_capacity <= 0) return HYQ_ERR_INVALID;
  const void *ptrs[] = {c->blocks, c->win_k,  c->win_v,    c->vl_k,
                        c->vl_v,   c->vl_pos, c->vl_count, c->seq_len};
  for (const void *p : ptrs) {
    if (!p) return HYQ_ERR_INVALID;
    if (!al16(p)) return HYQ_ERR_ALIGN;
  }
  if (c->dev_status && (reinterpret_cast<uintptr_t>(c->dev_status) & 3u)) return HYQ_ERR_ALIGN;
  if (c->block_table) {
    if (c->n_pages < 1) return HYQ_ERR_INVALID;
    if (reinterpret_cast<uintptr_t>(c->block_table) & 3u) return HYQ_ERR_ALIGN;
  }
  if (c->stage_rows < 0 || c->stage_rows > 1024) return HYQ_ERR_INVALID;
  if (c->stage_rows > 0) {
    if (!c->stage_k || !c->stage_v) return HYQ_ERR_INVALID;
    if (!al16(c->stage_k) || !al16(c->stage_v)) return HYQ_ERR_ALIGN;
  }
  return HYQ_OK;
}

extern "C" int32_t hyq_sm_count(void) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

extern "C" const char *hyq_status_string(hyq_status s) {
  switch (s) {
    case HYQ_OK: return "ok";
    case HYQ_ERR_INVALID: return "invalid argument";
    case HYQ_ERR_UNSUPPORTED: return "unsupported shape";
    case HYQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case HYQ_ERR_WORKSPACE: return "workspace missing or too small";
    case HYQ_ERR_CUDA: return "CUDA launch error";
    default: return "unknown status";
  }
}

extern "C" int32_t hyq_version(void) { return 100; }

// ---------------------------------------------------------------- hyq_copy
// A small transfer as a kernel: 16-byte loads and stores through the
// addresses the device sees (device memory, or pinned host memory mapped
// into the device's address space).  Unlike a copy-engine transfer it keeps
// the programmatic launch overlap with the kernels around it.
namespace hyq {
__global__ void __launch_bounds__(256) io_copy_kernel(uint4 *dst, const uint4 *src, int64_t n16) {
  pdl_trigger();  // the next kernel may be scheduled
  pdl_wait();     // the previous kernel's reads of dst and writes of src are complete
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * 256)
    dst[i] = src[i];
}
}  // namespace hyq

namespace {

// The address the current device may dereference for p, or nullptr: device
// and managed memory as they are; page-locked host memory only where it is
// mapped for the device; unregistered host memory never.
void *device_view(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return const_cast<void *>(p);
  if (at.type == cudaMemoryTypeHost) return at.devicePointer;
  return nullptr;
}
}  // namespace

extern "C" hyq_status hyq_copy(void *dst, const void *src, size_t bytes, void *stream) {
  HYQ_RANGE("hyq_copy");
  if (!dst || !src) return HYQ_ERR_INVALID;
  if (bytes == 0) return HYQ_OK;
  if (bytes & 15u) return HYQ_ERR_INVALID;
  if (!al16(dst) || !al16(src)) return HYQ_ERR_ALIGN;
  void *d = device_view(dst);
  const void *s = device_view(src);
  if (!d || !s) return HYQ_ERR_INVALID;
  const int64_t n16 = static_cast<int64_t>(bytes / 16);
  const int64_t cap = 4 * static_cast<int64_t>(hyq_sm_count());
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>((n16 + 255) / 256, cap));
  const cudaError_t e = hyq::launch(hyq::io_copy_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream),
                                    static_cast<uint4 *>(d), static_cast<const uint4 *>(s), n16);
  return e == cudaSuccess ? HYQ_OK : HYQ_ERR_CUDA;
}

// hyq_api.cu -- host-side helpers of the libhyq C ABI: descriptor
// validation, status strings, version, cached SM count.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hyq.h"

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

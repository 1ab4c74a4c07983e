/*
 * hyq_debug.h -- extra entry point of the debug build of the library,
 * libhyq_debug.so (the sources of libhyq.so compiled with -DHYQ_DEBUG).
 * The paper has no counterpart: this is test support for the library's
 * failure handling.
 *
 * The debug build exports every entry point of hyq.h with the same
 * behaviour, plus:
 *   - device-side index checks in the decode kernels: the block's share of
 *     the split, each tile's source rows (a quantized block below capacity,
 *     vertical-line rows below vl_capacity, window rows below the window),
 *     the partial records merged and the row leaving the window.  A failed
 *     check ORs HYQ_DEV_OOB into the cache's dev_status and skips the access
 *     (no trap); the outputs are then undefined.
 *   - the entry point below, which sets how long the decode kernels' tile
 *     waits may take before they give up with HYQ_DEV_TIMEOUT, and can make
 *     them wait on a barrier that nothing completes (a test of the bounded
 *     waits that faults and hangs nothing).
 */
#ifndef HYQ_DEBUG_H
#define HYQ_DEBUG_H

#include <stdint.h>

#include "hyq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * hyq_debug_set_wait -- the bounded waits of the decode kernels (hyq_decode,
 * hyq_decode_step, hyq_decode_vl_only, hyq_decode_noalloc, hyq_decode_fp16)
 * on the current device.
 *   limit_ns          wall-time limit of each wait for a tile's bulk copy,
 *                     1 us .. 10 s (default 2 s); else HYQ_ERR_INVALID
 *   stall_first_wait  nonzero: every warp's first tile wait waits instead on
 *                     a barrier that nothing completes, so it runs out after
 *                     limit_ns.  The warp then raises HYQ_DEV_TIMEOUT, stops
 *                     issuing copies, lets the copies already in flight land
 *                     (bounded), the block finishes its merges, and the
 *                     launch returns with undefined outputs.  0: normal waits.
 * Synchronous (copies to device variables); HYQ_ERR_CUDA when one fails.
 */
hyq_status hyq_debug_set_wait(uint64_t limit_ns, int32_t stall_first_wait);

#ifdef __cplusplus
}
#endif
#endif /* HYQ_DEBUG_H */

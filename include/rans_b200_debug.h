/*
 * rans_b200_debug.h -- test hooks of librans_b200 (not needed to code).
 *
 * They exercise the library's device-side failure handling without faulting
 * the GPU; the tests call them through the same C ABI as the coders.
 */
#ifndef RANS_B200_DEBUG_H
#define RANS_B200_DEBUG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Runs the bounded wait of the shared-memory table staging (an mbarrier
 * try-wait with a suspend hint, limited to `limit` tries) on a barrier that
 * expects 16 bytes no copy will deliver, so the wait gives up: the kernel
 * records RANS_ERR_TIMEOUT in the status word of `workspace` (device, >= 256
 * bytes, 256-byte aligned; read it with rans_get_status) and returns,
 * leaving the context usable.  limit must be in [1, 2^21].  Asynchronous.
 */
int rans_debug_wait_timeout(void *workspace, uint32_t limit, void *stream);

#ifdef __cplusplus
}
#endif

#endif

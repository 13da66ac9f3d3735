/*
 * ssa_debug.h - test hooks of the block-sparse attention library.
 *
 * This entry point exists so that a test can check, on the GPU, the bounded
 * waits of the prefill attention kernel in isolation.  They are not part of the method
 * the pages describe.  Same conventions as ssa.h (device pointers, caller's
 * stream, host-side argument checks).
 */
#ifndef SSA_DEBUG_H
#define SSA_DEBUG_H

#include "ssa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Launches one CTA that waits on an mbarrier nothing will arrive on, with the
 * attention kernel's bounded wait cut to `limit_us` microseconds (1..1000000).
 * The wait expires, the kernel records SSA_ERR_TIMEOUT in the device error
 * word and returns; read it with ssa_device_error.  No fault, no hang.
 */
ssa_status ssa_debug_wait_timeout(int limit_us, ssa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SSA_DEBUG_H */

/*
 * ple_debug.h -- test and tuning hooks of libple, beside the C ABI of ple.h.
 *
 * Not part of the lookup itself (the pages have no counterpart): these calls
 * let a test drive the library's failure paths from the host without
 * faulting, trapping or hanging a GPU.
 */
#ifndef PLE_DEBUG_H_
#define PLE_DEBUG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Set the limit, in nanoseconds, of every bounded wait between the blocks
 * of one kernel (the radix sort's look-back waits of ple_grad_scatter,
 * ple_grad_prepare, ple_grad_scatter_cache, ple_grad_scatter_noalloc and
 * ple_prefetch) for the calls launched from now on, in this process, on
 * every device; returns the previous limit.  A wait that passes its limit
 * raises the async PLE_ERR_TIMEOUT and ends the call's sort: the gradient
 * is then not applied (table_grad and cache_grad are left as they were) and
 * a prefetch reports zero distinct rows, with every memory access still
 * inside the caller's buffers.  0 makes every wait that does not succeed
 * at its first poll give up (used by the tests to reach that path).  Host
 * only; thread-safe.  The default is ple_debug_default_wait_limit_ns(). */
uint64_t ple_debug_set_wait_limit_ns(uint64_t ns);

/* The library's default wait limit (100 ms). */
uint64_t ple_debug_default_wait_limit_ns(void);

#ifdef __cplusplus
}
#endif

#endif /* PLE_DEBUG_H_ */

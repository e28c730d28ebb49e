/*
 * pa_test.h — test hooks of the paged-attention library, exported only by
 * libpa_test.so (the library compiled with PA_TEST_HOOKS defined); the
 * product library libpa.so has none of them.  They exist so that tests can
 * make a bounded wait run out on purpose and check that the kernels give up,
 * report PA_DEVERR_TIMEOUT and leave the GPU context usable, without a fault
 * or a hang.  The pages have no counterpart to them.
 */
#ifndef PA_TEST_H_
#define PA_TEST_H_

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * pa_test_set_hooks — set the limit of every bounded wait of the decode
 * kernels (nanoseconds, > 0; the product value is 1 s) and the skip switch:
 * while skip_first_copy is non-zero, the first warp of the decode thread
 * block of (sequence 0, kv head 0, partition 0) never issues the copies of
 * its first ring stage, so its wait on that stage runs out after the limit;
 * the block then waits (bounded) for its other copies, flags
 * PA_DEVERR_TIMEOUT and ends (a split partition is recorded as empty).
 * Synchronous (cudaMemcpyToSymbol on the current device).
 */
pa_status pa_test_set_hooks(int64_t wait_limit_ns, int skip_first_copy);

/*
 * pa_test_wait_timeout — one warp waits, with limit limit_ns, on an mbarrier
 * that nothing completes (no copy is issued); it then flags
 * PA_DEVERR_TIMEOUT and writes the time it waited (ns) to *elapsed_ns
 * (device int64, 8-byte aligned).  Asynchronous on `stream`.
 */
pa_status pa_test_wait_timeout(int64_t limit_ns, int64_t* elapsed_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_TEST_H_ */

/*
 * bitlinear_test_hooks.h -- one extra entry point that exists only in the
 * test build of the library (libbitlinear_testhooks.so, compiled from the
 * same sources with -DBITLINEAR_TEST_HOOKS).  The product library does not
 * export it.  The pages have no counterpart: it serves the failure-handling
 * convention of bitlinear.h (a kernel that gives up on a bounded wait writes
 * a code to the device status word instead of trapping).
 */
#ifndef BITLINEAR_TEST_HOOKS_H_
#define BITLINEAR_TEST_HOOKS_H_

#include <stdint.h>

#include "bitlinear.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Sets, on the current device, the limit of every bounded wait in the
 * kernels (nanoseconds of %globaltimer; the product value is one second) and
 * a number of bytes added to the copy count that the M = 1 decode GEMVs
 * expect on their weight barrier.  With extra_tx_bytes > 0 every issued copy
 * still lands in shared memory but the barrier never completes, so each CTA
 * gives up after wait_limit_ns, records BITLINEAR status 1 (or 5 when the
 * bounded drain wait also runs out), writes no output and exits.  Pass
 * (1000000000, 0) to restore the product behaviour.  Synchronises the device
 * before and after.  Errors: DEVICE, CUDA. */
bitlinear_status bitlinear_test_set_wait_fault(uint64_t wait_limit_ns, uint32_t extra_tx_bytes);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_TEST_HOOKS_H_ */

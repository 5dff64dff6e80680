/*
 * bitlinear_test_hooks.h -- two extra entry points that exist only in the
 * test build of the library (libbitlinear_testhooks.so, compiled from the
 * same sources with -DBITLINEAR_TEST_HOOKS).  The product library does not
 * export them.  The pages have no counterpart: the first serves the
 * failure-handling convention of bitlinear.h (a kernel that gives up on a
 * bounded wait writes a code to the device status word instead of trapping),
 * the second reads the phase stamps the test build's kernels record
 * (python -m ternary_weight_linear_fwd_b200.timeline prints them).
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

/* Phase timeline of the test build.  At its end, each CTA of the dense
 * decode GEMV (kind 1) and of the pair GEMM (kind 2) appends one record of
 * 10 uint64 to a ring of 131072 records in device memory: kind; launch facts
 * (K or M << 32 | blockIdx.x << 16 | gridDim.x); eight %globaltimer stamps
 * in ns (0 where a phase was not reached).  Decode GEMV, thread 0: entry,
 * past the dependency wait, x quantised, weights landed, contracted, stored.
 * Pair GEMM: entry, set-up done, producer past the dependency wait, first
 * stage landed, first tile's MMAs issued, first accumulator ready, last
 * epilogue done, end.  Synchronises the device, copies min(records written,
 * max_records, 131072) records oldest slot first into records (host memory;
 * NULL or max_records <= 0 copies none), clears the ring and returns the
 * number written since the last call (which may exceed the ring: the ring
 * then holds the newest, wrapped), or -1 on a CUDA error. */
int32_t bitlinear_test_timeline(uint64_t* records, int32_t max_records);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_TEST_HOOKS_H_ */

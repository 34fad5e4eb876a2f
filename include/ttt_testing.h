/*
 * ttt_testing.h — host-side fault injection of the TTT-E2E library, for tests.
 *
 * The library's failure paths (a device allocation that fails, a bounded device
 * wait that runs out) must be exercised without faulting, trapping or hanging a
 * GPU. These hooks make the failure on the host instead: an allocation request
 * that the library's single allocation routine refuses, or an error code written
 * into a device status word while no kernel is running. Production code never
 * calls them. They have no counterpart on the pages; they test this library's
 * own error contract (include/ttt.h, "Conventions for every entry point").
 */
#ifndef TTT_TESTING_H
#define TTT_TESTING_H

#include <stdint.h>

#include "ttt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Make the library's n-th device allocation request from now fail as if the
 * device were out of memory (n = 0: the next request). n < 0 cancels a pending
 * failure. Process-wide. Every device allocation of the library (handle state,
 * call buffers, the weight staging buffer) goes through the one routine this
 * controls; the per-kernel entry points of ttt_kernels.h allocate nothing. */
void ttt_test_fail_allocation(int64_t n);

/* Device allocations the library has made successfully since the process
 * loaded it (process-wide count; frees do not decrease it). */
int64_t ttt_test_allocation_count(void);

/* Write `code` (a nonzero device status, e.g. 1 = a wait for a full pipeline
 * stage ran out) into the handle's device status word after synchronising its
 * stream. The next call that synchronises reports TTT_ERR_TIMEOUT and poisons
 * the handle, exactly as after a real expired wait. Returns TTT_OK, or
 * TTT_ERR_INVALID_ARG for a NULL handle, or TTT_ERR_CUDA. */
int ttt_test_set_device_status(ttt_handle* h, int32_t code);

/* Same for the status word of the per-kernel entry points on the current
 * device (synchronises the device first): the next ttt_k_status() returns
 * TTT_ERR_TIMEOUT and clears it. */
int ttt_k_test_set_status(int32_t code);

#ifdef __cplusplus
}
#endif

#endif /* TTT_TESTING_H */

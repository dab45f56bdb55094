/*
 * ot_sinkhorn_testing.h -- failure-injection hooks of the B200 Sinkhorn
 * library (libot_sinkhorn.so), for tests of its error paths. Not for
 * production use: each hook changes process-wide behaviour until it is
 * switched off again. The pages have no counterpart; these calls exist so
 * that the library's failure handling can be exercised without faulting,
 * trapping or hanging a GPU.
 */
#ifndef OT_SINKHORN_TESTING_H
#define OT_SINKHORN_TESTING_H

#include "ot_sinkhorn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The device-workspace allocation that follows `after` more successful ones
 * fails as cudaMalloc does when device memory runs out, so the call that asked
 * for it returns OT_ERR_OOM (and releases what it had taken). The hook fires
 * once; after < 0 switches it off. */
OT_API void ot_testing_fail_device_allocs(int after);

/* Makes one bounded device wait give up, so that the call reports the timeout
 * as OT_ERR_CUDA and leaves the device usable:
 *  mode 1: in the device-resident loop kernel (d <= 3, small problems) block 0
 *          returns before its first grid-barrier arrival, and the barrier's
 *          time limit is 2 ms instead of 10 s; the other blocks give up there.
 *  mode 2: in the tensor-core half-step (16 <= d <= 64) block 0's producer
 *          skips the load of its first column chunk, and every mbarrier wait
 *          gives up after 2^12 polls instead of 2^22; that block records the
 *          timeout, drains what it issued, frees its tensor memory and returns.
 *  mode 0: off (the default).
 * The mode is read when a solve builds its launches. */
OT_API void ot_testing_wait_fault(int mode);

#ifdef __cplusplus
}
#endif
#endif /* OT_SINKHORN_TESTING_H */

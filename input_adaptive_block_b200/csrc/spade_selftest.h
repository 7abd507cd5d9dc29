/*
 * spade_selftest.h -- entry points of libspade.so that exist for its tests,
 * not for users of the method (so they are not part of include/spade.h).
 */
#ifndef SPADE_SELFTEST_H_
#define SPADE_SELFTEST_H_

#include "spade.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Runs a kernel whose single wait can never be satisfied, bounded by
 * timeout_ns (1 .. 10^10); afterwards spade_last_device_status() must read
 * SPADE_ERR_TIMEOUT.  Exercises the bounded-wait error path of the kernels
 * without faulting or hanging the GPU. */
spade_status spade_selftest_bounded_wait(int64_t timeout_ns, spade_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SPADE_SELFTEST_H_ */

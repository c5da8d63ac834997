/*
 * prox_testing.h -- test-only hook of libprox (not part of the product API).
 *
 * prox_test_set_wait: sets the wall-clock bound, in microseconds, of every
 * bounded device-side wait (0 restores the default of 2 s) and, when
 * skip_position >= 0, makes the Stage-2
 * producer of CTA 0 never fill that channel position of its share, so that a
 * test can drive the consumers' bounded wait to its limit and then read
 * PROX_ETIMEOUT from prox_last_device_status. Nothing faults: the kernel
 * records the timeout in the workspace status word and returns. Host-side
 * state, affects launches made after the call; not thread-safe.
 */
#ifndef PROX_TESTING_H
#define PROX_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

void prox_test_set_wait(uint32_t wait_us, int skip_position);

#ifdef __cplusplus
}
#endif

#endif /* PROX_TESTING_H */

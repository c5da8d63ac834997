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

/*
 * prox_test_set_stamps: measurement hook. While `slots` is non-NULL, every
 * CUDA-core forward pass launched (or captured into a CUDA graph) records
 * %globaltimer phase stamps of its two kernels into slots[0..15], device
 * memory owned by the caller: each slot is the minimum or the maximum over
 * the kernel's CTAs of the time one phase began or ended (Stage 1: entry,
 * past the wait for the previous kernel, stream start, stream end, partials
 * summed, end; Stage 2: entry, past the wait for Stage 1, channel list
 * ready, first stage full, last channel accumulated, end). The caller sets
 * the minimum slots (0, 1, 8, 9, 12) to all ones and the others to zero
 * before the pass runs. NULL turns stamping off. The stamps are a few
 * atomics per CTA; the results of the pass are unchanged. Host-side state,
 * affects launches made after the call; not thread-safe.
 */
void prox_test_set_stamps(unsigned long long *slots);

/*
 * prox_test_set_skip: makes one arrival in CTA 0 of a tensor-core kernel
 * never happen, so that the bounded wait on it runs out (use with a short
 * bound from prox_test_set_wait). `where`:
 *   1  Stage 1 on the tensor cores: for passes of 1-4 tokens, warp 0 never
 *      signals K step `position` ready (status bit 4); for passes of 8 tokens,
 *      the MMA thread never signals group `position` done (status bit 5);
 *   3  the tensor-core Stage 2: the up/gate loaders never complete their
 *      step `position` (status bit 5);
 *   0  off.
 * Nothing faults: the kernel records the timeout in the status word, skips
 * the rest of its MMAs, waits (with the default bound) for those already
 * issued, frees its tensor memory and returns. Host-side state, affects
 * launches made after the call; not thread-safe.
 */
void prox_test_set_skip(int where, int position);

#ifdef __cplusplus
}
#endif

#endif /* PROX_TESTING_H */

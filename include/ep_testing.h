/*
 * ep_testing.h -- failure-detection knob of libep_b200.so, for tests.
 *
 * Every device-side wait in the library is bounded: a wait for a TMA copy
 * (ep_dispatch, ep_route_dispatch) or for the other blocks of a grid
 * (ep_route_dispatch) polls at most a fixed number of times, then gives up,
 * ORs EP_DEV_TIMEOUT into the call's dev_status word and returns, leaving
 * that call's output incomplete instead of hanging the GPU.  The paper has
 * no counterpart of this entry point: it exists so that a test can make such
 * a wait give up on purpose, on a healthy GPU, and check that the error is
 * reported and that the next call works.
 */
#ifndef EP_B200_TESTING_H
#define EP_B200_TESTING_H

#include "ep.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sets the number of polls every bounded wait makes in launches enqueued
 * after this call, process-wide and for every device: polls = 0 makes each
 * such wait give up at once (the last block to reach a grid barrier still
 * passes it, since it waits for nobody); polls < 0 restores the default
 * (2^22).  Waits that drain copies still in flight after a give-up always
 * use the default, so shared memory is never released under a pending copy.
 * Returns EP_ERR_INVALID for polls >= 2^32, else EP_OK.  Not for production
 * use: a limit that is too small makes healthy calls fail.
 */
ep_status ep_testing_set_wait_limit(long long polls);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_TESTING_H */

/*
 * la_testing.h — testing hook of the B200 causal linear-attention library.
 *
 * The pages describe no counterpart: this entry point exists so that a test can
 * exercise the failure-detection path of the kernels on a GPU without faulting
 * or hanging it.
 *
 * Every wait inside the library's kernels (an mbarrier phase: a copy landing,
 * an MMA finishing, another warp group's hand-off) is bounded.  A wait that runs
 * out raises the timeout bit of the device error word (la_check_device then
 * returns LA_ERR_TIMEOUT); the CTA stops issuing work, lets every copy and MMA
 * it has in flight finish, releases its tensor memory and exits, so the context
 * stays usable.  The default limit is about one second of clock cycles, which
 * no correct call comes near, so without this hook the path cannot be reached.
 */
#ifndef LA_TESTING_H_
#define LA_TESTING_H_

#include <stdint.h>

#include "la.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sets the limit, in SM clock cycles, of the ordinary waits of kernels launched
 * afterwards on the CURRENT device; `cycles` <= 0 restores the default
 * (2e9 cycles).  `previous` (may be NULL) receives the limit in force before.
 * The waits that guard the release of tensor memory and the exit of a CTA with
 * copies in flight always keep the default, so a short limit ends calls early
 * with LA_ERR_TIMEOUT but never lets a CTA exit with work outstanding.
 * Synchronous with respect to the device (a symbol copy); do not call it while
 * kernels of the library are running, and restore the default before any call
 * whose results matter.  Returns LA_OK or LA_ERR_CUDA.
 */
la_status la_testing_set_wait_limit(int64_t cycles, int64_t *previous);

#ifdef __cplusplus
}
#endif

#endif /* LA_TESTING_H_ */

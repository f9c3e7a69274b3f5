/*
 * kq_debug.h -- extra entry points of the KQ_DEBUG build of the library
 * (libkq_debug.so, built beside libkq.so from the same sources).
 *
 * The KQ_DEBUG build differs from the release build in two ways:
 *   * Device bounds checks: every index a kernel takes from data -- a
 *     position or pair id of the expert grouping, an entry of the
 *     tensor-core tile list -- is checked before use.  A value out of range
 *     sets the error word (kq_device_status then returns
 *     KQ_ERR_DEVICE_BOUNDS) and the kernel skips the store or reads a row
 *     that exists instead; it never traps.
 *   * Short bounded waits: each mbarrier wait gives up after
 *     kq_debug_spin_limit() rounds (milliseconds, against seconds in the
 *     release build) and sets KQ_ERR_DEVICE_TIMEOUT.
 * Every call of kq.h behaves as in the release build otherwise.  The
 * failure-detection pattern this follows: mlx-kquant bindings.cpp
 * `shared_event_wait(timeout_ms)`, a wait that returns False when its limit
 * runs out instead of blocking; Ternary Bonsai's `SAFE` build, which clamps
 * illegal inputs instead of faulting.
 */
#ifndef KQ_DEBUG_H
#define KQ_DEBUG_H

#include "kq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * kq_debug_wait_timeout -- make one bounded wait run out.  Launches one warp
 * on `stream` that waits on an mbarrier whose phase cannot complete (it
 * expects two arrivals and gets one), with the library's own wait loop:
 * mode 0 the suspending try_wait loop, mode 1 the test-and-sleep loop.
 * The wait gives up after kq_debug_spin_limit() rounds and sets the error
 * word; the kernel then returns, so the context stays usable.  Returns
 * KQ_OK once launched (the next kq_device_status returns
 * KQ_ERR_DEVICE_TIMEOUT), KQ_ERR_ARG for another mode, KQ_ERR_UNSUPPORTED
 * off sm_100.
 */
KQ_API int kq_debug_wait_timeout(int mode, void *stream);

/* Rounds of one bounded wait in this build (KQ_SPIN_LIMIT). */
KQ_API int kq_debug_spin_limit(void);

#ifdef __cplusplus
}
#endif

#endif /* KQ_DEBUG_H */

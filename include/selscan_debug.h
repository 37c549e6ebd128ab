/*
 * selscan_debug.h -- test hooks of libselscan.  Not needed by normal
 * callers; they exist so that the failure paths of the device-side bounded
 * waits can be exercised without faulting or hanging a GPU.
 */
#ifndef SELSCAN_DEBUG_H
#define SELSCAN_DEBUG_H

#include "selscan.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Withhold the carry flag of work unit `unit` in subsequent selscan_fwd
 * calls (-1 switches the hook off).  The unit that waits for that carry
 * gives up after its time limit (SELSCAN_WAIT_TIMEOUT_MS, default 2000 ms),
 * continues from a zero state and records the event; the next
 * selscan_check() returns SELSCAN_ERR_TIMEOUT.  Work units are numbered
 * segment-major: unit = segment * tiles + tile.
 */
SELSCAN_API void selscan_debug_withhold_carry(int unit);

/*
 * Choose how the fast bf16 diagonal scan links the segments of a channel
 * tile in subsequent selscan_fwd calls: 0 = one pass with carries chained
 * from segment to segment; 1 = two passes (every segment's end state from
 * zero and its sum of step sizes, then the output pass folding those into
 * each segment's initial state); -1 (default) = the library's choice (two
 * passes when there are at most half as many tiles as SMs).  Both forms
 * compute the same recurrence; the hook lets tests cover both on the same
 * inputs.  Single-segment launches are unaffected.
 */
SELSCAN_API void selscan_debug_diag_mode(int mode);

/*
 * Number of time segments per channel tile in subsequent selscan_bwd calls
 * (0, the default, = the library's choice: as many as fill one wave of
 * resident warps, with at least 32 checkpoint chunks each).  Capped at the
 * number of checkpoint chunks.  Every segment count computes the same
 * gradients; the hook lets tests cover the segment folds on small inputs
 * and lets the choice be timed.
 */
SELSCAN_API void selscan_debug_bwd_segments(int segs);

/*
 * Number of time segments per channel tile in subsequent selscan_fwd calls
 * (0, the default, = the library's choice).  Capped at the number of 64-token
 * chunks and rounded to whole chunks per segment.  Every segment count gives
 * the same result up to the order of the chained fold; the hook lets the
 * choice be timed and lets tests cover many-segment chains on small inputs.
 */
SELSCAN_API void selscan_debug_fwd_segments(int segs);

/*
 * The number of time segments per channel tile that selscan_bwd would pick
 * for `tiles` tiles of (batch row, 32 channels), `nchunks` 8-token
 * checkpoint chunks and `slots` warps resident at once (blocks per SM x
 * SMs), before rounding to whole chunks per segment.  Host arithmetic only:
 * no CUDA call.  Lets the choice be tested without a GPU.
 */
SELSCAN_API long long selscan_debug_bwd_plan(long long tiles, long long nchunks, long long slots);

/*
 * The time segments per channel tile that selscan_fwd would pick in its
 * automatic mode (bf16) for `tiles` tiles of 128 channels, `chunks` 64-token
 * chunks and `ctas` persistent CTAs, before rounding to whole chunks per
 * segment: positive for the one-pass form with chained carries, negative
 * (minus the count) for the two-pass form.  Host arithmetic only: no CUDA
 * call.  Lets the choice be tested without a GPU.
 */
SELSCAN_API long long selscan_debug_fwd_plan(long long tiles, long long chunks, long long ctas);

#ifdef __cplusplus
}
#endif

#endif /* SELSCAN_DEBUG_H */

/*
 * pa_testing.h -- test hooks of libpa.so.  Not for use in production code.
 *
 * Every wait inside the decode kernels is bounded: a warp waiting for a
 * stage of its shared-memory ring to be filled (or emptied) gives up after
 * a time limit, sets PA_DEV_WAIT_TIMEOUT in *dev_status, and the kernel
 * returns normally, leaving the CUDA context usable.  The outputs of every
 * sequence whose remaining work that CTA held are then zeros.  No warp of
 * the decode kernels ever waits for another CTA.  These hooks let a test
 * make such a wait run out, on purpose and quickly, without any fault or
 * hang: one CTA's producer leaves the copies of one tile unissued, so the
 * stage they would fill never completes and the waits on it expire after
 * the limit.  The pages have no counterpart; the hooks exist to test this
 * library's failure handling.
 *
 * Both settings are process-wide, apply to decode launches made after the
 * call, and are not thread-safe with respect to concurrent launches.
 */
#ifndef PA_TESTING_H_
#define PA_TESTING_H_

#ifdef __cplusplus
extern "C" {
#endif

/* Limit of every bounded wait of the decode kernels, in nanoseconds; 0
 * restores the default (2 s). */
void pa_testing_set_wait_limit_ns(unsigned long long ns);

/* CTA `cta` of every following decode launch (when its range holds at
 * least two tiles) issues no copy for its second tile.  Its waits then run
 * out: PA_DEV_WAIT_TIMEOUT is set, and the outputs of the sequences whose
 * work from that tile on the CTA held are zeros.  A negative value turns
 * the hook off. */
void pa_testing_withhold_copy(int cta);

#ifdef __cplusplus
}
#endif

#endif /* PA_TESTING_H_ */

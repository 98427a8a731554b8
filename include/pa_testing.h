/*
 * pa_testing.h -- test hooks of libpa.so.  Not for use in production code.
 *
 * The decode kernels bound every wait: on a stage barrier of their
 * shared-memory ring, and, in a merge of a sequence split over many CTAs,
 * on the count of the pieces the other CTAs have published.  A wait that
 * runs out sets PA_DEV_WAIT_TIMEOUT in *dev_status and the kernel returns
 * normally, leaving the CUDA context usable.  These hooks let a test make
 * such a wait run out, on purpose and quickly, without any fault or hang:
 * one CTA simply does not count its pieces in, so the waits of the CTAs
 * merging with it expire after the limit.  The pages have no counterpart;
 * the hooks exist to test this library's failure handling.
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

/* CTA `cta` of every following stream-K decode launch publishes no piece
 * of a sequence split across CTAs and does not count it in; it still takes
 * its share of the merges of sequences split into more than 8 pieces.
 * Those merges then run out of time: their outputs are zeros and
 * PA_DEV_WAIT_TIMEOUT is set.  A negative value turns the hook off. */
void pa_testing_withhold_pieces(int cta);

#ifdef __cplusplus
}
#endif

#endif /* PA_TESTING_H_ */

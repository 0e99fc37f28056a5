/*
 * mcs_test.h — test hooks of the MC-Sparse library. Not for production use.
 */
#ifndef MCS_TEST_H_
#define MCS_TEST_H_

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Process-wide debug flags read by every later call (0 = off).
 * Bit 0: the attention producer never delivers its first K/V tile, so the
 * consumers' bounded waits expire; the call's status block then reports
 * MCS_ERR_TIMEOUT through mcs_poll_status, and the CUDA context stays usable.
 * Bit 1: the anchor's top-K takes its general seven-sweep path for every
 * group (the two-sweep path must give the same selection).
 * Bit 2: mcs_dense at d = 128 runs the one-query-tile kernel instead of the
 * kernel over pairs of query tiles (both compute the same attention; for
 * comparisons).
 */
void mcs_debug_set_flags(int flags);

/* Number of kernel launches the library has enqueued in this process. */
long long mcs_debug_launch_count(void);

/*
 * Per-launch timing of the anchor's selection passes (a measurement hook).
 * With ev non-NULL, every later mcs_anchor records, for each head chunk c of
 * its mass and top-K passes, ev[3c] before the chunk's mass launch, ev[3c+1]
 * between the mass and top-K launches and ev[3c+2] after the top-K launch, on
 * the call's stream, for c < n / 3 (chunks beyond that record nothing). The
 * events are the caller's (cudaEvent_t handles created with timing enabled)
 * and must outlive those calls; NULL turns the hook off. Process-wide, like
 * the debug flags.
 */
void mcs_debug_set_anchor_chunk_events(void* const* ev, int n);

#ifdef __cplusplus
}
#endif

#endif /* MCS_TEST_H_ */

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
 */
void mcs_debug_set_flags(int flags);

/* Number of kernel launches the library has enqueued in this process. */
long long mcs_debug_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MCS_TEST_H_ */

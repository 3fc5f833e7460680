/*
 * moga_testing.h -- test-only hook of libmoga.so (not part of the layer's API).
 *
 * moga_test_set_attn_debug(timeout_cycles, flags) sets, for the calling host
 * thread, the bounded-wait limit (in SM clock cycles; <= 0 restores the
 * default of about two seconds) and debug flags used by the next
 * moga_group_attn / stga_attn launches:
 *   flags bit 0: the producer warp skips the query-tile load, so the MMA
 *   warp's wait on it runs out; the kernel then records MOGA_ERR_TIMEOUT in
 *   the device error word, drains its in-flight copies, frees its tensor
 *   memory and exits (no trap, no hang).  moga_device_status() reports it.
 * Pass (0, 0) to restore normal operation.
 */
#ifndef MOGA_TESTING_H
#define MOGA_TESTING_H

#ifdef __cplusplus
extern "C" {
#endif

void moga_test_set_attn_debug(long long timeout_cycles, int flags);

#ifdef __cplusplus
}
#endif

#endif /* MOGA_TESTING_H */

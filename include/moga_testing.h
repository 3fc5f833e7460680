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
 *
 * moga_test_stga_groups(geom, out, cap) validates geom as stga_attn does and
 * returns the number n of temporal groups its launches use (-1 if stga_attn
 * would reject the geometry; moga_last_error() says why), writing for group
 * i < min(n, cap) the four int32 values out[4i .. 4i+3] = (first frame, end
 * frame (exclusive), frames borrowed from the previous shot, frames borrowed
 * from the next shot).  Host code only: no device is touched.
 */
#ifndef MOGA_TESTING_H
#define MOGA_TESTING_H

#include "moga.h"

#ifdef __cplusplus
extern "C" {
#endif

void moga_test_set_attn_debug(long long timeout_cycles, int flags);
int32_t moga_test_stga_groups(const moga_stga_geom* geom, int32_t* out, int32_t cap);

#ifdef __cplusplus
}
#endif

#endif /* MOGA_TESTING_H */

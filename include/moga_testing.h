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
 * moga_test_set_attn_events(before, after) takes two cudaEvent_t handles
 * (created by the caller, on the device of the calls) for the calling host
 * thread: the next forward attention-kernel launch of moga_group_attn,
 * stga_attn, stga_attn_mean, visual_attn_branches or their batched forms
 * records `before` on its stream just in front of it, and every attention-
 * kernel launch from then on records `after` just behind it, so that after
 * one call the two events bracket that call's attention launches without
 * its gather copies.  Set it again before each call to be timed; (NULL,
 * NULL) switches it off.  A failed record returns MOGA_ERR_CUDA from the
 * call.  Profiling use only: it changes no result.
 *
 * moga_test_stga_groups(geom, out, cap) validates geom as stga_attn does and
 * returns the number n of temporal groups its launches use (-1 if stga_attn
 * would reject the geometry; moga_last_error() says why), writing for group
 * i < min(n, cap) the four int32 values out[4i .. 4i+3] = (first frame, end
 * frame (exclusive), frames borrowed from the previous shot, frames borrowed
 * from the next shot).  Host code only: no device is touched.
 *
 * moga_test_attn_tiles(mode, cu_seqlens, M, N, H, geom, out, cap) returns the
 * number n of work tiles one attention launch processes (-1 on invalid
 * arguments) and writes for tile L < min(n, cap), in launch order, the five
 * int32 values out[5L .. 5L+4] = (head, query begin, query end, key begin,
 * key end), rows in the launch's index space: segment order for mode 0
 * (MoGA; cu_seqlens is a HOST array of M+1 entries, N tokens), the
 * window-major order for mode 1 (windows; geom), token order for mode 2
 * (frames; geom).  moga_test_window_tokens(geom, begin, end, out) writes the
 * tokens at window-major positions [begin, end) to out and returns their
 * count (-1 on invalid arguments).  Both run the kernels' own index code
 * compiled for the host; no device is touched.
 *
 * moga_test_bwd_units(mode, keys, cu_seqlens, M, N, H, geom, grid, out, cap)
 * does the same for the backward: *grid receives the number of CTAs the
 * launch uses (the dQ kernel for keys = 0, the dK/dV kernel for keys = 1),
 * the return value is the number n of valid units among them (-1 on invalid
 * arguments), and unit i < min(n, cap) is written as the seven int32 values
 * out[7i .. 7i+6] = (head, query begin, query end, key begin, key end, tile
 * begin, tile end), the tile being a range of queries (keys = 0) or of keys
 * (keys = 1) of at most 128 rows.
 */
#ifndef MOGA_TESTING_H
#define MOGA_TESTING_H

#include "moga.h"

#ifdef __cplusplus
extern "C" {
#endif

void moga_test_set_attn_debug(long long timeout_cycles, int flags);
void moga_test_set_attn_events(void* before, void* after);
int32_t moga_test_stga_groups(const moga_stga_geom* geom, int32_t* out, int32_t cap);
int32_t moga_test_attn_tiles(int32_t mode, const int32_t* cu_seqlens, int32_t M, int64_t N, int32_t H,
                             const moga_stga_geom* geom, int32_t* out, int32_t cap);
int32_t moga_test_window_tokens(const moga_stga_geom* geom, int32_t begin, int32_t end, int32_t* out);
int32_t moga_test_bwd_units(int32_t mode, int32_t keys, const int32_t* cu_seqlens, int32_t M, int64_t N,
                            int32_t H, const moga_stga_geom* geom, int32_t* grid, int32_t* out, int32_t cap);

#ifdef __cplusplus
}
#endif

#endif /* MOGA_TESTING_H */

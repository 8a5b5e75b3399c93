/*
 * ts_moe_debug.h -- helpers exported for tests.  All but the last expose the
 * pure arithmetic the kernels use to split work between CTAs and the open-time
 * validation, so both can be checked on a machine without a GPU; they touch
 * neither device memory nor the CUDA runtime.  The last one changes a
 * handle's device counters so that a test can make a bounded wait run out.
 */
#ifndef TS_MOE_DEBUG_H
#define TS_MOE_DEBUG_H

#include <stdint.h>

#include "ts_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* First unit of CTA b when U units are cut into NB contiguous ranges:
 * floor(b * U / NB).  Range of CTA b = [start(b), start(b + 1)). */
uint64_t ts_moe_debug_range_start(uint64_t U, int NB, int b);
/* The CTA whose range holds unit u (0 <= u < U, U >= 1). */
int ts_moe_debug_owner_of(uint64_t U, int NB, uint64_t u);
/* Partial-sum slot (0 or 1) CTA b uses for the group whose first unit is g0. */
int ts_moe_debug_partial_slot(uint64_t U, int NB, int b, uint64_t g0);
/* Group-aligned gate/up partition (used when ts_moe_debug_use_aligned(G, NB)):
 * first unit of CTA b (0 <= b <= NB) when G groups of `chunks` units each
 * are split so that every CTA stays inside one group. */
uint64_t ts_moe_debug_aligned_start(int G, int NB, int chunks, int b);
int ts_moe_debug_use_aligned(int G, int NB);
/* Tiles per group chosen for an expert matrix of `tiles` 16-row tiles. */
int ts_moe_debug_group_size(int tiles);
/* CTAs per layer-kernel launch on a device with `sm_count` SMs (one per SM). */
int ts_moe_debug_layer_ctas(int sm_count);
/* 1 when `nb` CTAs of the layer kernel can all be resident at once given
 * `per_sm` of them per SM (the occupancy calculator's answer) on `sm_count`
 * SMs; ts_moe_open refuses with TS_MOE_EUNSUPPORTED when this is 0. */
int ts_moe_debug_coresident(int per_sm, int sm_count, int nb);
/* The validation ts_moe_open performs before any CUDA call; same status and
 * message (ts_moe_last_error(NULL)). */
ts_moe_status ts_moe_debug_validate(const ts_moe_config* cfg, const ts_moe_layer_weights* layers);

/* Failure-path test hook.  Synchronises `stream`, then marks the handle so
 * that in the next layer-kernel launch CTA 0 does not arrive at the grid
 * barrier.  The barrier cannot complete: every CTA gives up after the bounded
 * wait (2 s), sets the "grid barrier wait gave up" bit (0x40) of the device
 * error word, and the kernel runs to its end.  The next ts_moe_device_status
 * returns TS_MOE_EDEVICE and re-zeroes the counters, after which calls work
 * normally again.  Not for production use. */
ts_moe_status ts_moe_debug_skew_barrier(ts_moe* h, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* TS_MOE_DEBUG_H */

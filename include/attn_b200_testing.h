/*
 * attn_b200_testing.h - testing hooks of the attention library (not part of the
 * operation; the pages define no counterpart).
 *
 * attn_fwd_inject_timeout - attn_fwd for BF16, d = 128, always on the
 * two-Q-tile schedule (attn_fwd itself runs launches with fewer two-tile units
 * than SMs on the one-tile schedule, which gives bit-identical results), with
 * one failure planted on purpose so that the bounded-wait path of the kernel
 * can be run on a GPU without faulting it (a fault_unit at or past the number
 * of units plants nothing): the TMA producer of the CTA that processes work
 * unit `fault_unit` never loads that unit's first K tile, so the mbarrier the
 * MMA warp waits on is never completed. Every pipeline wait of the launch
 * gives up after `wait_limit_cycles` SM cycles (instead of the 2^31 that
 * attn_fwd uses); the CTA then sets its abort word, lets its in-flight copies
 * and MMAs land, releases its tensor memory and exits, and the launch records
 * ATTN_ERR_TIMEOUT in the device status word (read and cleared by
 * attn_get_device_status). Other CTAs are not affected; the CUDA context stays
 * usable, and the output of the failed unit is undefined.
 *
 * Work units are numbered as the kernel walks them: unit u covers one head and
 * two consecutive 128-row Q tiles (u < B*H*ceil(ceil(N/128)/2)).
 *
 * Arguments as for attn_fwd (device pointers, [B, H, N, 128] bf16, 16-byte
 * aligned), plus fault_unit >= 0 and wait_limit_cycles >= 1024.
 * Returns the launch status (ATTN_OK when the kernel was launched) or the same
 * host-side argument errors as attn_fwd; ATTN_ERR_UNSUPPORTED unless d == 128.
 */
#ifndef ATTN_B200_TESTING_H
#define ATTN_B200_TESTING_H

#include "attn_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

ATTN_API attn_status attn_fwd_inject_timeout(const void* q, const void* k, const void* v, void* o, float* lse,
                                             int B, int H, int N, int d, float scale, int causal, int fault_unit,
                                             unsigned long long wait_limit_cycles, void* stream);

/*
 * attn_fwd_one_tile_inject_timeout - the same hook on the one-Q-tile schedule
 * (the kernel attn_fwd runs for launches with few units, and the one
 * attn_fwd_mxfp8 runs): work unit u covers one head and ONE 128-row Q tile
 * (u < B*H*ceil(N/128)), numbered as for the two-tile schedule with one tile per
 * pair. Arguments, limits and results as for attn_fwd_inject_timeout.
 */
ATTN_API attn_status attn_fwd_one_tile_inject_timeout(const void* q, const void* k, const void* v, void* o,
                                                      float* lse, int B, int H, int N, int d, float scale,
                                                      int causal, int fault_unit,
                                                      unsigned long long wait_limit_cycles, void* stream);

/*
 * attn_fwd_mxfp8_inject_timeout - attn_fwd_mxfp8 (same arguments, same kernel)
 * with the same planted failure: the producer of work unit `fault_unit` (one
 * head and one 128-row Q tile, numbered as for attn_fwd_one_tile_inject_timeout)
 * never loads that unit's first K tile, and every pipeline wait gives up after
 * `wait_limit_cycles`. Besides the producer / MMA / softmax waits this runs out
 * the MXFP8 kernel's own: the converter warps' V-tile waits, the exchange of
 * half-row maxima and sums between its two softmax warpgroups, and the hand-over
 * of a unit's V scale maxima. fault_unit >= 0 and wait_limit_cycles >= 1024
 * (else ATTN_ERR_INVALID_ARG); other results as for attn_fwd_inject_timeout.
 */
ATTN_API attn_status attn_fwd_mxfp8_inject_timeout(const void* q8, const void* k8, const void* v8,
                                                   const void* q_sf, const void* k_sf, const void* v_sf, void* o,
                                                   float* lse, int B, int H, int N, int d, float scale, int causal,
                                                   int fault_unit, unsigned long long wait_limit_cycles,
                                                   void* stream);

/*
 * attn_fwd_debug_row_limit - debug builds only (ATTN_ERR_UNSUPPORTED otherwise):
 * attn_fwd (BF16, same arguments, same schedule choice) with the kernels told
 * that O and LSE hold only `row_limit` rows (rows counted over all heads,
 * b * H * N + h * N + i). The debug checks then reject, skip and record
 * (ATTN_ERR_BOUNDS, site 1 or 2, index = a rejected row) every store of
 * a row at or past the limit, while the caller's buffers still hold all
 * B*H*N rows, so the check can be seen to fire without any access outside
 * them. Rows below the limit are written as attn_fwd writes them.
 * 0 <= row_limit <= B*H*N, else ATTN_ERR_INVALID_ARG.
 */
ATTN_API attn_status attn_fwd_debug_row_limit(const void* q, const void* k, const void* v, void* o, float* lse,
                                              int B, int H, int N, int d, float scale, int causal,
                                              long long row_limit, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_TESTING_H */

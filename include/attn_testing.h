/*
 * attn_testing.h - test hooks of the B200 masked attention library (not needed to use it).
 *
 * These entry points expose internal device routines so that tests can check them in
 * isolation. No page of the masked-attention pages has a counterpart: the first routine
 * is the share of the softmax exponentials the forward kernel can evaluate on the FMA pipes
 * instead of the MUFU unit, the second the backward planner's mask-tile transposition, the
 * third forces a bounded wait to expire inside attn_masked_fwd_noalloc().
 */
#ifndef MASKED_ATTN_B200_ATTN_TESTING_H
#define MASKED_ATTN_B200_ATTN_TESTING_H

#include <stdint.h>

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* y[i] = 2^x[i] by the forward kernel's polynomial path (range reduction x = n + f,
 * degree-3 minimax polynomial for 2^f on [-1/2, 1/2], max relative error 7.5e-5; inputs
 * below -125 are clamped to -125). x and y are DEVICE fp32 arrays of n elements; the work
 * is enqueued on `stream`. Errors: INVALID_ARG (null pointer with n > 0), CUDA. */
attn_status_t attn_test_exp2_poly(const float* x, float* y, int64_t n, attn_stream_t stream);

/* The planner's transposition of a 2 KiB mask tile (host memory): src row r (four 32-bit
 * words, bit c of word c / 32 = key c, LSB first) becomes dst row c (bit r = query r), the
 * layout the dK/dV kernel reads. No GPU involved. Errors: INVALID_ARG (null pointer). */
attn_status_t attn_test_transpose_mask_tile(const uint32_t* src, uint32_t* dst);

/* Debug settings of the following attn_masked_fwd_noalloc() calls in this process, as
 * attn_plan_set_debug() sets them for a plan: flags bit 0 skips the first work item's query
 * load in every CTA (its wait then expires after timeout_ns), timeout_ns bounds every wait
 * (default 2 s). (0, 2000000000) restores the defaults. Errors: INVALID_ARG (flags < 0 or
 * timeout_ns <= 0). */
attn_status_t attn_test_noalloc_debug(int32_t flags, int64_t timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* MASKED_ATTN_B200_ATTN_TESTING_H */

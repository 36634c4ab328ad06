/*
 * attn_testing.h - test hooks of the B200 masked attention library (not needed to use it).
 *
 * These entry points expose internal device routines so that tests can check them in
 * isolation. No page of the masked-attention pages has a counterpart; the routine below
 * is the share of the softmax exponentials the forward kernel evaluates on the FMA pipes
 * instead of the MUFU unit.
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

#ifdef __cplusplus
}
#endif

#endif /* MASKED_ATTN_B200_ATTN_TESTING_H */

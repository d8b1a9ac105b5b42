/*
 * sparse_attn_testing.h - test hooks of libsparse_attn.so. Not part of the
 * attention API; they expose internal device routines so that tests can
 * check them against their stated error bounds.
 */
#ifndef SPARSE_ATTN_TESTING_H
#define SPARSE_ATTN_TESTING_H

#include "sparse_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* y[i] = the attention kernel's software 2^x (Cody-Waite range reduction and
 * a degree-3 Remez polynomial on the FMA pipe) for x[i], i < n. x and y are
 * device pointers to fp32 arrays of n elements; the call is asynchronous on
 * `stream`. Valid inputs are x <= 8 (the kernel never evaluates larger
 * arguments); x = -inf gives 0. */
sa_status sparse_attn_test_exp2_poly(const float* x, float* y, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_TESTING_H */

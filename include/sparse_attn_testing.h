/*
 * sparse_attn_testing.h - test hooks of libsparse_attn.so. Not part of the
 * attention API: they let tests drive paths that normal inputs never reach.
 */
#ifndef SPARSE_ATTN_TESTING_H
#define SPARSE_ATTN_TESTING_H

#include "sparse_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Failure detection of the attention kernel (no counterpart in the papers).
 * Runs sparse_attn_fwd (same arguments, same validation) with two changes:
 * every pipeline wait of the kernel is bounded by wait_limit_ns instead of
 * the library's 4 s, and the TMA producer of the first row pipeline of the
 * first CTA never issues the copy of its first K tile, so the waits that
 * depend on that copy cannot complete. The kernel then records
 * SA_ERR_TIMEOUT in the device error record (its info field names the wait
 * that ran out first), the roles of that CTA leave their loops, wait for the
 * copies and matrix products they had already issued, free their tensor
 * memory and return; the other CTAs finish normally. O is undefined for the
 * query-block rows of that CTA. The call itself returns SA_OK once the
 * launch is enqueued; read the outcome with sparse_attn_check_device_error.
 * wait_limit_ns must lie in [1e6, 4e9] (1 ms to 4 s), else SA_ERR_INVALID_ARG. */
sa_status sparse_attn_test_fwd_withheld_copy(const sa_shape* shape, const void* Q, const void* K,
                                             const void* V, const int32_t* cnt, const int32_t* idx,
                                             void* O, int o_dtype, uint64_t wait_limit_ns,
                                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_TESTING_H */

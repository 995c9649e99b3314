/*
 * libspecverify test hooks. These entry points are not part of the verify
 * step: they expose pieces of the library that the step's outputs only show
 * indirectly, so that tests can check them directly.
 *
 *   sv_testing_philox4x32_10   the device Philox4x32-10 block function that
 *                              sv_accept draws its uniforms from (Salmon,
 *                              Moraes, Dror, Shaw, "Parallel random numbers:
 *                              as easy as 1, 2, 3", SC'11), applied to a list
 *                              of counters, so that it can be compared word by
 *                              word with published known answers and with an
 *                              independent implementation.
 *   sv_testing_verify_attention_stalled
 *                              sv_verify_attention in which one wait of every
 *                              CTA waits on a barrier that nothing arrives on.
 *                              Every device-side wait of the attention kernel is
 *                              bounded; this makes one run out on purpose, with
 *                              a short bound, so that a test can check that the
 *                              call returns, that every sequence is flagged
 *                              SV_FLAG_TIMEOUT, and that the context is still
 *                              usable afterwards. Nothing faults or hangs: the
 *                              kernel takes its ordinary abort path.
 * Conventions as in specverify.h: device pointers owned by the caller,
 * asynchronous on `stream`, argument errors returned before any launch.
 */
#ifndef SPECVERIFY_TESTING_H
#define SPECVERIFY_TESTING_H

#include "specverify.h"

#ifdef __cplusplus
extern "C" {
#endif

/* out[i][0..3] = Philox4x32-10(counter = counters[i][0..3], key = {key_lo32,
 * key_hi32}) for i < n. counters and out: uint32 [n][4], 16-byte aligned
 * device memory; 0 <= n <= 2^31. key_lo32/key_hi32 are the low and high words
 * of the 64-bit seed that sv_accept takes as philox_seed. */
SV_API sv_status sv_testing_philox4x32_10(uint64_t key, const uint32_t *counters, uint32_t *out,
                                          int64_t n, void *stream);

/* Arguments and results of sv_verify_attention, except that each CTA makes one
 * wait that cannot succeed and every wait gives up after wait_limit_ns
 * (1 ms .. 2 s; SV_ERR_INVALID_ARG outside). Expected result: SV_OK, every
 * sequence's status_flags has SV_FLAG_TIMEOUT set, out is undefined. */
SV_API sv_status sv_testing_verify_attention_stalled(const sv_attn_desc *desc, const void *q,
                                                     const sv_paged_kv *paged_kv, const int32_t *block_table,
                                                     const int32_t *ctx_lens, const uint64_t *draft_mask,
                                                     void *out, void *workspace, size_t workspace_bytes,
                                                     int32_t *status_flags, uint64_t wait_limit_ns,
                                                     void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SPECVERIFY_TESTING_H */

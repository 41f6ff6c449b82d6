/*
 * omnikv_testing.h -- failure-injection hooks of the OmniKVQuant library, for
 * tests. The pages have no counterpart: these entry points exist so that the
 * error paths of the kernels can be run on a GPU without faulting or hanging it.
 */
#ifndef OMNIKV_TESTING_H_
#define OMNIKV_TESTING_H_

#include "omnikv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The decode launch of a decode step (omnikv_append_decode) without its append: the
 * cache is read as if one token had been appended to every sequence, and the copy of
 * each sequence's last window waits until cache->step_flags[b][h] holds
 * seq_lens[b] + 1, for at most flag_wait_ns nanoseconds. Nothing in this call writes
 * the flags, so unless the caller does, every such wait runs out: the launch then
 * sets OMNIKV_DEVERR_TIMEOUT in cache->error_word, copies no stale record, and
 * writes the affected splits empty (weight 0 in the combine). Arguments as
 * omnikv_decode_attention (partials sized for the split count of the cache with
 * max_seq_len + 1), plus
 *   flag_wait_ns : wait limit of the flag (the library's own launches use 2 s).
 * Requires cache->step_flags (OMNIKV_ERR_INVALID_ARG without it); does not change
 * the cache. */
OMNIKV_API omnikv_status omnikv_test_decode_pending(const omnikv_config* cfg, const omnikv_cache* cache,
                                                    const void* q, void* partials, int32_t num_splits,
                                                    uint64_t flag_wait_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* OMNIKV_TESTING_H_ */

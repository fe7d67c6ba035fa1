/*
 * kvq_check.h -- entry points of the bounds-check build of libkvq only
 * (libkvq_check.so, compiled with -DKVQ_CHECK); the product library does not
 * export them.  In that build every kernel that indexes through a list made on
 * the host or by the caller (the quantizer's input rows, the gather of retained
 * rows, the LogQuant compaction) checks each index against its buffer, raises
 * bit 3 of the cache's status word for a bad one and reads row 0 instead (or
 * writes nothing); kvq_check_device reports it as KVQ_ERR_DEVICE_CHECK.  The
 * pages have no counterpart: these exist so that tests can make the checks and
 * the bounded waits fire without a fault.
 */
#ifndef KVQ_CHECK_H
#define KVQ_CHECK_H

#include "kvq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * From the next decode on, warp 0 of the first CTA of the bf16-MMA decode kernel
 * first waits on a shared-memory barrier that nothing arrives at, for at most
 * `polls` polls (each a bounded suspend of up to 0.2 ms), then gives up: it
 * raises bit 0 of the status word, contributes no tokens and returns through the
 * normal exit.  0 turns it off.  The output of such a decode is wrong for that
 * warp's sequence and head group; the context stays usable.
 */
KVQ_API kvq_status kvq_debug_set_stall(kvq_cache *cache, int32_t polls);

/*
 * dst[i] = src[idx[i]] for i < n (rows of head_dim e elements of this cache's
 * geometry; src has src_rows rows), through the gather kernel the LogQuant
 * prefill uses, raising bit 3 of the cache's status word for an index outside
 * [0, src_rows).  src and dst: device, 16-byte aligned.
 */
KVQ_API kvq_status kvq_debug_gather_rows(kvq_cache *cache, const void *src, int64_t src_rows, const int32_t *idx,
                                         int32_t n, void *dst, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_CHECK_H */

/*
 * xgr_sched.h -- C ABI of the host-side batch former (libxgr.so): the Chunked
 * Hash Tree that groups prefix-homogeneous requests.
 *
 * What it computes, per the Feather page ("Requests of the same feather must
 * flock together", "Methodology", 1. Chunked Hash Tree): a request is
 * represented by cumulative hashes over fixed-size chunks of its prompt
 * tokens; the batch being formed keeps a working set of the hashes of its
 * members; waiting requests sit in a min-heap keyed by their missing count,
 * the number of their chunks the working set does not cover, so the best
 * request to add next is found in O(log W) for W waiting requests.  The page's
 * operations are insert, find-best, add-to-batch and remove, with lazy heap
 * updates and incremental maintenance of the batch's shared-prefix tip.  The
 * batches it forms are the prefix-homogeneous groups the attention serves
 * (one shared KV segment per group: xgr_prefill_kv's shared_id).
 *
 * Readings where the page is silent (each also in the repository's design
 * notes):
 *  - Only full chunks are hashed; a prompt's trailing partial chunk never
 *    counts as shared.
 *  - Chunk hash i is the SplitMix64 finaliser (Steele, Lea, Flood, 2014)
 *    folded over every token of chunks 0..i, starting from 0:
 *    h = splitmix64(h ^ (uint32_t)token) token by token.  Two requests share
 *    chunk i iff their hash i is equal (a 64-bit collision is taken as
 *    sharing).
 *  - Missing count of a waiting request = its chunks whose hash is not in the
 *    working set (the set is closed under prefixes, so this is its chunk count
 *    minus its longest prefix present in the batch).
 *  - Best request: smallest missing count, then the earliest inserted.  An
 *    empty batch takes the earliest-inserted waiting request (first come,
 *    first served seeds each batch).
 *  - Tip: the number of leading chunks shared by every member of the batch.
 *    For a candidate, depth_after = min(tip, chunks it shares with the first
 *    member) and delta = tip - depth_after (the page's loss of shared prefix
 *    depth).  w = waiting requests other than the candidate whose chunk
 *    depth_after - 1 is the batch's (the page's count of requests sharing the
 *    new depth; 0 when depth_after is 0).
 *  - Stopping policy (xgr_cht_form_batches): the page's learned policies need
 *    live traffic and are not built; the static rule here adds, while the
 *    batch holds fewer than max_batch requests, the best waiting request among
 *    those whose depth_after >= min_shared_chunks (smallest missing count,
 *    then the earliest inserted), and dispatches when none qualifies.  A
 *    request that shares too little with the batch (a short or unrelated
 *    prompt: few chunks, so a small missing count) is passed over, not allowed
 *    to end the batch while requests sharing its prefix still wait.
 *
 * Conventions: host memory only, no CUDA calls; a handle is not thread-safe
 * (one caller at a time); request ids are non-negative int64s unique among
 * live requests (a negative id is XGR_ERR_ARG: -1 reports "none waiting").  Every call returns an xgr_status (XGR_OK = 0); XGR_ERR_ARG for a
 * null handle or pointer, an unknown or duplicate id, or max_batch < 1;
 * XGR_ERR_STATE for a request in the wrong state (adding or removing one that
 * is not waiting); XGR_ERR_SHAPE for a negative length or a chunk size < 1.
 */
#ifndef XGR_SCHED_H
#define XGR_SCHED_H

#include <stdint.h>

#include "xgr.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct xgr_cht xgr_cht;

/* A new, empty tree with chunks of chunk_tokens tokens.  Free with
 * xgr_cht_destroy. */
xgr_status xgr_cht_create(int32_t chunk_tokens, xgr_cht **out);
xgr_status xgr_cht_destroy(xgr_cht *t);

/* A waiting request: its prompt tokens (host, int32 [n_tokens], copied).  Its
 * missing count is taken against the batch being formed, if any. */
xgr_status xgr_cht_insert(xgr_cht *t, int64_t request_id, const int32_t *h_tokens, int64_t n_tokens);

/* A waiting request leaves (completed or cancelled elsewhere).  Members of the
 * batch being formed cannot be removed. */
xgr_status xgr_cht_remove(xgr_cht *t, int64_t request_id);

/* The best waiting request for the batch being formed (see above), or
 * *request_id = -1 when none waits.  Any of missing / depth_after / delta / w
 * may be null. */
xgr_status xgr_cht_find_best(xgr_cht *t, int64_t *request_id, int32_t *missing, int32_t *depth_after,
                             int32_t *delta, int32_t *w);

/* A waiting request joins the batch being formed: its chunk hashes enter the
 * working set and the missing counts of the waiting requests that share them
 * drop (lazily, in the heap). */
xgr_status xgr_cht_add_to_batch(xgr_cht *t, int64_t request_id);

/* Closes the batch being formed: writes up to cap member ids in the order they
 * joined to h_ids, their number to *n, the batch's shared depth in chunks to
 * *shared_chunks (either of the last two may be null), then empties the batch
 * and the working set.  The members leave the tree. */
xgr_status xgr_cht_dispatch(xgr_cht *t, int64_t *h_ids, int32_t cap, int32_t *n, int32_t *shared_chunks);

/* Requests waiting, and members of the batch being formed. */
xgr_status xgr_cht_counts(xgr_cht *t, int32_t *waiting, int32_t *in_batch);

/* Forms batches from every waiting request with the static policy above,
 * starting from an empty batch (one being formed is dispatched first as batch
 * 0).  Writes, in dispatch order, each batch's member ids contiguously to
 * h_ids (cap_ids entries), each batch's member count to h_sizes and its shared
 * depth in chunks to h_shared (cap_batches entries each), and the number of
 * batches to *n_batches.  XGR_ERR_CAPACITY when an array is too small (nothing
 * is formed then). */
xgr_status xgr_cht_form_batches(xgr_cht *t, int32_t max_batch, int32_t min_shared_chunks, int64_t *h_ids,
                                int64_t cap_ids, int32_t *h_sizes, int32_t *h_shared, int32_t cap_batches,
                                int32_t *n_batches);

#ifdef __cplusplus
}
#endif

#endif /* XGR_SCHED_H */

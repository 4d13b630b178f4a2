/*
 * xgr.h -- C ABI of the B200 beam-decode hot path (libxgr.so).
 *
 * What the library computes, per the xGR page ("xGR: Efficient Generative
 * Recommendation Serving at Scale"):
 *   2.1 xAttention  The KV cache is split in two.  The Shared part holds the
 *                   prompt (user history), computed once at prefill and read
 *                   once per request for all beams.  The Unshared part holds
 *                   only the tokens generated at each decode step, managed
 *                   token by token (no block padding, no block copy when
 *                   beams fork).  Attention runs in three stages: Shared and
 *                   Unshared each produce local scores with max/sum
 *                   statistics; a Merging stage combines them by online
 *                   softmax.  The Unshared cache is updated in place through
 *                   direct indices, without write-before-read hazards.
 *   2.2 xBeam       Candidates are filtered by masks built from a pre-built
 *                   vocabulary of valid items: dense, pre-generated masks for
 *                   the first step, sparse masks afterwards.  The top
 *                   candidates are chosen with early termination (a global
 *                   threshold cuts every beam's sorted candidate list).
 * The same split-KV attention serves prefix-homogeneous LLM batches (several
 * requests sharing one prompt prefix plus a private suffix), the batching the
 * Feather page argues for ("Requests of the same feather must flock
 * together", "Methodology").
 *
 * Conventions for every call:
 *  - Ownership: the caller allocates every device buffer, including the one
 *    workspace handed to xgr_create; the library allocates no device memory.
 *    The context (host struct) is owned by the library and freed by
 *    xgr_destroy.
 *  - Pointers named d_* are device pointers, h_* host pointers.  Device
 *    pointers must be 16-byte aligned.  bf16 means IEEE bfloat16 bits.
 *  - Streams: hot calls (xgr_decode_step, xgr_build_mask, xgr_beam_select,
 *    xgr_begin when its plan is unchanged, xgr_get_sequences) only enqueue
 *    kernels on the given stream; they never synchronise the host.  Setup
 *    calls (xgr_create, xgr_build_trie, xgr_prefill_kv, xgr_begin after a
 *    prefill) may synchronise.  xgr_device_status synchronises.
 *  - Errors: host-side validation returns a negative xgr_status at once and
 *    enqueues nothing.  Faults found on the device (an index out of range, a
 *    NaN score, a capacity overflow, a token outside the vocabulary) never
 *    trap: the kernel records a code in the device status word, skips the
 *    faulty element and carries on; xgr_device_status reports it.
 *  - Row layout: request r, beam b lives at row r * BW + b of every
 *    [B][BW]... array; beams b >= n_live(r) are dead: their attention output
 *    is 0 with LSE -inf, their selection slots hold parent -1, token -1,
 *    cum -inf.
 */
#ifndef XGR_H_
#define XGR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *xgr_stream_t;

typedef struct xgr_ctx xgr_ctx;
typedef int32_t xgr_status;

enum {
    XGR_OK = 0,
    XGR_ERR_ARG = -1,           /* null/misaligned pointer, unknown flag or kind */
    XGR_ERR_SHAPE = -2,         /* a size inconsistent with the config */
    XGR_ERR_CAPACITY = -3,      /* more than a capacity fixed at xgr_create */
    XGR_ERR_STATE = -4,         /* call out of order (e.g. step != current step) */
    XGR_ERR_CUDA = -5,          /* a CUDA runtime call failed */
    XGR_ERR_DEVICE = -6,        /* the device status word was non-zero */
    XGR_ERR_UNIMPLEMENTED = -7  /* configuration not supported by this build */
};

/* Device status word bits (xgr_device_status). */
enum {
    XGR_DEV_NAN = 1,            /* NaN among the scores or cumulative scores read */
    XGR_DEV_INDEX = 2,          /* ancestry slot / trie node out of range */
    XGR_DEV_MASK = 4,           /* a mask token that is not a child in the trie, or >= V */
    XGR_DEV_CAPACITY = 8,       /* mask rows exceeded the CSR capacity */
    XGR_DEV_TIMEOUT = 16        /* a bounded on-chip wait gave up (the CTA unwound, results invalid) */
};

/* Score input of xgr_beam_select. */
enum {
    XGR_SCORES_LOGPROB = 0,     /* fp32 log-probs; score = fp32(cum + lp), bit-exact contract */
    XGR_SCORES_LOGITS = 1       /* fp32 logits; lp = logit - logsumexp(row) over the full vocabulary */
};

/* KV kinds of xgr_prefill_kv. */
enum {
    XGR_KV_SHARED = 0,          /* prompt / shared prefix, stored once per shared id */
    XGR_KV_SUFFIX = 1           /* a request's private prefix continuation (beam width 1 use) */
};

/* Mask kinds (xGR 2.2 "Hybrid dense/sparse storage": dense, pre-generated
 * masks for the first steps, sparse masks updated in place afterwards). */
enum {
    XGR_MASK_DENSE = 0,         /* step 0: one bitset shared by every live beam */
    XGR_MASK_CSR = 1,           /* explicit CSR rows (xgr_mask_to_csr, or a caller's) */
    XGR_MASK_NODE_BITS = 2,     /* a pre-generated bitset per trie node, picked by each row's node */
    XGR_MASK_TRIE_ROWS = 3      /* each row = the sorted children of its trie node (no copy) */
};

typedef struct {
    int32_t max_requests;   /* B: requests per batch */
    int32_t max_shared;     /* number of shared ids (distinct prompt prefixes) */
    int64_t kv_tokens;      /* capacity of the prompt KV store, in tokens (all ids and suffixes) */
    int32_t beam_width;     /* BW (1..1024) */
    int32_t top_k;          /* K >= BW: candidates kept per beam before the global cut */
    int32_t steps;          /* S decode steps == item length (1..8) */
    int32_t n_q_heads;      /* Hq */
    int32_t n_kv_heads;     /* Hkv, divides Hq (query head h reads kv head h / (Hq/Hkv)) */
    int32_t head_dim;       /* D: 64 or 128 */
    int32_t vocab;          /* V: tokens per level (0: no selection, attention only) */
    int64_t max_items;      /* trie capacity, items */
    int32_t max_fanout;     /* bound on the children of any node below the root (0: V) */
    int32_t max_partials;   /* partial-attention slots per row for split-K (0: 8) */
} xgr_config;

/* A mask as produced by xgr_build_mask: views into the workspace, valid until
 * the next selection (which rewires the trie nodes the row views read).
 *  DENSE:      bits[w] bit j set <=> token 32w+j valid (every live beam of
 *              step 0); n_words = ceil(V/32).
 *  CSR:        the valid next tokens of row r*BW+b are cols[row_ptr[row] ..
 *              row_ptr[row+1]), ascending (device arrays; nnz = row_ptr[n_rows]).
 *  NODE_BITS:  row `row` may take token t iff bit t of the bitset
 *              bits + row_node[row] * n_words is set; the table holds one
 *              bitset per node of trie level `step`, pre-generated by
 *              xgr_build_trie.
 *  TRIE_ROWS:  row `row`'s valid tokens are cols[node_ptr[nd] ..
 *              node_ptr[nd+1]) with nd = row_node[row] (ascending): the trie
 *              level's own child lists, nothing copied.
 * row_node is the context's per-beam trie node, which the selection rewires in
 * place; rows of dead beams hold -1 and are empty.  row_stride bounds the
 * valid tokens of one row (the level's largest child count). */
typedef struct {
    int32_t kind;
    int32_t step;
    const uint32_t *bits;
    int32_t n_words;
    int32_t n_rows;
    const int32_t *row_ptr;
    const int32_t *cols;
    int64_t cols_capacity;
    const int32_t *row_node;
    const int32_t *node_ptr;
    int32_t n_nodes;
    int32_t row_stride;
} xgr_mask;

/* Bytes of device workspace a context with this config needs (256-byte
 * aligned regions: prompt KV store, Unshared pool, beam state, trie, masks,
 * selection and split-K scratch).  Returns XGR_ERR_ARG / XGR_ERR_SHAPE for an
 * invalid config. */
xgr_status xgr_workspace_bytes(const xgr_config *cfg, size_t *bytes);

/* Creates a context over a caller-owned device workspace of at least
 * xgr_workspace_bytes bytes (256-byte aligned), on the current device.
 * The workspace must outlive the context. */
xgr_status xgr_create(const xgr_config *cfg, void *d_workspace, size_t bytes, xgr_ctx **out);
xgr_status xgr_destroy(xgr_ctx *ctx);
const char *xgr_status_string(xgr_status s);

/* Builds the item trie (xGR 2.2 "Valid-path constraint") from h_items
 * [n_items][item_len] int32 (host; any order; duplicates are merged), and the
 * pre-generated dense mask of step 0.  item_len must equal cfg.steps; tokens
 * must lie in [0, V).  Synchronous (setup).  XGR_ERR_CAPACITY when n_items >
 * max_items or a node below the root has more than max_fanout children. */
xgr_status xgr_build_trie(xgr_ctx *ctx, const int32_t *h_items, int64_t n_items, int32_t item_len);

/* Loads prompt KV (xGR 2.1 "Separate KV cache": computed once at prefill).
 * d_k, d_v: bf16 [Hkv][len][D] (device).  Copied into the library's store;
 * the caller may free them after the call returns (the copy is complete on
 * return: this call synchronises the stream).
 *  kind XGR_KV_SHARED: links request -> shared_id; when d_k is non-null it
 *    (re)loads that id's prefix, when null the id must already be loaded.
 *  kind XGR_KV_SUFFIX: loads request's private suffix (shared_id ignored).
 * XGR_ERR_CAPACITY when the store (kv_tokens) is full. */
xgr_status xgr_prefill_kv(xgr_ctx *ctx, int32_t request, int32_t shared_id,
                          const void *d_k, const void *d_v, int32_t len, int32_t kind,
                          xgr_stream_t stream);

/* Forgets every prefilled prefix and suffix (the store is reused). */
xgr_status xgr_reset_kv(xgr_ctx *ctx);

/* Starts a beam decode of requests 0..n_requests-1: one live beam per request
 * with cumulative score 0 at the trie root.  Re-plans the attention work when
 * KV was prefilled since the last plan (then it synchronises). */
xgr_status xgr_begin(xgr_ctx *ctx, int32_t n_requests, xgr_stream_t stream);

/* Staged attention of decode step `step` (xGR 2.1), for every live beam:
 *   d_q     bf16 [B][BW][Hq][D]   this step's queries (rows of dead beams ignored)
 *   d_k_new bf16 [B][BW][Hkv][D]  this step's keys of each live beam's fed token,
 *   d_v_new bf16 [B][BW][Hkv][D]  appended to the Unshared pool at slot (step, b)
 *   d_out   bf16 [B][BW][Hq][D]   softmax(q K^T / sqrt(D)) V over the beam's
 *                                  shared prompt (+ suffix) and its own step+1
 *                                  Unshared tokens
 *   d_lse   fp32 [B][BW][Hq]      natural-log log-sum-exp of the scaled scores
 * B is n_requests of xgr_begin.  step must be the current step. */
xgr_status xgr_decode_step(xgr_ctx *ctx, int32_t step, const void *d_q, const void *d_k_new,
                           const void *d_v_new, void *d_out, float *d_lse, xgr_stream_t stream);

/* Per-beam comparison path -- a baseline, not the product path.  xGR page, 1
 * "Problem definition": serving systems built around PagedAttention treat
 * each beam as an independent sequence, so every beam reloads the shared
 * prompt KV, and forking beams copies KV blocks; 4 "Kernel efficiency"
 * compares the staged kernel with that baseline.  Same contract as
 * xgr_decode_step (same arguments and outputs, equal within rounding), but
 * computed that way: each beam streams its request's whole prompt (+ suffix)
 * from the KV store itself, and its generated tokens live in a private block
 * of 16 tokens that a new beam copies whole from its parent (its ancestry slot
 * of the previous step) before appending this step's k / v.  The context's
 * Unshared pool is neither read nor written.
 *   d_blocks: caller-owned device memory of xgr_per_beam_bytes bytes (16-byte
 *             aligned) kept for the whole decode, the first call of which is
 *             step 0 (its blocks of the previous step are the parents').
 * head_dim 128 and at most 8 query heads per kv head (else
 * XGR_ERR_UNIMPLEMENTED); blocks_bytes below the size: XGR_ERR_CAPACITY.  Two
 * kernels on `stream`; advances the current step only for a context without
 * a vocabulary, like xgr_decode_step. */
xgr_status xgr_per_beam_bytes(const xgr_ctx *ctx, size_t *bytes);
xgr_status xgr_decode_step_per_beam(xgr_ctx *ctx, int32_t step, const void *d_q, const void *d_k_new,
                                    const void *d_v_new, void *d_out, float *d_lse, void *d_blocks,
                                    size_t blocks_bytes, xgr_stream_t stream);

/* Valid-path mask of step `step` (xGR 2.2 "Hybrid dense/sparse storage").
 * Enqueues nothing: every kind is a view of pre-built tables and of the beam
 * state.  Step 0: DENSE (the root's bitset).  Step 1: NODE_BITS when
 * xgr_build_trie pre-generated that level's per-node bitsets (levels with many
 * valid tokens per node, whose table fits the workspace), else TRIE_ROWS.
 * Later steps: TRIE_ROWS -- each beam's row follows its trie node, which the
 * selection updates in place.  Fills *out. */
xgr_status xgr_build_mask(xgr_ctx *ctx, int32_t step, xgr_mask *out, xgr_stream_t stream);

/* Writes the mask of a step >= 1 (any kind, as returned by xgr_build_mask for
 * the current step) as explicit CSR rows: d_row_ptr int32 [n_rows+1],
 * d_cols int32 [cols_capacity] (device, caller-owned).  One kernel on
 * `stream`.  Rows past cols_capacity are cut and XGR_DEV_CAPACITY is set in
 * the device status word.  For callers that want the rows themselves (a
 * check, or the CSR input of xgr_beam_topk_noalloc). */
xgr_status xgr_mask_to_csr(xgr_ctx *ctx, const xgr_mask *mask, int32_t *d_row_ptr, int32_t *d_cols,
                           int64_t cols_capacity, xgr_stream_t stream);

/* Masked top-K beam selection with in-place rewiring (xGR 2.2 "Early sort
 * termination", 2.1 "In-place updates").  Vocabularies up to 32768 tokens
 * (xgr_create returns XGR_ERR_UNIMPLEMENTED above):
 *   d_scores fp32 [B][BW][V]  log-probs or logits (flags); rows of dead beams
 *                             are not read
 *   mask                      as returned by xgr_build_mask for this step (or
 *                             its rows written by xgr_mask_to_csr, kind CSR)
 *   d_parent, d_token int32 [B][BW], d_cum fp32 [B][BW], d_n_out int32 [B]:
 *     the new beams in rank order (slot = rank): higher score first, then
 *     lower parent, then lower token.  Score = fp32(cum[parent] + lp).
 * Each beam first keeps its top-K valid candidates; the best BW of their
 * union survive.  The context's ancestry (Unshared slot of every earlier
 * step), trie node, token history and cumulative score are rewired in place
 * to the new beams, and the current step advances. */
xgr_status xgr_beam_select(xgr_ctx *ctx, int32_t step, const float *d_scores, int32_t flags,
                           const xgr_mask *mask, int32_t *d_parent, int32_t *d_token,
                           float *d_cum, int32_t *d_n_out, xgr_stream_t stream);

/* Tokens chosen so far by each current beam: d_seq int32 [B][BW][S]; entries
 * past the decoded steps and rows of dead beams are -1. */
xgr_status xgr_get_sequences(xgr_ctx *ctx, int32_t *d_seq, xgr_stream_t stream);

/* Synchronises `stream`, returns the device status word in *host_code (0 when
 * clean) and clears it.  Returns XGR_ERR_DEVICE when the word was non-zero. */
xgr_status xgr_device_status(xgr_ctx *ctx, xgr_stream_t stream, int32_t *host_code);

/* Masked beam top-K for callers that cannot allocate device memory.  The
 * pages have no counterpart of this call: it exists for code that may not
 * call cudaMalloc or create a workspace (a host framework that owns every
 * device byte, a plugin that must not allocate after start-up).  It needs no
 * context and writes no beam state: given
 *   d_scores  fp32 [B][BW][V]   log-probs or logits (flags, as xgr_beam_select)
 *   d_cum     fp32 [B][BW]      cumulative score of each live beam
 *   d_n_live  int32 [B]         live beams per request
 *   the mask: d_bits (dense, uint32 [ceil(V/32)], first step: only beam 0 of
 *             each request is read) or, when d_bits is NULL, the CSR rows
 *             d_row_ptr [B*BW+1] / d_cols (as built by xgr_build_mask)
 * it writes d_parent, d_token, d_cum_out [B][BW] and d_n_out [B] exactly as
 * xgr_beam_select does (same order, same tie-break, same bits).
 * Allocation: none.  Its scratch is one static device array of 8 MiB per GPU
 * (held by every GPU that loads the library until the process exits).  After
 * 120 bytes per beam row (its log-sum-exp, counts, ordered head of 8 best
 * keys with their entries and its next key; 4 keys from BW = 1024 on), the
 * rest is shared by the requests as key buffers (8 bytes per CSR entry); a
 * call returns XGR_ERR_CAPACITY unless every request gets room for
 * max(V, 8*BW, 4096) entries (e.g. 8 requests x 128 beams get about 129000
 * each).  A request with more CSR entries than its share is still selected
 * exactly, from the scores, on a slower path.  V above 32768 returns
 * XGR_ERR_UNIMPLEMENTED (a score row is staged whole in shared memory).
 * The first call on a device looks the array up (cudaGetSymbolAddress) and
 * may set a kernel attribute, so make that first call before any stream capture.
 * All calls share the array: calls that overlap on the GPU race and must be
 * serialised by the caller.  NaN scores and out-of-range mask tokens are
 * skipped, as in the context path, but not reported: the kernels set bits in
 * a status word inside the static array that this call neither clears nor
 * reads (use the context path and xgr_device_status to diagnose such inputs).
 * The tensor arguments must be device memory of the stated element types;
 * the call cannot check that.  Host-side argument
 * errors return XGR_ERR_ARG / XGR_ERR_SHAPE; nothing is enqueued then. */
xgr_status xgr_beam_topk_noalloc(int32_t n_requests, int32_t beam_width, int32_t top_k,
                                 int32_t vocab, const float *d_scores, int32_t flags,
                                 const float *d_cum, const int32_t *d_n_live,
                                 const uint32_t *d_bits, const int32_t *d_row_ptr,
                                 const int32_t *d_cols, int32_t *d_parent, int32_t *d_token,
                                 float *d_cum_out, int32_t *d_n_out, xgr_stream_t stream);

/* ---------------------------------------------------------------- whole-decode graph
 * xGR page, 2.3 xSchedule: "Graph-based execution" (a decode's device work is
 * captured in a static graph and dispatched in one go) and "Dynamic batching
 * and multi-stream" (independent request groups on their own streams).  One
 * graph runs a whole decode of n_groups request groups, each with its own
 * context: per group, xgr_begin, then for s = 0 .. steps-1 xgr_build_mask,
 * xgr_decode_step and xgr_beam_select -- on a stream of its own, forked from
 * and joined back to the stream the graph is launched on, so one group's
 * attention may run beside another group's selection (inside a group every
 * kernel follows the one before through a programmatic dependent launch).
 *
 * A group (all device pointers caller-owned and fixed for the graph's life):
 *   ctx          its context: trie built, the requests' KV prefilled; no two
 *                groups may share one
 *   n_requests   xgr_begin's n_requests
 *   score_flags  XGR_SCORES_LOGPROB or XGR_SCORES_LOGITS
 *   d_q, d_k_new, d_v_new, d_scores: HOST arrays of `steps` device pointers,
 *                step s's inputs as xgr_decode_step / xgr_beam_select take
 *                them (read at creation only; the pointers are baked in)
 *   d_out, d_lse, d_parent, d_token, d_cum, d_n_out: the step outputs,
 *                rewritten every step (the last step's remain)
 * Creation runs the decode once eagerly (planning, launch attributes and
 * tensor maps are set up then; its results are left in the output buffers),
 * then captures and instantiates it; every launch re-runs it from xgr_begin on
 * the inputs' current contents.  Host-side errors of any of the calls above
 * are returned as they are; XGR_ERR_ARG for a NULL or repeated context, NULL
 * pointer arrays, n_groups outside [1, 64] or steps < 1.  Each context's host
 * state afterwards is that of a finished decode (xgr_get_sequences works; a
 * new decode through the calls above starts with xgr_begin). */
typedef struct {
    xgr_ctx *ctx;
    int32_t n_requests;
    int32_t score_flags;
    const void *const *d_q;
    const void *const *d_k_new;
    const void *const *d_v_new;
    const float *const *d_scores;
    void *d_out;
    float *d_lse;
    int32_t *d_parent;
    int32_t *d_token;
    float *d_cum;
    int32_t *d_n_out;
} xgr_decode_group;

typedef struct xgr_decode_graph xgr_decode_graph;

xgr_status xgr_decode_graph_create(const xgr_decode_group *groups, int32_t n_groups, int32_t steps,
                                   xgr_decode_graph **out);
/* Enqueues the whole decode on `stream` (one graph launch). */
xgr_status xgr_decode_graph_launch(xgr_decode_graph *graph, xgr_stream_t stream);
/* Kernel launches of one decode (the graph's kernel nodes). */
xgr_status xgr_decode_graph_kernels(const xgr_decode_graph *graph, int32_t *n_kernels);
/* Frees the graph (not the contexts or buffers); the caller makes sure no
 * launch of it is still running. */
xgr_status xgr_decode_graph_destroy(xgr_decode_graph *graph);

#ifdef __cplusplus
}
#endif

#endif /* XGR_H_ */

// kernels.h -- argument blocks and launchers of the device kernels (internal).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace xgr {

// Shared stage, few rows per work item (SIMT).
struct SmallArgs {
    const WorkItem *items;
    const int32_t *members;
    const __nv_bfloat16 *q;        // [B][BW][Hq][D]
    const __nv_bfloat16 *kstore;   // [Hkv][kv_tokens][D]
    const __nv_bfloat16 *vstore;
    int64_t kv_tokens;
    Dims dims;
    int nb;                        // beams per request of the plan (1 at step 0, BW after)
    const int32_t *n_live;
    Partials part;
};
cudaError_t launch_attn_small(const SmallArgs &a, int n_items, cudaStream_t st);

// Shared stage on the tensor cores: 128-row tiles, D = 128, TMA-fed K/V.
struct TcArgs {
    const WorkItem *items;
    const int32_t *members;
    const __nv_bfloat16 *q;        // [B][BW][Hq][D]
    int64_t kv_tokens;
    Dims dims;
    int nb;
    const int32_t *n_live;
    Partials part;
    int32_t *status;
    // fused epilogue of final items (Unshared stage, Merging stage, append)
    const __nv_bfloat16 *k_new;    // [B][BW][Hkv][D]
    const __nv_bfloat16 *v_new;
    __nv_bfloat16 *pool_k;         // [S][Bcap][BW][Hkv][D]
    __nv_bfloat16 *pool_v;
    __nv_bfloat16 *out;            // [B][BW][Hq][D]
    float *lse;                    // [B][BW][Hq]
    BeamState st;
    int Bcap;
    int step;
    int shared_o;                  // one O for both softmax warpgroups and three S buffers (the
                                   //   launch's items are short), else an O per warpgroup
};
// 2-D tensor map over a [rows][128] bf16 store, 64 x 128 boxes, 128-byte swizzle.
cudaError_t make_kv_tensor_map(CUtensorMap *map, const void *base, int64_t rows);
// 3-D tensor map over q [beam rows][Hq][128] bf16 with boxes 64 x G x (128 / G)
cudaError_t make_q_tensor_map(CUtensorMap *map, const void *q, int64_t beam_rows, int Hq, int G);
cudaError_t launch_attn_tc(const CUtensorMap &tmk, const CUtensorMap &tmv, const CUtensorMap &tmq,
                           const TcArgs &a, int n_items, cudaStream_t st);

// Unshared stage + Merging stage (+ append of this step's k/v).
struct MergeArgs {
    const __nv_bfloat16 *q;        // [B][BW][Hq][D]
    const __nv_bfloat16 *k_new;    // [B][BW][Hkv][D]
    const __nv_bfloat16 *v_new;
    __nv_bfloat16 *pool_k;         // [S][Bcap][BW][Hkv][D]
    __nv_bfloat16 *pool_v;
    __nv_bfloat16 *out;            // [B][BW][Hq][D]
    float *lse;                    // [B][BW][Hq]
    BeamState st;
    Dims dims;
    int Bcap;
    int step;
    const int32_t *n_slots;        // [B] partial slots of each request; -1: done by a fused item
    Partials part;
};
cudaError_t launch_attn_merge(const MergeArgs &a, cudaStream_t st);

// Beam state reset of xgr_begin.
// mask_sync: the mask builder's look-back words [Bcap] and ticket, zeroed here
// sel_ticket: the selection's tickets [Bcap], zeroed here
cudaError_t launch_begin(BeamState st, Dims dm, int Bcap, int all_live, uint64_t *mask_sync,
                         cudaStream_t s);

// Sparse masks of steps >= 1: one CSR row per beam.
struct MaskArgs {
    BeamState st;
    TrieView trie;
    Dims dims;
    int step;
    int32_t *row_ptr;   // [B*BW + 1]
    int32_t *cols;      // [cap]
    int64_t cap;
    uint64_t *flags;    // [Bcap] published request totals (zero between calls)
    uint32_t *ticket;   // [2]: CTAs done, CTAs started (zero between calls)
};
// parts: CTAs per request that share the copy of its children
cudaError_t launch_build_mask(const MaskArgs &a, int parts, cudaStream_t s);

// Beam selection (+ in-place rewiring of the context's beam state).
struct SelectArgs {
    const float *cum;           // [B][BW] cumulative scores before this step
    const int32_t *n_live;      // [B] live beams before this step
    int32_t *status;            // device status word
    int rewire;                 // 1: rewrite st (anc, seq, node, cum, n_live) in place
    BeamState st;
    TrieView trie;
    Dims dims;
    int step;
    int logits;                 // XGR_SCORES_LOGITS
    const float *scores;        // [B][BW][V]
    int dense;                  // mask kind (dense: only beam 0 of each request is read)
    const uint32_t *bits;
    // sparse steps: mask_kind XGR_MASK_CSR (row_ptr, cols), XGR_MASK_TRIE_ROWS
    // (row_node, node_ptr, node_tok) or XGR_MASK_NODE_BITS (row_node, node_ptr,
    // node_bits with n_words words per node)
    int mask_kind;
    const int32_t *row_ptr;
    const int32_t *cols;
    const int32_t *row_node;    // [B*BW] trie node of each row
    const int32_t *node_ptr;    // [n_nodes+1] child range of each node of the level
    const int32_t *node_tok;    // the level's child tokens
    const uint32_t *node_bits;  // [n_nodes][n_words]
    int32_t n_nodes;
    int32_t n_words;
    int32_t row_stride;         // most valid tokens of one row (TRIE_ROWS / NODE_BITS entry stride)
    // scratch (select_scratch_carve)
    float *row_lse;             // [B][BW] each live row's log-sum-exp (logits mode)
    int32_t *row_cnt;           // [B][BW] valid candidates of each row
    int32_t *row_len;           // [B][BW] mask entries of each row
    int32_t *row_cb;            // [B][BW] first trie child of each row's node (-1: none)
    uint64_t *head_k;           // [B][BW][m] each beam's m best keys, ascending (kNoKey pads)
    int32_t *head_e;            // [B][BW][m] their CSR entries (relative to the request)
    uint64_t *head_next;        // [B][BW] each row's (m+1)-th best key (kNoKey: none)
    int head_m;                 // m
    uint64_t *keys;             // [B][key_cap] key of each CSR entry (relative to the request)
    int64_t key_cap;
    int prep_early;             // the kernel before writes no beam state: the mask lookups may
                                //   run before the programmatic-launch wait
    int sp_parts;               // set by the launcher: CTAs per request of the sparse kernel
    int sp_rows;                //   and the beams each of them takes (one per warp)
    int num_sms;                // SMs of the device
    int32_t *parent;            // outputs [B][BW]
    int32_t *token;
    float *cum_out;
    int32_t *n_out;             // [B]
};
// Largest vocabulary of the selection: a score row is staged whole in shared memory.
constexpr int kSelectMaxVocab = 32768;
// Scratch of the selection for B requests of BW beams: per beam row its
// log-sum-exp, valid-candidate count, entry count, first trie child and head
// (its m best keys and their entries), a ticket per request, and the key
// buffer [B][key_cap] (CSR masks: entry e of the request at e - row_ptr[r*BW];
// node masks: entry j of beam b at b * row_stride + j; a request whose CSR
// entries exceed key_cap takes the exact fallback over the scores).
// Everything read is written by the same call first, except the tickets,
// which must be zero before a call (xgr_begin zeroes them, each call leaves
// them zero).
int select_head_m(int BW);
size_t select_scratch_bytes(int B, int BW, int64_t key_cap);
void select_scratch_carve(uint8_t *base, int B, int BW, int64_t key_cap, SelectArgs &a);
cudaError_t launch_beam_select(const SelectArgs &a, cudaStream_t s);

cudaError_t launch_get_sequences(BeamState st, Dims dm, int32_t *seq, cudaStream_t s);

// ---- the per-beam comparison path (attn_per_beam.cu)
constexpr int kPerBeamBlock = 16;   // tokens of a beam's private block (>= kMaxSteps)
struct PerBeamArgs {
    const __nv_bfloat16 *q;        // [B][BW][Hq][D]
    const __nv_bfloat16 *k_new;    // [B][BW][Hkv][D]
    const __nv_bfloat16 *v_new;
    const __nv_bfloat16 *kstore;   // [Hkv][kv_tokens][D]
    const __nv_bfloat16 *vstore;
    __nv_bfloat16 *blk_k;          // [2][Bcap][BW][Hkv][kPerBeamBlock][D] (step parity first)
    __nv_bfloat16 *blk_v;
    __nv_bfloat16 *out;            // [B][BW][Hq][D]
    float *lse;                    // [B][BW][Hq]
    const int32_t *req_seg;        // [B][4]: prompt offset, length, suffix offset, length
    const int32_t *n_live;         // [B]
    BeamState st;
    int32_t *status;
    Dims dims;
    int Bcap, step;
    int64_t kv_tokens;
};
cudaError_t launch_per_beam(const PerBeamArgs &a, cudaStream_t st);
size_t per_beam_block_bytes(int Bcap, int BW, int Hkv, int D);

// Launches `kernel` on `s` with programmatic stream serialization: the
// kernel may start while the previous kernel in the stream is still running,
// so it must call griddep_wait() before it reads or writes anything that
// kernel (or an earlier one) produces or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

}  // namespace xgr

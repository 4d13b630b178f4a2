// common.cuh -- device helpers and the structures shared by the kernels and
// the host glue of libxgr.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "../../include/xgr.h"

namespace xgr {

constexpr int kMaxSteps = 8;          // item length / decode steps supported
constexpr int kSmallRows = 16;        // row cap of one small-row attention work item
constexpr int kTcRows = 128;          // row tile of the tensor-core Shared stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Problem dimensions fixed at xgr_create (B = requests of the current decode).
struct Dims {
    int B, BW, K, S, Hq, Hkv, D, V, G;
};

// Per-request beam state in the workspace, rewired in place by the selection.
struct BeamState {
    int32_t *status;   // device status word (XGR_DEV_* bits)
    int32_t *n_live;   // [B]
    float *cum;        // [B][BW]   cumulative fp32 score of each beam
    int32_t *node;     // [B][BW]   trie node of each beam at the current level
    int32_t *anc;      // [B][BW][S] Unshared slot of step i for the beam (direct indices)
    int32_t *seq;      // [B][BW][S] token chosen at step i
};

// Level-wise CSR trie: node n of level l has children tok[l][ptr[l][n] .. ptr[l][n+1]),
// ascending; the child at position p of tok[l] is node p of level l+1.
struct TrieView {
    const int32_t *ptr[kMaxSteps];
    const int32_t *tok[kMaxSteps];
    int32_t n_nodes[kMaxSteps + 1];
    const uint32_t *root_bits;   // dense mask of step 0
    int32_t levels;
};

// One unit of Shared-stage work: a kv head of one KV segment (a shared prompt
// prefix or a request suffix), a range of its rows, and a range of its keys.
// Row i of a segment (0-based) maps to member m = i / (nb*G), beam
// b = (i / G) % nb, query head g*G + i % G, where nb is the beams per request
// of the plan (1 at step 0, BW afterwards) and members are requests.
struct WorkItem {
    int32_t kv_off;      // token offset of the segment in the KV store
    int32_t key_begin;   // [key_begin, key_end) within the segment
    int32_t key_end;
    int32_t g;           // kv head
    int32_t member_off;  // into the plan's member list
    int32_t n_members;
    int32_t row_begin;   // first segment row of this item
    int32_t n_rows;      // rows of this item
    int32_t slot;        // partial slot this item writes for its rows
    int32_t flags;       // bit 0: final -- the item covers its requests' only KV segment
                         // whole, so it also runs the Unshared and Merging stages;
                         // bit 1: its query rows form one TMA box (a single request);
                         // bit 2: zero fill -- no attention: O = 0 and LSE = -inf for
                         // beams [row_begin, row_begin + n_rows) of request r0, every
                         // query head (beams not live yet at step 0)
    int32_t r0;          // the item's first member request
    int32_t pad;
};
static_assert(sizeof(WorkItem) == 48, "WorkItem layout");

// Split-K partial results: O (unnormalised, relative to m) and (m, l) per row,
// m in log2 units of the scaled score, l = sum exp2(s*log2e*scale - m).
struct Partials {
    float *o;        // [slots][rows][D]
    float2 *ml;      // [slots][rows]
    int64_t rows;    // B*BW*Hq of the workspace capacity
};

// Host-side diagnostics on stderr, only when the environment sets XGR_DEBUG.
inline void debug_log(const char *fmt, ...) {
    static const bool on = getenv("XGR_DEBUG") != nullptr;
    if (!on) return;
    va_list ap;
    va_start(ap, fmt);
    fprintf(stderr, "[xgr] ");
    vfprintf(stderr, fmt, ap);
    fprintf(stderr, "\n");
    va_end(ap);
}

__device__ __forceinline__ void set_status(int32_t *status, int32_t bit) {
    atomicOr(status, bit);
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// 8 bf16 packed in a uint4 -> 8 floats
__device__ __forceinline__ void unpack8(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---- composite selection keys -------------------------------------------
// Ascending order of the 64-bit key == rank order: higher score first, then
// lower parent beam, then lower token.  High word: the score's bits mapped to
// an order-reversing unsigned integer; low word: parent * V + token.
__device__ __forceinline__ uint32_t score_to_desc_bits(float x) {
    uint32_t u = __float_as_uint(x);
    uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // monotone increasing
    return ~asc;                                                   // monotone decreasing
}

__device__ __forceinline__ float desc_bits_to_score(uint32_t d) {
    uint32_t asc = ~d;
    uint32_t u = (asc & 0x80000000u) ? (asc & 0x7fffffffu) : ~asc;
    return __uint_as_float(u);
}

constexpr uint64_t kNoKey = ~0ull;   // sorts after every real key

}  // namespace xgr

// select.cu -- masked beam Top-K with a global threshold (early termination)
// and the in-place rewiring of the beam state.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"):
//  2.2 "Valid-path constraint" / "Hybrid dense/sparse storage": candidates
//      come only from the valid-item vocabulary -- a dense bitset of first
//      tokens at step 0, sparse rows (each beam's sorted trie children) later.
//      "Early sort termination": the page orders each beam's candidates and
//      cuts every list at a global min-heap threshold.  Here the threshold tau
//      is the worst of the live beams' best keys: with all BW beams live these
//      are BW real candidates, so every one of the BW winners ranks at or
//      above tau, and only the candidates at or above it ("survivors") reach
//      the exact selection.
//  2.1 "In-place updates": the beam state (ancestry slots, trie node, token
//      history, cumulative score) is rewritten in place; every row a new beam
//      reads is staged in shared memory before any row is written.
//
// Keys: 64-bit integers whose ascending order is the rank order (higher fp32
// score, then lower parent beam, then lower token), so every comparison is an
// exact integer comparison and ties resolve identically everywhere.
//
// Kernels:
//  * dense mask (one live beam per request, step 0): select_dense_kernel, one
//    CTA per request, stages the beam's score row with one bulk copy, takes its
//    log-sum-exp (logits), computes every token's key once into registers and
//    radix-selects the best BW there.
//  * sparse (CSR) masks: select_rows_kernel, one persistent 1024-thread CTA per
//    SM over a contiguous block of beam rows: the rows' metadata and CSR tokens
//    in two round trips, the score rows (logits mode) through bulk-copy slots,
//    eight 128-thread groups on eight rows at a time; per row the log-sum-exp,
//    each entry's key beside its CSR position and the row's best key.  Then one
//    of two picks: select_pick_one_kernel (one CTA per request, when the
//    request's pool fits its registers and shared memory) radix-selects the
//    pool directly; select_pick_kernel (a few CTAs per request) reduces tau
//    from the best keys, filters its slices of the request's keys and appends
//    the survivors, and the request's last CTA to finish (an atomic ticket the
//    rows kernel resets) selects among them.  Both end in finish_request: the
//    ordering, the outputs and the rewiring.
#include <algorithm>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr int kDenseThreads = 1024;
constexpr int kPickThreads = 512;
constexpr int kPickKeys = 4096;    // keys one pick CTA filters per slice (8 per thread)
constexpr int kSmemSurv = 4096;    // survivors selected in shared memory
constexpr int kMaxPickParts = 16;

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// key of (beam b, token t): one fp32 add of the beam's cumulative score and
// the token's log-prob; -0.0 is canonical +0.0; NaN is reported and skipped
__device__ __forceinline__ bool make_key(float cum, float lp, int b, int t, int V, int32_t *status,
                                         uint64_t &key) {
    float k = cum + lp;
    if (isnan(k)) {
        set_status(status, XGR_DEV_NAN);
        return false;
    }
    if (k == 0.f) k = 0.f;
    key = ((uint64_t)score_to_desc_bits(k) << 32) | (uint32_t)(b * V + t);
    return true;
}

__device__ __forceinline__ uint64_t warp_min_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t u = __shfl_xor_sync(0xffffffffu, v, o);
        v = u < v ? u : v;
    }
    return v;
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t u = __shfl_xor_sync(0xffffffffu, v, o);
        v = u > v ? u : v;
    }
    return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// block-wide reductions; every thread gets the result; red holds 32 entries
__device__ uint64_t block_min_u64(uint64_t v, uint64_t *red) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
    v = warp_min_u64(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = warp_min_u64(lane < nw ? red[lane] : kNoKey);
    __syncthreads();
    return v;
}
__device__ uint64_t block_max_u64(uint64_t v, uint64_t *red) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
    v = warp_max_u64(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = warp_max_u64(lane < nw ? red[lane] : 0);
    __syncthreads();
    return v;
}
__device__ int block_sum_int(int v, int *red) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
    v = warp_sum_int(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = warp_sum_int(lane < nw ? red[lane] : 0);
    __syncthreads();
    return v;
}
// block-wide exclusive scan of one int per thread; *total gets the block sum
__device__ int block_exclusive_scan_int(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int wt = lane < nw ? warp_tot[lane] : 0, wi = wt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
    }
    const int before = __shfl_sync(0xffffffffu, wi - wt, warp);   // warps before this one
    *total = __shfl_sync(0xffffffffu, wi, 31);
    __syncthreads();
    return before + incl - v;
}

// A set of threads that reduce together: the whole block (barrier 0) or a
// group of warps with its own named barrier.
struct Group {
    int bar, n, t;   // barrier id (0: __syncthreads), threads, this thread's index in the group
    __device__ __forceinline__ void sync() const {
        if (bar == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(n) : "memory");
    }
};
__device__ __forceinline__ Group whole_block() { return Group{0, (int)blockDim.x, (int)threadIdx.x}; }

// log-sum-exp of the values x[i], i < n, in shared memory, over a group: the
// row max first, then the sum of exponentials, each reduced without
// branches; reports NaN.  red: 33 floats of shared memory for the group.
// log-sum-exp of x[0..n) (shared memory) over a group, in one pass: each thread
// keeps its own (max, sum of 2^((x - max) log2 e)) over blocks of 16 values
// (16-byte loads when x is 16-byte aligned), rescaling its sum when its max
// grows; the pairs are then combined across the group.  red holds 2 floats per
// warp of the group.
__device__ __forceinline__ void lse_pair_merge(float &m, float &s, float m2, float s2) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;   // both empty
    s = (m == -INFINITY ? 0.f : s * ex2f((m - M) * kLog2e)) +
        (m2 == -INFINITY ? 0.f : s2 * ex2f((m2 - M) * kLog2e));
    m = M;
}
__device__ float group_lse(const float *x, int n, float *red, int32_t *status, const Group &g) {
    const int lane = g.t % 32, w = g.t / 32, nw = g.n / 32;
    float m = -INFINITY, s = 0.f;
    bool nan = false;
    auto fold = [&](const float *v, int k) {   // k values already in registers
        float mv = -INFINITY;
        for (int e = 0; e < k; ++e) {
            nan |= isnan(v[e]);
            mv = fmaxf(mv, v[e]);
        }
        if (mv > m) {
            s = m == -INFINITY ? 0.f : s * ex2f((m - mv) * kLog2e);
            m = mv;
        }
        if (m != -INFINITY) {
            const float mk = m * kLog2e;
            for (int e = 0; e < k; ++e) s += ex2f(fmaf(v[e], kLog2e, -mk));
        }
    };
    const int n4 = (reinterpret_cast<uintptr_t>(x) & 15) == 0 ? n / 4 : 0;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    for (int b = 0; b < n4; b += 4 * g.n) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = b + k * g.n + g.t;
            const float4 q = i < n4 ? x4[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            v[4 * k] = q.x;
            v[4 * k + 1] = q.y;
            v[4 * k + 2] = q.z;
            v[4 * k + 3] = q.w;
        }
        fold(v, 16);
    }
    for (int i = 4 * n4 + g.t; i < n; i += g.n) fold(x + i, 1);
    if (nan) set_status(status, XGR_DEV_NAN);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_pair_merge(m, s, m2, s2);
    }
    if (lane == 0) {
        red[2 * w] = m;
        red[2 * w + 1] = s;
    }
    g.sync();
    m = red[0];
    s = red[1];
    for (int k = 1; k < nw; ++k) lse_pair_merge(m, s, red[2 * k], red[2 * k + 1]);
    g.sync();   // red is reused
    return m + logf(s);
}
__device__ float block_lse(const float *x, int n, float *red, int32_t *status) {
    return group_lse(x, n, red, status, whole_block());
}
__device__ uint64_t group_min_u64(uint64_t v, uint64_t *red, const Group &g) {
    const int lane = g.t % 32, w = g.t / 32, nw = g.n / 32;
    v = warp_min_u64(v);
    if (lane == 0) red[w] = v;
    g.sync();
    v = red[0];
    for (int k = 1; k < nw; ++k) v = red[k] < v ? red[k] : v;
    g.sync();
    return v;
}

// One radix pass's bucket search over the digit of `width` bits at `shift`:
// the bin holding the k_rem-th key, by a one-warp scan of the 256-bin
// histogram.  Returns whether the digit is resolved exactly (the bin's keys are
// all taken); updates prefix, mask and k_rem.
__device__ __forceinline__ bool radix_bucket(const int *hist, int *sc, int shift, int width, int &k_rem,
                                             uint64_t &prefix, uint64_t &mask) {
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int h[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            h[i] = hist[lane * 8 + i];
            sum += h[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        int acc = incl - sum;   // keys in the bins before this lane's 8
        // the lane whose range crosses k_rem owns the bucket
        if (acc < k_rem && acc + sum >= k_rem) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (acc + h[i] >= k_rem) {
                    sc[0] = lane * 8 + i;
                    sc[1] = h[i] - (k_rem - acc);   // 0 <=> the whole bucket is taken
                    sc[2] = k_rem - acc;
                    break;
                }
                acc += h[i];
            }
        }
    }
    __syncthreads();
    const int d = sc[0], surplus = sc[1];
    k_rem = sc[2];
    prefix |= (uint64_t)d << shift;
    mask |= ((1ull << width) - 1ull) << shift;
    __syncthreads();
    return surplus == 0;
}

// add one key (if `in`) to its bin; lanes whose keys share a bin add them with
// one atomic (keys cluster in few bins in the leading digits).  All lanes call it.
__device__ __forceinline__ void hist_add(int *hist, bool in, uint64_t key, int shift) {
    const int bin = in ? (int)((key >> shift) & 255) : 256;
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

// Exact block-wide radix select over E candidates given by `cand(e, key)`
// (false for a non-candidate).  Keys are unique.  On return exactly `want`
// candidates satisfy (key & mask) <= prefix (want <= number of candidates).
// hist: 256 ints of shared memory; sc: 3 shared ints.
template <class Cand>
__device__ void radix_select(const Cand &cand, int64_t E, int want, int *hist, int *sc,
                             uint64_t &prefix, uint64_t &mask) {
    prefix = 0;
    mask = 0;
    int k_rem = want;
    const int64_t E_up = (E + blockDim.x - 1) / blockDim.x * blockDim.x;   // same trip count for all
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int64_t e = threadIdx.x; e < E_up; e += blockDim.x) {
            uint64_t key = 0;
            const bool in = e < E && cand(e, key) && (key & mask) == prefix;
            hist_add(hist, in, key, shift);
        }
        __syncthreads();
        if (radix_bucket(hist, sc, shift, 8, k_rem, prefix, mask)) break;
    }
}

// The same over keys held in registers (KPT per thread, kNoKey for none) plus
// an optional tail of n_tail keys in shared memory, with 11-bit digits (2048
// bins, bucket found by a block-wide scan: half the passes of 8-bit digits).
// The digits start at the highest bit where the smallest and largest key
// differ (the bits above are common to all keys), so the first histogram
// already spreads the keys over many bins and the shared-memory atomics do not
// pile onto a few counters.  hist: kWideBins ints; scan_w: 32 ints; red: 32
// u64 of shared memory.
constexpr int kWideBits = 11, kWideBins = 1 << kWideBits;

template <int KPT>
__device__ void radix_select_regs(const uint64_t (&k)[KPT], int want, int *hist, int *sc, int *scan_w,
                                  uint64_t *red, uint64_t &prefix, uint64_t &mask,
                                  const uint64_t *tail = nullptr, int n_tail = 0) {
    uint64_t lo = kNoKey, hi = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u)
        if (k[u] != kNoKey) {
            lo = k[u] < lo ? k[u] : lo;
            hi = k[u] > hi ? k[u] : hi;
        }
    for (int i = threadIdx.x; i < n_tail; i += blockDim.x)
        if (tail[i] != kNoKey) {
            lo = tail[i] < lo ? tail[i] : lo;
            hi = tail[i] > hi ? tail[i] : hi;
        }
    lo = block_min_u64(lo, red);
    hi = block_max_u64(hi, red);
    const uint64_t diff = lo ^ hi;
    if (diff == 0) {   // one distinct key (keys are unique: one candidate)
        prefix = lo;
        mask = ~0ull;
        return;
    }
    int pos = 64 - __clzll((long long)diff);   // bits [pos, 64) are common to every key
    mask = pos == 64 ? 0ull : ~((1ull << pos) - 1ull);
    prefix = lo & mask;
    int k_rem = want;
    const int bpt = kWideBins / blockDim.x;   // bins per thread in the bucket scan (1, 2 or 4)
    while (pos > 0) {
        const int shift = pos > kWideBits ? pos - kWideBits : 0, width = pos - shift;
        const uint64_t dmask = (1ull << width) - 1ull;
        for (int i = threadIdx.x; i < kWideBins; i += blockDim.x) hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            if (k[u] != kNoKey && (k[u] & mask) == prefix) atomicAdd(&hist[(k[u] >> shift) & dmask], 1);
        for (int i = threadIdx.x; i < n_tail; i += blockDim.x) {
            const uint64_t key = tail[i];
            if (key != kNoKey && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
        }
        __syncthreads();
        // the bin holding the k_rem-th key: thread t scans bins [t*bpt, t*bpt + bpt)
        int h[4] = {0, 0, 0, 0}, sum = 0;
        for (int j = 0; j < bpt; ++j) {
            h[j] = hist[threadIdx.x * bpt + j];
            sum += h[j];
        }
        int total;
        int acc = block_exclusive_scan_int(sum, scan_w, &total);
        if (acc < k_rem && acc + sum >= k_rem) {
            for (int j = 0; j < bpt; ++j) {
                if (acc + h[j] >= k_rem) {
                    sc[0] = threadIdx.x * bpt + j;
                    sc[1] = h[j] - (k_rem - acc);   // 0 <=> the whole bucket is taken
                    sc[2] = k_rem - acc;
                    break;
                }
                acc += h[j];
            }
        }
        __syncthreads();
        const int d = sc[0], surplus = sc[1];
        k_rem = sc[2];
        prefix |= (uint64_t)d << shift;
        mask |= dmask << shift;
        __syncthreads();
        if (surplus == 0) break;
        pos = shift;
    }
}

// ---- candidate spaces

// the dense first step: token t of beam 0, score row staged in shared memory
struct DenseCand {
    const float *x;
    const uint32_t *bits;
    float cum, lse;
    int V, logits;
    int32_t *status;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        const int t = (int)e;
        if (!((bits[t >> 5] >> (t & 31)) & 1u)) return false;
        float lp = x[t];
        if (logits) lp -= lse;
        return make_key(cum, lp, 0, t, V, status, key);
    }
};

// survivor keys in shared memory (kGlobal = false) or, written by other CTAs
// of the same launch, in global memory (read through L2)
template <bool kGlobal>
struct ListCand {
    const uint64_t *k;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        key = kGlobal ? __ldcg(k + e) : k[e];
        return true;
    }
};

// the request's key buffer, restricted to the survivors of tau
struct KeyCand {
    const uint64_t *k;
    uint64_t tau;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        key = __ldcg(k + e);
        return key != kNoKey && key <= tau;
    }
};

// every CSR entry of the request's live beams, keys recomputed from the scores
// (rp = per-beam entry offsets relative to the request's first entry)
struct ReqCand {
    const float *x;          // scores of the request's first row
    const int32_t *cols;     // CSR entries of the request's first row
    const int *rp;           // [n+1] in shared memory
    const float *cum, *lse;  // [n] in shared memory
    int32_t *status;
    int n, logits, V;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        int lo = 0, hi = n;   // beam b with rp[b] <= e < rp[b+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (rp[mid] <= e) lo = mid; else hi = mid;
        }
        const int b = lo, t = cols[e];
        if (t < 0 || t >= V) return false;
        float lp = x[(int64_t)b * V + t];
        if (logits) lp -= lse[b];
        return make_key(cum[b], lp, b, t, V, status, key);
    }
};

__device__ int find_child(const TrieView &tr, int level, int node, int t) {
    if (level >= tr.levels || node < 0 || node >= tr.n_nodes[level]) return -1;
    int lo = tr.ptr[level][node];
    const int end = tr.ptr[level][node + 1];
    int hi = end;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (tr.tok[level][mid] < t) lo = mid + 1; else hi = mid;
    }
    return (lo < end && tr.tok[level][lo] == t) ? lo : -1;
}

// ---- shared memory of the finishing CTA (carved from dynamic shared memory)

struct FinishSmem {
    uint64_t *win_k;   // [BW] winners (unordered)
    int *win_e;        // [BW] their entry: CSR entry relative to the request (sparse) or token
    int *rank;         // [BW]
    int *rp;           // [BW+1] sparse: entry offset of each live beam
    int *st_node;      // [n_stage] staged old rows (rewiring)
    int *st_anc;       // [n_stage*S]
    int *st_seq;       // [n_stage*S]
    int *cb, *ce;      // [n_stage] sparse: child range of each staged row's trie node
    uint32_t *root;    // dense: [nw] root-children bitset, [nw] prefix popcounts
    int *cnt;          // winners appended
};

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~(size_t)15; }

// n_stage: old rows staged for the rewiring (the live beams: BW, or 1 for a dense step)
__host__ __device__ inline size_t finish_bytes(int BW, int n_stage, int S, int nw_root) {
    return al16((size_t)BW * 8) + 2 * al16((size_t)BW * 4) + al16((size_t)(BW + 1) * 4) +
           3 * al16((size_t)n_stage * 4) + 2 * al16((size_t)n_stage * S * 4) + al16((size_t)nw_root * 8) +
           16;
}

__device__ FinishSmem carve_finish(uint8_t *p, int BW, int n_stage, int S, int nw_root) {
    FinishSmem f;
    f.win_k = reinterpret_cast<uint64_t *>(p);
    p += al16((size_t)BW * 8);
    f.win_e = reinterpret_cast<int *>(p);
    p += al16((size_t)BW * 4);
    f.rank = reinterpret_cast<int *>(p);
    p += al16((size_t)BW * 4);
    f.rp = reinterpret_cast<int *>(p);
    p += al16((size_t)(BW + 1) * 4);
    f.st_node = reinterpret_cast<int *>(p);
    p += al16((size_t)n_stage * 4);
    f.st_anc = reinterpret_cast<int *>(p);
    p += al16((size_t)n_stage * S * 4);
    f.st_seq = reinterpret_cast<int *>(p);
    p += al16((size_t)n_stage * S * 4);
    f.cb = reinterpret_cast<int *>(p);
    p += al16((size_t)n_stage * 4);
    f.ce = reinterpret_cast<int *>(p);
    p += al16((size_t)n_stage * 4);
    f.root = reinterpret_cast<uint32_t *>(p);
    p += al16((size_t)nw_root * 8);
    f.cnt = reinterpret_cast<int *>(p);
    return f;
}

// stage the request's old beam rows (n live beams) for the rewiring
__device__ void stage_rows(const SelectArgs &a, int64_t rb, int n, const FinishSmem &f) {
    const int S = a.dims.S;
    for (int i = threadIdx.x; i < n * S; i += blockDim.x) {
        f.st_anc[i] = a.st.anc[rb * S + i];
        f.st_seq[i] = a.st.seq[rb * S + i];
    }
    for (int b = threadIdx.x; b < n; b += blockDim.x) f.st_node[b] = a.st.node[rb + b];
}

// child range of every staged row's trie node (sparse steps; after stage_rows)
__device__ void stage_children(const SelectArgs &a, int n, const FinishSmem &f) {
    const int s = a.step;
    for (int b = threadIdx.x; b < n; b += blockDim.x) {
        const int node = f.st_node[b];
        const bool ok = s < a.trie.levels && node >= 0 && node < a.trie.n_nodes[s];
        f.cb[b] = ok ? a.trie.ptr[s][node] : -1;
        f.ce[b] = ok ? a.trie.ptr[s][node + 1] : -1;
    }
}

// append the winners among the candidates [0, E) of `cand` ((key & mask) <= prefix)
template <class Cand, class Entry>
__device__ void collect(const Cand &cand, int64_t E, uint64_t prefix, uint64_t mask, int BW,
                        const Entry &entry, const FinishSmem &f) {
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x) {
        uint64_t key;
        if (cand(e, key) && (key & mask) <= prefix) {
            const int pos = atomicAdd(f.cnt, 1);
            if (pos < BW) {
                f.win_k[pos] = key;
                f.win_e[pos] = entry(e);
            }
        }
    }
}

// the same for keys held in registers (KPT per thread; entry(u) names key u's entry)
template <int KPT, class Entry>
__device__ void collect_regs(const uint64_t (&k)[KPT], uint64_t prefix, uint64_t mask, int BW,
                             const Entry &entry, const FinishSmem &f) {
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        if (k[u] != kNoKey && (k[u] & mask) <= prefix) {
            const int pos = atomicAdd(f.cnt, 1);
            if (pos < BW) {
                f.win_k[pos] = k[u];
                f.win_e[pos] = entry(u);
            }
        }
    }
}

// Rank the n_win winners (unique keys; a winner's rank is its number of better
// winners, counted by one warp per winner), write the outputs in rank order
// and, when a.rewire, rewrite the request's beam state in place.  The caller
// has staged the old rows (stage_rows) and rp / root.
__device__ void finish_request(const SelectArgs &a, int r, int n_win, const FinishSmem &f) {
    const Dims dm = a.dims;
    const int BW = dm.BW, S = dm.S, V = dm.V;
    const int64_t rb = (int64_t)r * BW;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nwarps = blockDim.x / 32;
    const int s = a.step;
    // sparse rewiring: each winner's trie child and the check of its token load
    // while the winners are ranked (winners i = threadIdx.x + u * blockDim.x)
    constexpr int kWinPerThread = 2;   // BW <= 1024 <= 2 * blockDim.x
    int child_c[kWinPerThread], child_t[kWinPerThread];
#pragma unroll
    for (int u = 0; u < kWinPerThread; ++u) {
        const int i = threadIdx.x + u * blockDim.x;
        child_c[u] = -1;
        child_t[u] = -1;
        if (!a.rewire || a.dense || i >= n_win) continue;
        const uint32_t lo = (uint32_t)f.win_k[i];
        const int p = (int)(lo / (uint32_t)V);
        if (f.cb[p] < 0) continue;
        const int c = f.cb[p] + (f.win_e[i] - f.rp[p]);
        if (c < f.ce[p]) {
            child_c[u] = c;
            child_t[u] = a.trie.tok[s][c];
        }
    }
    for (int i = warp; i < n_win; i += nwarps) {
        const uint64_t k = f.win_k[i];
        int c = 0;
        for (int j = lane; j < n_win; j += 32) c += f.win_k[j] < k;
        c = warp_sum_int(c);
        if (lane == 0) f.rank[i] = c;
    }
#pragma unroll
    for (int u = 0; u < kWinPerThread; ++u) {   // the checked child of winner i, in rank
        const int i = threadIdx.x + u * blockDim.x;
        if (i < n_win && !a.dense && a.rewire)
            f.win_e[i] = (child_c[u] >= 0 && child_t[u] == (int)((uint32_t)f.win_k[i] % (uint32_t)V)) ? child_c[u] : -1;
    }
    __syncthreads();   // every rank is written
    for (int i = threadIdx.x; i < BW; i += blockDim.x) {
        if (i < n_win) {
            const int nb = f.rank[i];
            const int64_t o = rb + nb;
            const uint64_t key = f.win_k[i];
            const uint32_t lo = (uint32_t)key;
            const int p = (int)(lo / (uint32_t)V), t = (int)(lo % (uint32_t)V);
            const float sc = desc_bits_to_score((uint32_t)(key >> 32));
            a.parent[o] = p;
            a.token[o] = t;
            a.cum_out[o] = sc;
            if (!a.rewire) continue;
            for (int j = 0; j < S; ++j) {
                int av = -1, sv = -1;
                if (j < s) {
                    av = f.st_anc[p * S + j];
                    sv = f.st_seq[p * S + j];
                } else if (j == s) {
                    av = p;    // the parent's own token of step s sits at slot (s, p)
                    sv = t;
                } else if (j == s + 1) {
                    av = nb;   // the new beam's token of step s+1 will sit at slot (s+1, nb)
                }
                a.st.anc[o * S + j] = av;
                a.st.seq[o * S + j] = sv;
            }
            // the trie child of the parent's node through token t
            int child = -1;
            const int node = f.st_node[p];
            if (a.dense) {
                if (s == 0 && node == 0 && a.trie.levels > 0 && a.trie.root_bits) {
                    // the root's children in trie order are its bitset in token order
                    const int nw = (V + 31) / 32;
                    const uint32_t w = f.root[t >> 5], bit = 1u << (t & 31);
                    if (w & bit) child = (int)f.root[nw + (t >> 5)] + __popc(w & (bit - 1u));
                } else {
                    child = find_child(a.trie, s, node, t);
                }
            } else {
                // the mask row of parent p lists its children in trie order, so
                // the entry index located the child (checked above)
                child = f.win_e[i];
            }
            if (child < 0) set_status(a.status, XGR_DEV_MASK);
            a.st.node[o] = child;
            a.st.cum[o] = sc;
        } else {
            const int64_t o = rb + i;
            a.parent[o] = -1;
            a.token[o] = -1;
            a.cum_out[o] = -INFINITY;
            if (!a.rewire) continue;
            for (int j = 0; j < S; ++j) {
                a.st.anc[o * S + j] = -1;
                a.st.seq[o * S + j] = -1;
            }
            a.st.node[o] = -1;
            a.st.cum[o] = -INFINITY;
        }
    }
    if (threadIdx.x == 0) {
        a.n_out[r] = n_win;
        if (a.rewire) a.st.n_live[r] = n_win;
    }
}

// ------------------------------------------------------------------ dense step

__host__ __device__ inline size_t dense_x_bytes(int V) { return al16((size_t)V * 4); }
__host__ __device__ inline size_t dense_bits_bytes(int V) { return al16((size_t)((V + 31) / 32) * 4); }

size_t dense_smem(const Dims &dm) {
    return dense_x_bytes(dm.V) + dense_bits_bytes(dm.V) + finish_bytes(dm.BW, 1, dm.S, (dm.V + 31) / 32);
}

__global__ void __launch_bounds__(kDenseThreads, 1) select_dense_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar_mem;
    __shared__ float red_f[72];
    __shared__ int red_i[32];
    __shared__ uint64_t red_k[32];
    __shared__ int hist[256];
    __shared__ int whist[kWideBins];
    __shared__ int sc[4];
    const Dims dm = a.dims;
    const int V = dm.V, BW = dm.BW, nw = (V + 31) / 32;
    const int r = blockIdx.x, tid = threadIdx.x;
    const int64_t rb = (int64_t)r * BW;
    float *x = reinterpret_cast<float *>(smem);
    uint32_t *bits = reinterpret_cast<uint32_t *>(smem + dense_x_bytes(V));
    const FinishSmem f = carve_finish(smem + dense_x_bytes(V) + dense_bits_bytes(V), BW, 1, dm.S, nw);
    const float *xg = a.scores + rb * V;   // beam 0 of request r
    const uint32_t bar = smem_u32(&bar_mem);
    const bool bulk = (V & 3) == 0 && (reinterpret_cast<uintptr_t>(xg) & 15) == 0;
    if (tid == 0) {
        *f.cnt = 0;
        if (bulk) {
            mbar_init(bar, 1);
            fence_mbar_init();
            mbar_expect_tx(bar, (uint32_t)V * 4u);
            bulk_g2s(smem_u32(x), xg, (uint32_t)V * 4u, bar);
        }
    }
    const int n = min(a.n_live[r], 1);
    const float cum = a.cum[rb];
    for (int w = tid; w < nw; w += blockDim.x) bits[w] = a.bits[w];
    if (a.rewire) {
        stage_rows(a, rb, n, f);
        // root children: bitset and exclusive prefix popcounts (trie order = token order)
        if (a.trie.root_bits) {
            int c = 0;
            for (int w = tid; w < nw; w += blockDim.x) {   // nw <= blockDim.x (V <= 32768)
                const uint32_t v = a.trie.root_bits[w];
                f.root[w] = v;
                c = __popc(v);
            }
            // block exclusive scan of one count per thread
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid % 32 >= o) incl += t;
            }
            if (tid % 32 == 31) red_i[tid / 32] = incl;
            __syncthreads();
            if (tid < 32) {
                const int wv = red_i[tid];
                int wi = wv;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, wi, o);
                    if (tid >= o) wi += t;
                }
                red_i[tid] = wi - wv;
            }
            __syncthreads();
            if (tid < nw) f.root[nw + tid] = (uint32_t)(red_i[tid / 32] + incl - c);
            __syncthreads();
        }
    }
    if (!bulk)
        for (int i = tid; i < V; i += blockDim.x) x[i] = xg[i];
    __syncthreads();
    if (bulk && !mbar_wait(bar, 0, nullptr)) set_status(a.status, XGR_DEV_TIMEOUT);
    float lse = 0.f;
    if (a.logits && n > 0) lse = block_lse(x, V, red_f, a.status);
    int c = 0;   // candidates: mask bits below V
    for (int w = tid; w < nw; w += blockDim.x)
        c += __popc(bits[w] & (32 * w + 32 <= V ? ~0u : (1u << (V & 31)) - 1u));
    const int total = n > 0 ? block_sum_int(c, red_i) : 0;
    const int want = min(BW, total);
    DenseCand cand{x, bits, cum, lse, V, a.logits, a.status};
    const int64_t E = n > 0 ? V : 0;
    uint64_t prefix = ~0ull, mask = 0;
    if (V <= 8 * kDenseThreads) {   // every key computed once, held in registers
        uint64_t kr[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = tid + u * kDenseThreads;
            uint64_t key = kNoKey;
            kr[u] = (t < E && cand(t, key)) ? key : kNoKey;
        }
        if (want < total) radix_select_regs(kr, want, whist, sc, red_i, red_k, prefix, mask);
        collect_regs(kr, prefix, mask, BW, [&](int u) { return tid + u * kDenseThreads; }, f);
    } else {
        if (want < total) radix_select(cand, E, want, hist, sc, prefix, mask);
        collect(cand, E, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
    }
    __syncthreads();
    finish_request(a, r, min(*f.cnt, want), f);
}

// ------------------------------------------------------------------ sparse steps

// One persistent CTA per SM takes a contiguous block of beam rows.  It reads
// the metadata of a window of its rows (row pointers, cumulative scores, live
// counts) in one round trip and the window's CSR tokens -- one contiguous range
// -- in another (log-prob mode: then the tokens' scores), all into shared
// memory.  In logits mode the score rows stream through nbuf slots by bulk
// copies issued nbuf rows ahead, so the HBM traffic overlaps the work on
// earlier rows.  Eight groups of four warps work on eight rows at a time.  Per row:
// the log-sum-exp (logits), each entry's key beside its CSR position, the
// row's best key.
constexpr int kRowsThreads = 1024;
constexpr int kRowsGroups = 8;   // rows in work at once (more, smaller groups measured faster)
constexpr int kRowsGroup = kRowsThreads / kRowsGroups;
constexpr int kRowsMaxBuf = 8;
constexpr int kRowsWin = 256;     // rows per metadata window
constexpr int kRowsTok = 8192;    // CSR entries staged per window (a longer row reads the rest in place)

__host__ __device__ inline size_t rows_fixed_bytes(bool logits) {
    return (size_t)kRowsTok * 4 * (logits ? 1 : 2) + (size_t)(kRowsWin + 1) * 4 + (size_t)kRowsWin * 12;
}

__global__ void __launch_bounds__(kRowsThreads, 1) select_rows_kernel(SelectArgs a, int nbuf) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kRowsMaxBuf];
    __shared__ int slot_row[kRowsMaxBuf];   // the row (index in the block) whose copy a slot holds
    constexpr int kGroupWarps = kRowsGroup / 32;
    __shared__ float red_f[2 * kGroupWarps * kRowsGroups];   // per group: (m, s) of each warp
    __shared__ uint64_t red_k[kGroupWarps * kRowsGroups];   // per group: each warp's min
    __shared__ int win_end;
    const Dims dm = a.dims;
    const int V = dm.V, BW = dm.BW, tid = threadIdx.x;
    const int64_t n_rows = (int64_t)dm.B * BW;
    const int64_t per = (n_rows + gridDim.x - 1) / gridDim.x;
    const int64_t r0 = (int64_t)blockIdx.x * per, r1 = min(n_rows, r0 + per);
    const bool stage = a.logits;   // logits: whole rows (their log-sum-exp)
    const bool bulk = stage && (V & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0;
    const size_t xb = stage ? al16((size_t)V * 4) : 0;
    uint8_t *p = smem + nbuf * xb;
    int *tok = reinterpret_cast<int *>(p);
    p += (size_t)kRowsTok * 4;
    float *val = reinterpret_cast<float *>(p);   // log-prob mode only
    if (!stage) p += (size_t)kRowsTok * 4;
    int *rp = reinterpret_cast<int *>(p);        // [kRowsWin + 1]
    p += (size_t)(kRowsWin + 1) * 4;
    float *cum_w = reinterpret_cast<float *>(p);  // [kRowsWin]
    int *nl_w = reinterpret_cast<int *>(cum_w + kRowsWin);   // [kRowsWin] live beams of the row's request
    int *base_w = nl_w + kRowsWin;                           // [kRowsWin] first entry of the row's request
    auto x_of = [&](int64_t row) { return reinterpret_cast<float *>(smem + ((row - r0) % nbuf) * xb); };
    auto issue = [&](int64_t row) {   // one thread: the bulk copy of a row into its slot
        const uint32_t bar = smem_u32(&full[(row - r0) % nbuf]);
        reinterpret_cast<volatile int *>(slot_row)[(row - r0) % nbuf] = (int)(row - r0);
        mbar_expect_tx(bar, (uint32_t)V * 4u);
        bulk_g2s(smem_u32(x_of(row)), a.scores + row * V, (uint32_t)V * 4u, bar);
    };
    // The last thread (it has no window metadata to load while the windows hold
    // far fewer rows than threads) sets up the slots and starts the first rows'
    // bulk copies at once; the other threads meanwhile load the first window.
    constexpr int kIssuer = kRowsThreads - 1;
    static_assert(kRowsWin < kIssuer, "the issuing thread loads no window metadata");
    if (tid == kIssuer && bulk) {
        for (int k = 0; k < nbuf; ++k) {
            mbar_init(smem_u32(&full[k]), 1);
            slot_row[k] = -1;
        }
        fence_mbar_init();
        for (int64_t row = r0; row < min(r1, r0 + nbuf); ++row) issue(row);
    }
    // Every other load of a row's work happens per window, ahead of the rows: a
    // global load issued behind the bulk traffic waits microseconds.
    for (int64_t w0 = r0; w0 < r1;) {
        // ---- window metadata: one round trip
        const int64_t wmax = min(r1, w0 + kRowsWin);
        for (int64_t row = w0 + tid; row <= wmax; row += kRowsThreads) {
            rp[row - w0] = a.row_ptr[row];
            if (row < wmax) {
                cum_w[row - w0] = a.cum[row];
                nl_w[row - w0] = a.n_live[row / BW];
                base_w[row - w0] = a.row_ptr[row / BW * BW];
            }
        }
        __syncthreads();
        // rows whose entries fit the token area (at least one row)
        if (tid == 0) {
            int64_t w1 = w0 + 1;
            while (w1 < wmax && rp[w1 + 1 - w0] - rp[0] <= kRowsTok) ++w1;
            win_end = (int)(w1 - w0);
        }
        __syncthreads();
        const int64_t w1 = w0 + win_end;
        const int t0 = rp[0], nt = min(rp[w1 - w0] - t0, kRowsTok);
        // ---- the window's tokens (one contiguous range), then log-prob scores
        for (int j = tid; j < nt; j += kRowsThreads) {
            const int t = a.cols[t0 + j];
            tok[j] = t;
            if (!stage) {
                // entry j's row: the last window row whose first entry is <= j
                int l = 0, h = (int)(w1 - w0);
                while (h - l > 1) {
                    const int m = (l + h) >> 1;
                    if (rp[m] - t0 <= j) l = m; else h = m;
                }
                const int64_t row = w0 + l;
                val[j] = (t >= 0 && t < V) ? a.scores[row * V + t] : 0.f;
            }
        }
        __syncthreads();
        // ---- the window's rows: group g (256 threads, named barrier 1 + g) takes
        // rows w0 + g, w0 + g + 4, ...; when it is done with a row it starts the
        // copy of the row nbuf places later into the same slot
        const Group grp{1 + tid / kRowsGroup, kRowsGroup, tid % kRowsGroup};
        const int gi = tid / kRowsGroup;
        for (int64_t row = w0 + gi; row < w1; row += kRowsGroups) {
            const int r = (int)(row / BW), b = (int)(row % BW);
            const int i = (int)(row - w0);
            const bool live = b < nl_w[i];
            if (b == 0 && grp.t == 0) {   // the pick kernel counts from 0
                a.surv_cnt[r] = 0;
                a.ticket[r] = 0;
            }
            const float *xg = a.scores + row * V;
            float *x = x_of(row);
            if (stage && !bulk) {   // unaligned rows: plain loads into the slot
                for (int t = grp.t; t < V; t += kRowsGroup) x[t] = xg[t];
                grp.sync();
            }
            if (bulk) {
                // a slot serves rows nbuf apart, taken by different groups: wait until
                // this row's copy is the one in flight, then for its bytes
                const int k = (int)((row - r0) % nbuf);
                bool ok = false;
                for (uint32_t it = 0; it < kSpinLimit && !ok; ++it)
                    ok = reinterpret_cast<volatile int *>(slot_row)[k] == (int)(row - r0);
                if (!ok || !mbar_wait(smem_u32(&full[k]), (int)((row - r0) / nbuf) & 1, nullptr))
                    set_status(a.status, XGR_DEV_TIMEOUT);
            }
            float lse = 0.f;
            if (stage && live) lse = group_lse(x, V, red_f + 2 * kGroupWarps * gi, a.status, grp);
            const int beg = rp[i], end = rp[i + 1], n_e = max(0, end - beg);
            uint64_t *keys = a.keys + (int64_t)r * a.key_cap;
            const int base = base_w[i];
            const float cum = cum_w[i];
            uint64_t best = kNoKey;
            for (int j = grp.t; j < n_e; j += kRowsGroup) {
                const int e = beg + j, ew = e - t0;   // entry, its place in the window's tokens
                const bool staged = ew >= 0 && ew < nt;
                uint64_t key = kNoKey;
                if (live) {
                    const int t = staged ? tok[ew] : a.cols[e];
                    if (t < 0 || t >= V) {
                        set_status(a.status, XGR_DEV_MASK);
                    } else {
                        float lp = stage ? x[t] : (staged ? val[ew] : xg[t]);
                        if (a.logits) lp -= lse;
                        uint64_t k2;
                        if (make_key(cum, lp, b, t, V, a.status, k2)) key = k2;
                    }
                }
                if (e >= base && (int64_t)(e - base) < a.key_cap) keys[e - base] = key;
                best = key < best ? key : best;
            }
            best = group_min_u64(best, red_k + kGroupWarps * gi, grp);   // (its barriers end every read of the slot)
            if (grp.t == 0) {
                a.best[row] = best;
                a.row_lse[row] = lse;
                if (bulk && row + nbuf < r1) issue(row + nbuf);
            }
        }
        w0 = w1;
        __syncthreads();   // the window's shared metadata is reused
    }
}

size_t pick_smem(const Dims &dm) {
    return (size_t)kSmemSurv * 12 + finish_bytes(dm.BW, dm.BW, dm.S, 0) + al16((size_t)dm.BW * 8);
}

__global__ void __launch_bounds__(kPickThreads, 1) select_pick_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t red_k[32];
    __shared__ int hist[256];
    __shared__ int sc[4];
    __shared__ int last;
    __shared__ int scan_w[32];
    __shared__ int red_i[32];
    __shared__ int whist[kWideBins];
    __shared__ int slice_base;
    const Dims dm = a.dims;
    const int BW = dm.BW, P = a.pick_parts;
    const int r = blockIdx.x / P, part = blockIdx.x % P;
    const int tid = threadIdx.x;
    const int64_t rb = (int64_t)r * BW;
    const int n = a.n_live[r];
    const int base = a.row_ptr[rb];
    const int64_t E = (int64_t)a.row_ptr[rb + BW] - base;   // dead rows' entries hold kNoKey
    // tau: the worst of the live beams' best keys, when all BW beams are live
    uint64_t worst = 0;
    for (int b = tid; b < BW; b += kPickThreads) {
        const uint64_t k = a.best[rb + b];
        if (b < n) worst = k > worst ? k : worst;
    }
    worst = block_max_u64(worst, red_k);
    const uint64_t tau = n == BW ? worst : kNoKey;
    const bool fits = E <= a.key_cap;
    const uint64_t *keys = a.keys + (int64_t)r * a.key_cap;
    uint64_t *sk_g = a.surv_key + (int64_t)r * a.surv_cap;
    int32_t *se_g = a.surv_e + (int64_t)r * a.surv_cap;
    if (fits) {
        // survivors of each slice: a block scan of the per-thread counts, one
        // atomic per slice for the slice's place in the request's buffer
        constexpr int U = kPickKeys / kPickThreads;
        for (int64_t s0 = (int64_t)part * kPickKeys; s0 < E; s0 += (int64_t)P * kPickKeys) {
            uint64_t k[U];
            int c = 0;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t e = s0 + tid + u * kPickThreads;
                k[u] = e < E ? __ldcg(keys + e) : kNoKey;
                c += k[u] != kNoKey && k[u] <= tau;
            }
            int n_slice;
            int pos = block_exclusive_scan_int(c, scan_w, &n_slice);
            if (tid == 0) slice_base = n_slice ? atomicAdd(&a.surv_cnt[r], n_slice) : 0;
            __syncthreads();
            pos += slice_base;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (k[u] == kNoKey || k[u] > tau) continue;
                if (pos < a.surv_cap) {
                    sk_g[pos] = k[u];
                    se_g[pos] = (int32_t)(s0 + tid + u * kPickThreads);
                }
                ++pos;
            }
            __syncthreads();   // slice_base is reused
        }
    }
    // the last CTA of the request to finish its slices takes the selection
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(&a.ticket[r], 1u) == (unsigned)(P - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();

    uint64_t *sk = reinterpret_cast<uint64_t *>(smem);
    int *se = reinterpret_cast<int *>(smem + (size_t)kSmemSurv * 8);
    uint8_t *fin = smem + (size_t)kSmemSurv * 12;
    const FinishSmem f = carve_finish(fin, BW, BW, dm.S, 0);
    float *cum_s = reinterpret_cast<float *>(fin + finish_bytes(BW, BW, dm.S, 0));
    float *lse_s = cum_s + BW;
    const int T = __ldcg(&a.surv_cnt[r]);
    if (tid == 0) *f.cnt = 0;
    for (int b = tid; b <= n; b += kPickThreads) f.rp[b] = a.row_ptr[rb + b] - base;
    if (a.rewire) stage_rows(a, rb, n, f);
    if (!fits)
        for (int b = tid; b < n; b += kPickThreads) {
            cum_s[b] = a.cum[rb + b];
            lse_s[b] = a.logits ? a.row_lse[rb + b] : 0.f;
        }
    __syncthreads();
    // the survivors and the parents' child ranges load together
    const bool in_smem = fits && T <= kSmemSurv;
    if (in_smem) {
        for (int i = tid; i < T; i += kPickThreads) {
            sk[i] = __ldcg(sk_g + i);
            se[i] = __ldcg(se_g + i);
        }
    }
    if (a.rewire) stage_children(a, n, f);
    __syncthreads();
    uint64_t prefix = ~0ull, mask = 0;
    int want;
    if (fits) {
        // every winner survived tau; T >= BW whenever tau cuts anything
        want = min(BW, T);
        if (in_smem) {   // the survivors' keys in registers, 8 per thread
            static_assert(kSmemSurv == 8 * kPickThreads, "survivors per thread");
            uint64_t kr[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = tid + u * kPickThreads;
                kr[u] = i < T ? sk[i] : kNoKey;
            }
            if (want < T) radix_select_regs(kr, want, whist, sc, red_i, red_k, prefix, mask);
            collect_regs(kr, prefix, mask, BW, [&](int u) { return se[tid + u * kPickThreads]; }, f);
        } else if (T <= a.surv_cap) {
            const ListCand<true> cand{sk_g};
            if (want < T) radix_select(cand, T, want, hist, sc, prefix, mask);
            collect(cand, T, prefix, mask, BW, [&](int64_t i) { return __ldcg(se_g + i); }, f);
        } else {
            const KeyCand cand{keys, tau};
            if (want < T) radix_select(cand, E, want, hist, sc, prefix, mask);
            collect(cand, E, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
        }
    } else {
        // the key buffer overflowed: exact selection over every candidate
        ReqCand cand;
        cand.x = a.scores + rb * dm.V;
        cand.cols = a.cols + base;
        cand.rp = f.rp;
        cand.cum = cum_s;
        cand.lse = lse_s;
        cand.status = a.status;
        cand.n = n;
        cand.logits = a.logits;
        cand.V = dm.V;
        const int total = f.rp[n];
        want = min(BW, total);
        if (want < total) radix_select(cand, total, want, hist, sc, prefix, mask);
        collect(cand, total, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
    }
    __syncthreads();
    finish_request(a, r, min(*f.cnt, want), f);
}

// ---- requests of few CSR entries: one CTA each, every key in registers

constexpr int kPickOneThreads = 1024;
constexpr int kPickOneKpt = 16;          // keys per thread in registers
constexpr int kPickOneTail = 16384;      // further keys in shared memory
constexpr int kPickOneMax = kPickOneKpt * kPickOneThreads + kPickOneTail;

size_t pick_one_smem(const Dims &dm) {
    return (size_t)kPickOneTail * 8 + finish_bytes(dm.BW, dm.BW, dm.S, 0) + al16((size_t)dm.BW * 8);
}

// One CTA per request: the request's keys go straight into registers and a
// shared-memory tail (no threshold pass, no survivor buffer), then the exact
// radix select, ordering, outputs and rewiring.  Requests with more entries
// select from the key buffer in global memory (or, past the buffer, from the
// scores), exactly as the multi-CTA pick does.
__global__ void __launch_bounds__(kPickOneThreads, 1) select_pick_one_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int hist[256];
    __shared__ int sc[4];
    __shared__ int red_i[32];
    __shared__ uint64_t red_k[32];
    __shared__ int whist[kWideBins];
    const Dims dm = a.dims;
    const int BW = dm.BW, r = blockIdx.x, tid = threadIdx.x;
    const int64_t rb = (int64_t)r * BW;
    uint64_t *tail = reinterpret_cast<uint64_t *>(smem);
    uint8_t *fin = smem + (size_t)kPickOneTail * 8;
    const FinishSmem f = carve_finish(fin, BW, BW, dm.S, 0);
    float *cum_s = reinterpret_cast<float *>(fin + finish_bytes(BW, BW, dm.S, 0));
    float *lse_s = cum_s + BW;
    const uint64_t *keys = a.keys + (int64_t)r * a.key_cap;
    constexpr int kReg = kPickOneKpt * kPickOneThreads;
    // every load below is independent of the others: one round trip
    const int n = a.n_live[r];
    const int base = a.row_ptr[rb];
    const int64_t E = (int64_t)a.row_ptr[rb + BW] - base;   // dead rows' entries hold kNoKey
    uint64_t kr[kPickOneKpt];
#pragma unroll
    for (int u = 0; u < kPickOneKpt; ++u) {
        const int64_t e = tid + u * kPickOneThreads;
        kr[u] = e < a.key_cap ? __ldcg(keys + e) : kNoKey;
    }
    if (tid == 0) *f.cnt = 0;
    for (int b = tid; b <= BW; b += kPickOneThreads) f.rp[b] = a.row_ptr[rb + b] - base;
    if (a.rewire) stage_rows(a, rb, BW, f);
    const bool in_smem = E <= a.key_cap && E <= kPickOneMax;
    const int n_tail = in_smem && E > kReg ? (int)(E - kReg) : 0;
    for (int i = tid; i < n_tail; i += kPickOneThreads) tail[i] = __ldcg(keys + kReg + i);
    if (E > a.key_cap)
        for (int b = tid; b < n; b += kPickOneThreads) {
            cum_s[b] = a.cum[rb + b];
            lse_s[b] = a.logits ? a.row_lse[rb + b] : 0.f;
        }
    __syncthreads();
    if (a.rewire) stage_children(a, n, f);
    uint64_t prefix = ~0ull, mask = 0;
    int want;
    if (in_smem) {
        int c = 0;
#pragma unroll
        for (int u = 0; u < kPickOneKpt; ++u) {
            if (tid + u * kPickOneThreads >= E) kr[u] = kNoKey;
            c += kr[u] != kNoKey;
        }
        for (int i = tid; i < n_tail; i += kPickOneThreads) c += tail[i] != kNoKey;
        const int T = block_sum_int(c, red_i);   // (its barriers also publish the staging)
        want = min(BW, T);
        if (want < T) radix_select_regs(kr, want, whist, sc, red_i, red_k, prefix, mask, tail, n_tail);
        collect_regs(kr, prefix, mask, BW, [&](int u) { return tid + u * kPickOneThreads; }, f);
        for (int i = tid; i < n_tail; i += kPickOneThreads) {
            const uint64_t key = tail[i];
            if (key != kNoKey && (key & mask) <= prefix) {
                const int pos = atomicAdd(f.cnt, 1);
                if (pos < BW) {
                    f.win_k[pos] = key;
                    f.win_e[pos] = kReg + i;
                }
            }
        }
    } else if (E <= a.key_cap) {
        __syncthreads();
        const KeyCand cand{keys, kNoKey};
        int c = 0;
        for (int64_t e = tid; e < E; e += kPickOneThreads) c += __ldcg(keys + e) != kNoKey;
        const int T = block_sum_int(c, red_i);
        want = min(BW, T);
        if (want < T) radix_select(cand, E, want, hist, sc, prefix, mask);
        collect(cand, E, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
    } else {
        __syncthreads();
        ReqCand cand;
        cand.x = a.scores + rb * dm.V;
        cand.cols = a.cols + base;
        cand.rp = f.rp;
        cand.cum = cum_s;
        cand.lse = lse_s;
        cand.status = a.status;
        cand.n = n;
        cand.logits = a.logits;
        cand.V = dm.V;
        const int total = f.rp[n];
        want = min(BW, total);
        if (want < total) radix_select(cand, total, want, hist, sc, prefix, mask);
        collect(cand, total, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
    }
    __syncthreads();
    finish_request(a, r, min(*f.cnt, want), f);
}

// opt in to the dynamic shared memory a launch needs: without it static plus
// dynamic shared memory may not pass 48 KB
template <class K>
cudaError_t ensure_smem(K kernel, size_t bytes) {
    if (bytes == 0) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

// ------------------------------------------------------------------ host side

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t select_scratch_bytes(int B, int BW, int64_t key_cap, int64_t surv_cap) {
    const size_t rows = (size_t)B * BW;
    return al256(rows * 4) + al256(rows * 8) + al256((size_t)B * 4) + al256((size_t)B * 4) +
           al256((size_t)B * key_cap * 8) + al256((size_t)B * surv_cap * 8) +
           al256((size_t)B * surv_cap * 4);
}

void select_scratch_carve(uint8_t *base, int B, int BW, int64_t key_cap, int64_t surv_cap,
                          SelectArgs &a) {
    const size_t rows = (size_t)B * BW;
    a.row_lse = reinterpret_cast<float *>(base);
    base += al256(rows * 4);
    a.best = reinterpret_cast<uint64_t *>(base);
    base += al256(rows * 8);
    a.surv_cnt = reinterpret_cast<int32_t *>(base);
    base += al256((size_t)B * 4);
    a.ticket = reinterpret_cast<uint32_t *>(base);
    base += al256((size_t)B * 4);
    a.keys = reinterpret_cast<uint64_t *>(base);
    base += al256((size_t)B * key_cap * 8);
    a.surv_key = reinterpret_cast<uint64_t *>(base);
    base += al256((size_t)B * surv_cap * 8);
    a.surv_e = reinterpret_cast<int32_t *>(base);
    a.key_cap = key_cap;
    a.surv_cap = surv_cap;
}

static cudaError_t launch_beam_select_impl(const SelectArgs &a_in, cudaStream_t s);

cudaError_t launch_beam_select(const SelectArgs &a, cudaStream_t s) {
    const cudaError_t e = launch_beam_select_impl(a, s);
    if (e != cudaSuccess)
        debug_log("beam select (B=%d BW=%d V=%d dense=%d): launch failed: %s", a.dims.B, a.dims.BW,
                  a.dims.V, a.dense, cudaGetErrorString(e));
    return e;
}

static cudaError_t launch_beam_select_impl(const SelectArgs &a_in, cudaStream_t s) {
    SelectArgs a = a_in;
    const Dims &dm = a.dims;
    if (dm.BW > 1024 || dm.V > kSelectMaxVocab || dm.V < 1) return cudaErrorInvalidValue;
    if (a.dense) {
        const size_t smem = dense_smem(dm);
        cudaError_t e = ensure_smem(select_dense_kernel, smem);
        if (e != cudaSuccess) return e;
        select_dense_kernel<<<dm.B, kDenseThreads, smem, s>>>(a);
        return cudaGetLastError();
    }
    {
        // one persistent CTA per SM, as many row slots as shared memory holds
        const size_t xb = a.logits ? dense_x_bytes(dm.V) : 0, fixed = rows_fixed_bytes(a.logits);
        const int nbuf = a.logits ? (int)std::min<size_t>(kRowsMaxBuf, ((210u << 10) - fixed) / xb) : 1;
        if (nbuf < 1) return cudaErrorInvalidValue;
        const size_t smem = nbuf * xb + fixed;
        cudaError_t e = ensure_smem(select_rows_kernel, smem);
        if (e != cudaSuccess) return e;
        const int64_t rows = (int64_t)dm.B * dm.BW;
        const int grid = (int)std::min<int64_t>(rows, a.num_sms > 0 ? a.num_sms : 148);
        select_rows_kernel<<<grid, kRowsThreads, smem, s>>>(a, nbuf);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // the one-CTA pick when the pool fits its registers and its shared memory fits the SM
    if (std::min<int64_t>(a.max_entries, a.key_cap) <= kPickOneMax && pick_one_smem(dm) <= (200u << 10)) {
        const size_t smem = pick_one_smem(dm);
        cudaError_t e = ensure_smem(select_pick_one_kernel, smem);
        if (e != cudaSuccess) return e;
        select_pick_one_kernel<<<dm.B, kPickOneThreads, smem, s>>>(a);
        return cudaGetLastError();
    }
    int64_t parts = (std::min<int64_t>(a.max_entries, a.key_cap) + kPickKeys - 1) / kPickKeys;
    a.pick_parts = (int)std::max<int64_t>(1, std::min<int64_t>(parts, kMaxPickParts));
    const size_t smem = pick_smem(dm);
    cudaError_t e = ensure_smem(select_pick_kernel, smem);
    if (e != cudaSuccess) return e;
    select_pick_kernel<<<dm.B * a.pick_parts, kPickThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace xgr

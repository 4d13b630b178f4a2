// select.cu -- masked beam Top-K with a global threshold (early termination)
// and the in-place rewiring of the beam state.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"):
//  2.2 "Valid-path constraint" / "Hybrid dense/sparse storage": candidates
//      come only from the valid-item vocabulary -- a dense bitset of first
//      tokens at step 0, sparse rows (each beam's sorted trie children) later.
//      "Early sort termination": the page orders each beam's candidates and
//      cuts every list at a global min-heap threshold.  Here each beam's list
//      is ordered as far as its head (its m best keys), the threshold tau is
//      the BW-th best of all heads (BW real candidates rank at or above it, so
//      every winner does), and only the candidates at or above it
//      ("survivors") reach the exact selection.
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
//    log-sum-exp (logits); tau = the BW-th best of the threads' best keys, and
//    the survivors at or above it are ranked by counting.
//  * sparse (CSR) masks: select_sparse_kernel, one launch per step.  Each
//    request gets several CTAs; a warp takes one beam row at a time: its
//    log-sum-exp (logits), the key of each of its CSR entries, and its head --
//    the beam's m best keys in order (the page's ordered per-beam candidate
//    list, cut at m).  The request's last CTA to finish (an atomic ticket)
//    takes tau = the BW-th best head key (at least BW real candidates rank at
//    or above it, so every winner does), gathers the survivors at or above tau
//    -- the head keys, and the further keys of beams whose whole head
//    survived -- and radix-selects the BW best of them.  It ends in
//    finish_request: the ordering, the outputs and the rewiring.
#include <algorithm>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {


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

// (m, s) <- the pair that stands for both (m, s) and (m2, s2), where each pair
// is a maximum m and a sum s of exp(x - m) over some values (natural units)
__device__ __forceinline__ void lse_pair_merge(float &m, float &s, float m2, float s2) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;   // both empty
    s = (m == -INFINITY ? 0.f : s * ex2f((m - M) * kLog2e)) +
        (m2 == -INFINITY ? 0.f : s2 * ex2f((m2 - M) * kLog2e));
    m = M;
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

// the request's key buffer, restricted to the survivors of tau; with a row
// stride (node masks) only the first rl[b] slots of row b hold keys
struct KeyCand {
    const uint64_t *k;
    uint64_t tau;
    const int *rp, *rl;   // shared memory
    int stride, n;        // stride 0: CSR numbering (every entry written)
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        if (stride) {
            const int b = (int)(e / stride), j = (int)(e % stride);
            if (b >= n || j >= rl[b]) return false;
        }
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
    int *rp;           // [BW+1] sparse: first entry of each beam's row (relative to the request)
    int *st_node;      // [n_stage] staged old rows (rewiring)
    int *st_anc;       // [n_stage*S]
    int *st_seq;       // [n_stage*S]
    int *cb, *ce;      // [n_stage] sparse: child range of each staged row's trie node
    int *rl;           // [n_stage] sparse: mask entries of each row
    uint32_t *root;    // dense: [nw] root-children bitset, [nw] prefix popcounts
    int *cnt;          // winners appended
};

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~(size_t)15; }

// n_stage: old rows staged for the rewiring (the live beams: BW, or 1 for a dense step)
__host__ __device__ inline size_t finish_bytes(int BW, int n_stage, int S, int nw_root) {
    return al16((size_t)BW * 8) + 2 * al16((size_t)BW * 4) + al16((size_t)(BW + 1) * 4) +
           4 * al16((size_t)n_stage * 4) + 2 * al16((size_t)n_stage * S * 4) + al16((size_t)nw_root * 8) +
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
    f.rl = reinterpret_cast<int *>(p);
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

// Rank the n_win winners (unique keys; a winner's rank is its number of better
// winners, counted by one warp per winner), write the outputs in rank order
// and, when a.rewire, rewrite the request's beam state in place.  The caller
// has staged the old rows (stage_rows) and rp / root.
__device__ void finish_request(const SelectArgs &a, int r, int n_win, const FinishSmem &f,
                               bool in_rank_order = false) {
    const Dims dm = a.dims;
    const int BW = dm.BW, S = dm.S, V = dm.V;
    const int64_t rb = (int64_t)r * BW;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nwarps = blockDim.x / 32;
    const int s = a.step;
    // sparse rewiring: each winner's trie child and the check of its token load
    // while the winners are ranked (winners i = threadIdx.x + u * blockDim.x)
    constexpr int kWinPerThread = 4;   // BW <= 1024 <= 4 * blockDim.x (blockDim.x >= 256)
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
    if (in_rank_order) {   // the winners already sit at their ranks
        for (int i = threadIdx.x; i < n_win; i += blockDim.x) f.rank[i] = i;
    } else {
        for (int i = warp; i < n_win; i += nwarps) {
            const uint64_t k = f.win_k[i];
            int c = 0;
            for (int j = lane; j < n_win; j += 32) c += f.win_k[j] < k;
            c = warp_sum_int(c);
            if (lane == 0) f.rank[i] = c;
        }
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

// ------------------------------------------------------------------ sparse steps

// One launch per sparse step.  Request r gets sp_parts CTAs of kSpThreads
// threads; CTA `part` takes beams [part*R, part*R + R) (R = sp_rows), one warp
// per beam at a time, so no reduction spans more than one warp.  Per beam:
//  * logits mode: the row's log-sum-exp over the full vocabulary, streamed
//    from HBM in 16-byte loads with the next batch in flight while the current
//    one is folded (online max / sum of exponentials per lane, then across
//    the warp);
//  * the key of every CSR entry (its score read back, an L2 hit in logits
//    mode), written to the request's key buffer;
//  * the beam's head: its m best keys with their entries, ascending (the
//    page's per-beam ordered candidate list, cut at m).
// Then each CTA takes a ticket; the last of the request's CTAs to arrive
// selects for the whole request (select_request), so no second launch and no
// grid-wide wait is needed.
constexpr int kSpThreads = 256;
constexpr int kSpWarps = kSpThreads / 32;
constexpr int kSpKpc = 8;   // CSR entries per lane in one pass of the key loop
constexpr int kLseU = 16;   // float4 per lane in one batch of the row stream (8 KB per warp)

__device__ __forceinline__ float4 ld_stream4(const float4 *p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// natural-log log-sum-exp of x[0..V), by one warp (every lane gets it); a NaN
// anywhere in the row sets XGR_DEV_NAN
__device__ float warp_row_lse(const float *x, int V, int32_t *status) {
    const int lane = threadIdx.x & 31;
    float m = -INFINITY, s = 0.f;
    bool nan = false;
    auto fold = [&](const float *v, int k) {
        float mv = -INFINITY;
        for (int e = 0; e < k; ++e) {
            nan |= v[e] != v[e];
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
    if ((V & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0) {
        const float4 *x4 = reinterpret_cast<const float4 *>(x);
        const int n4 = V >> 2;
        constexpr int kStep = 32 * kLseU;
        const float4 ninf = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        float4 cur[kLseU];
#pragma unroll
        for (int u = 0; u < kLseU; ++u) {
            const int i = u * 32 + lane;
            cur[u] = i < n4 ? ld_stream4(x4 + i) : ninf;
        }
        for (int b0 = 0; b0 < n4; b0 += kStep) {
            float4 nxt[kLseU];
#pragma unroll
            for (int u = 0; u < kLseU; ++u) {   // the next batch is in flight while this one folds
                const int i = b0 + kStep + u * 32 + lane;
                nxt[u] = i < n4 ? ld_stream4(x4 + i) : ninf;
            }
            float v[4 * kLseU];
#pragma unroll
            for (int u = 0; u < kLseU; ++u) {
                v[4 * u] = cur[u].x;
                v[4 * u + 1] = cur[u].y;
                v[4 * u + 2] = cur[u].z;
                v[4 * u + 3] = cur[u].w;
            }
            fold(v, 4 * kLseU);
#pragma unroll
            for (int u = 0; u < kLseU; ++u) cur[u] = nxt[u];
        }
    } else {
        for (int i = lane; i < V; i += 32) fold(x + i, 1);
    }
    if (__any_sync(0xffffffffu, nan)) {
        if (lane == 0) set_status(status, XGR_DEV_NAN);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_pair_merge(m, s, m2, s2);
    }
    return m + logf(s);
}

// Merges the keys c[] of every lane (entries ce[]) into the warp's running
// head: afterwards lanes 0..m-1 hold the m smallest keys seen so far, in
// ascending order (kNoKey pads), with their entries.  Keys are unique.  m
// rounds of a warp minimum; c[] is consumed.
template <int KPC>
__device__ __forceinline__ void warp_head_merge(uint64_t (&c)[KPC], const int (&ce)[KPC], uint64_t &run,
                                                int &run_e, int m) {
    const int lane = threadIdx.x & 31;
    uint64_t nrun = kNoKey;
    int nrun_e = -1;
    for (int i = 0; i < m; ++i) {
        uint64_t lm = run;
        int le = run_e, slot = KPC;
#pragma unroll
        for (int u = 0; u < KPC; ++u)
            if (c[u] < lm) {
                lm = c[u];
                le = ce[u];
                slot = u;
            }
        const uint64_t wm = warp_min_u64(lm);
        if (wm == kNoKey) break;   // (uniform across the warp)
        const int owner = __ffs(__ballot_sync(0xffffffffu, lm == wm)) - 1;   // keys are unique
        const int we = __shfl_sync(0xffffffffu, le, owner);
        if (lane == owner) {
            if (slot == KPC) run = kNoKey;
#pragma unroll
            for (int u = 0; u < KPC; ++u)
                if (u == slot) c[u] = kNoKey;
        }
        if (lane == i) {
            nrun = wm;
            nrun_e = we;
        }
    }
    run = nrun;
    run_e = nrun_e;
}

// the same over a row staged in shared memory (16-byte aligned, V % 4 == 0)
__device__ float warp_row_lse_smem(const float *x, int V, int32_t *status) {
    const int lane = threadIdx.x & 31;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    const int n4 = V >> 2;
    float m = -INFINITY, s = 0.f;
    bool nan = false;
    for (int b0 = 0; b0 < n4; b0 += 32 * 4) {   // 16 values per lane per pass
        float v[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = b0 + u * 32 + lane;
            const float4 q = i < n4 ? x4[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            v[4 * u] = q.x;
            v[4 * u + 1] = q.y;
            v[4 * u + 2] = q.z;
            v[4 * u + 3] = q.w;
        }
        float mv = -INFINITY;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            nan |= v[e] != v[e];
            mv = fmaxf(mv, v[e]);
        }
        if (mv > m) {
            s = m == -INFINITY ? 0.f : s * ex2f((m - mv) * kLog2e);
            m = mv;
        }
        if (m != -INFINITY) {
            const float mk = m * kLog2e;
#pragma unroll
            for (int e = 0; e < 16; ++e) s += ex2f(fmaf(v[e], kLog2e, -mk));
        }
    }
    if (__any_sync(0xffffffffu, nan)) {
        if (lane == 0) set_status(status, XGR_DEV_NAN);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_pair_merge(m, s, m2, s2);
    }
    return m + logf(s);
}

// The valid tokens of a NODE_BITS row, compacted into wtok[0..) in token
// order (the node's children in trie order) by one warp; returns their count.
__device__ int warp_bits_to_tokens(const uint32_t *wb, int nw, int *wtok, int cap) {
    const int lane = threadIdx.x & 31;
    int cnt = 0;
    for (int w0 = 0; w0 < nw; w0 += 32 * 8) {
        uint32_t wv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {   // up to 256 words in flight per pass
            const int w = w0 + u * 32 + lane;
            wv[u] = w < nw ? __ldg(wb + w) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = __popc(wv[u]);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            int pos = cnt + incl - c;
            uint32_t v = wv[u];
            const int tbase = 32 * (w0 + u * 32 + lane);
            while (v) {
                const int bit = __ffs(v) - 1;
                v &= v - 1;
                if (pos < cap) wtok[pos] = tbase + bit;
                ++pos;
            }
            cnt += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncwarp();
    return cnt;
}

// Phase 1 of one beam row, by one warp: keys of its mask entries into the key
// buffer, its head (m best keys and entries, lanes 0..m-1), its count of valid
// candidates, its entry count and the first trie child of its node.  The
// row's tokens come from the CSR rows, from its node's children in the trie
// level (TRIE_ROWS), or from its node's pre-generated bitset (NODE_BITS,
// compacted into wtok).
__device__ void sparse_row(const SelectArgs &a, int r, int b, int n_live, int base, uint64_t *keys,
                           int *wtok, const float *xs) {
    const int lane = threadIdx.x & 31;
    const Dims dm = a.dims;
    const int V = dm.V, m = a.head_m, s = a.step;
    const int64_t row = (int64_t)r * dm.BW + b;
    const bool live = b < n_live;
    const float cum = a.cum[row];
    const float *x = a.scores + row * V;
    // the first loads of the row's tokens go out before the row stream; the
    // rest (its tokens, the node's first child) follow its log-sum-exp
    const bool csr = a.mask_kind == XGR_MASK_CSR;
    const int beg = csr ? a.row_ptr[row] : 0, end = csr ? a.row_ptr[row + 1] : 0;
    const int node = (csr ? (a.rewire && live) : live) ? (csr ? a.st.node[row] : a.row_node[row]) : -1;
    float lse = 0.f;
    if (a.logits && live) lse = xs ? warp_row_lse_smem(xs, V, a.status) : warp_row_lse(x, V, a.status);
    // the row's tokens (tokp[0..n_e)), their entry base and the node's first child
    const int32_t *tokp = nullptr;
    int n_e = 0, cb = -1;
    int64_t ebase;
    if (csr) {
        tokp = a.cols + beg;
        n_e = max(0, end - beg);
        ebase = beg - base;
        if (s < a.trie.levels && node >= 0 && node < a.trie.n_nodes[s]) cb = a.trie.ptr[s][node];
    } else {
        ebase = (int64_t)b * a.row_stride;
        if (node >= 0 && node < a.n_nodes) {
            const int lo = a.node_ptr[node], hi = a.node_ptr[node + 1];
            cb = lo;
            n_e = min(max(0, hi - lo), a.row_stride);
            if (a.mask_kind == XGR_MASK_TRIE_ROWS) {
                tokp = a.node_tok + lo;
            } else {
                const int nb = warp_bits_to_tokens(a.node_bits + (int64_t)node * a.n_words, a.n_words, wtok,
                                                   a.row_stride);
                if (nb != hi - lo && lane == 0) set_status(a.status, XGR_DEV_MASK);   // table and trie disagree
                n_e = min(nb, a.row_stride);
                tokp = wtok;
            }
        } else if (live && lane == 0) {
            set_status(a.status, XGR_DEV_INDEX);
        }
    }
    uint64_t run = kNoKey;   // lane i < m: the i-th best key of the row so far
    int run_e = -1;
    int n_valid = 0;
    for (int j0 = 0; j0 < n_e; j0 += 32 * kSpKpc) {
        uint64_t c[kSpKpc];
        int ce[kSpKpc];
        int tk[kSpKpc];
#pragma unroll
        for (int u = 0; u < kSpKpc; ++u) {   // the entries' tokens (one round trip) ...
            const int j = j0 + u * 32 + lane;
            tk[u] = (j < n_e && live) ? tokp[j] : -1;
        }
        float sv[kSpKpc];
#pragma unroll
        for (int u = 0; u < kSpKpc; ++u)     // ... then their scores (staged, or another)
            sv[u] = (tk[u] >= 0 && tk[u] < V) ? (xs ? xs[tk[u]] : __ldg(x + tk[u])) : 0.f;
#pragma unroll
        for (int u = 0; u < kSpKpc; ++u) {
            const int j = j0 + u * 32 + lane;
            c[u] = kNoKey;
            ce[u] = -1;
            if (j >= n_e) continue;
            const int64_t e = ebase + j;   // the entry, relative to the request
            uint64_t key = kNoKey;
            if (live) {
                if (tk[u] < 0 || tk[u] >= V) {
                    set_status(a.status, XGR_DEV_MASK);
                } else {
                    const float lp = a.logits ? sv[u] - lse : sv[u];
                    uint64_t k2;
                    if (make_key(cum, lp, b, tk[u], V, a.status, k2)) key = k2;
                }
            }
            if (e >= 0 && e < a.key_cap) keys[e] = key;
            c[u] = key;
            ce[u] = (int)e;
            n_valid += key != kNoKey;
        }
        warp_head_merge(c, ce, run, run_e, m);
    }
    n_valid = warp_sum_int(n_valid);
    if (lane < m) {
        a.head_k[row * m + lane] = run;
        a.head_e[row * m + lane] = run_e;
    }
    if (lane == 0) {
        a.row_cnt[row] = n_valid;
        a.row_lse[row] = lse;
        a.row_len[row] = n_e;
        a.row_cb[row] = cb;
    }
}

// exact radix select over the keys k[0..n) in shared memory (unique keys;
// kNoKey entries are not candidates), by the whole block (blockDim a multiple
// of 256, at most 2048), with 11-bit digits starting at the highest bit where
// the smallest and largest key differ (so the first digit already spreads the
// keys).  On return exactly `want` keys satisfy (key & mask) <= prefix
// (0 < want <= number of candidates).  hist: kRadixBins ints; scan_w: 32 ints;
// red: 32 u64; sc: 3 ints of shared memory.
constexpr int kRadixBits = 11, kRadixBins = 1 << kRadixBits;
__device__ void smem_radix_select(const uint64_t *k, int n, int want, int *hist, int *scan_w,
                                  uint64_t *red, int *sc, uint64_t &prefix, uint64_t &mask) {
    const int tid = threadIdx.x, nt = blockDim.x;
    uint64_t lo = kNoKey, hi = 0;
    for (int i = tid; i < n; i += nt) {
        const uint64_t key = k[i];
        if (key == kNoKey) continue;
        lo = key < lo ? key : lo;
        hi = key > hi ? key : hi;
    }
    lo = block_min_u64(lo, red);
    hi = block_max_u64(hi, red);
    const uint64_t diff = lo ^ hi;
    if (diff == 0) {
        prefix = lo;
        mask = ~0ull;
        return;
    }
    int pos = 64 - __clzll((long long)diff);
    mask = pos == 64 ? 0ull : ~((1ull << pos) - 1ull);
    prefix = lo & mask;
    int k_rem = want;
    const int bpt = kRadixBins / nt;   // bins per thread in the bucket search (8, 4 or 2)
    while (pos > 0) {
        const int shift = pos > kRadixBits ? pos - kRadixBits : 0, width = pos - shift;
        const uint64_t dmask = (1ull << width) - 1ull;
        for (int i = tid; i < kRadixBins; i += nt) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += nt) {
            const uint64_t key = k[i];
            if (key != kNoKey && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
        }
        __syncthreads();
        int h[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            h[j] = j < bpt ? hist[tid * bpt + j] : 0;
            sum += h[j];
        }
        int total;
        int acc = block_exclusive_scan_int(sum, scan_w, &total);
        if (acc < k_rem && acc + sum >= k_rem) {
            bool found = false;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (found || j >= bpt) continue;
                if (acc + h[j] >= k_rem) {
                    sc[0] = tid * bpt + j;
                    sc[1] = h[j] - (k_rem - acc);   // 0 <=> the whole bin is taken
                    sc[2] = k_rem - acc;
                    found = true;
                } else {
                    acc += h[j];
                }
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

// The largest key of k[0..n) that the radix select kept ((key & mask) <= prefix).
__device__ uint64_t selected_max(const uint64_t *k, int n, uint64_t prefix, uint64_t mask, uint64_t *red) {
    uint64_t t = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        if (k[i] != kNoKey && (k[i] & mask) <= prefix) t = k[i] > t ? k[i] : t;
    return block_max_u64(t, red);
}

// The `want` best of the survivors sk[0..ns) (unique keys, ns >= want), placed
// in rank order: a survivor's rank is its number of better survivors (every
// thread counts for its own survivors over the whole list -- broadcast reads,
// no barrier in between), so the winners land at f.win_k[rank] directly.
constexpr int kRankDirect = 512;   // most survivors ranked by counting
__device__ void place_by_rank(const uint64_t *sk, const int *se, int ns, int want, const FinishSmem &f) {
    for (int i = threadIdx.x; i < ns; i += blockDim.x) {
        const uint64_t x = sk[i];
        int c = 0;
        for (int j = 0; j < ns; ++j) c += sk[j] < x;
        if (c < want) {
            f.win_k[c] = x;
            f.win_e[c] = se[i];
        }
    }
}

__host__ __device__ inline int sparse_cand_cap(int BW, int m) { return BW * m; }
__host__ __device__ inline int sparse_surv_cap(int BW) { return BW >= 1024 ? 4096 : (BW >= 256 ? 4 * BW : 1024); }

size_t sparse_smem(const Dims &dm, int m, int node_bits_stride, int slots) {
    const int cc = sparse_cand_cap(dm.BW, m), scap = sparse_surv_cap(dm.BW);
    const size_t pick = al16((size_t)cc * 8) + al16((size_t)cc * 4) + al16((size_t)scap * 8) +
                        al16((size_t)scap * 4) + al16((size_t)(dm.BW + 1) * 4) + 2 * al16((size_t)dm.BW * 4) +
                        finish_bytes(dm.BW, dm.BW, dm.S, 0) + 64;
    // phase 1: the staged rows, then the per-warp token lists
    const size_t rows = slots * al16((size_t)dm.V * 4) + (size_t)kSpWarps * node_bits_stride * 4;
    return pick > rows ? pick : rows;
}

// Phase 2, by the request's last CTA.  tau = the BW-th best of the beams'
// heads: at least BW real candidates rank at or above it, so every winner
// does.  Survivors = the head keys at or above tau, plus, for a beam whose
// whole head survived and that has more entries than its head holds, its
// further keys at or above tau from the key buffer.  Then the exact radix
// select of the BW best survivors, the ordering, the outputs and the
// rewiring.  Exact fallbacks: survivors beyond the shared-memory buffer select
// from the key buffer; a request with more CSR entries than the key buffer
// holds selects from the scores.
__device__ void select_request(const SelectArgs &a, int r, uint8_t *smem, int *hist, int *scan_w,
                               uint64_t *red_k, int *sc, int *red_i) {
    const Dims dm = a.dims;
    const int BW = dm.BW, m = a.head_m, tid = threadIdx.x;
    const int64_t rb = (int64_t)r * BW;
    const int cc = sparse_cand_cap(BW, m), scap = sparse_surv_cap(BW);
    uint8_t *p = smem;
    uint64_t *hk = reinterpret_cast<uint64_t *>(p);
    p += al16((size_t)cc * 8);
    int *he = reinterpret_cast<int *>(p);
    p += al16((size_t)cc * 4);
    uint64_t *sk = reinterpret_cast<uint64_t *>(p);
    p += al16((size_t)scap * 8);
    int *se = reinterpret_cast<int *>(p);
    p += al16((size_t)scap * 4);
    int *sat = reinterpret_cast<int *>(p);   // beams whose further keys must be read
    p += al16((size_t)(BW + 1) * 4);
    float *cum_s = reinterpret_cast<float *>(p);
    p += al16((size_t)BW * 4);
    float *lse_s = reinterpret_cast<float *>(p);
    p += al16((size_t)BW * 4);
    const FinishSmem f = carve_finish(p, BW, BW, dm.S, 0);
    int *cnts = reinterpret_cast<int *>(p + finish_bytes(BW, BW, dm.S, 0));   // [0] survivors, [1] saturated

    // every load below is independent of the others: one round trip.  Entry
    // numbering of the key buffer: CSR rows as in the mask; node masks row b
    // at b * row_stride.
    const bool csr = a.mask_kind == XGR_MASK_CSR;
    const int n = min(max(a.n_live[r], 0), BW);
    const int base = csr ? a.row_ptr[rb] : 0;
    const int64_t E = csr ? (int64_t)a.row_ptr[rb + BW] - base : (int64_t)BW * a.row_stride;
    for (int i = tid; i < BW * m; i += kSpThreads) {
        const int b = i / m;
        hk[i] = b < n ? __ldcg(a.head_k + rb * m + i) : kNoKey;
        he[i] = __ldcg(a.head_e + rb * m + i);
    }
    int c = 0;
    for (int b = tid; b < BW; b += kSpThreads) {
        c += b < n ? __ldcg(a.row_cnt + rb + b) : 0;
        const int len = b < n ? __ldcg(a.row_len + rb + b) : 0, cb = __ldcg(a.row_cb + rb + b);
        f.rl[b] = len;
        f.cb[b] = b < n ? cb : -1;
        f.ce[b] = (b < n && cb >= 0) ? cb + len : -1;
    }
    for (int b = tid; b <= BW; b += kSpThreads)
        f.rp[b] = csr ? a.row_ptr[rb + b] - base : b * a.row_stride;
    if (a.rewire) stage_rows(a, rb, n, f);
    if (E > a.key_cap)
        for (int b = tid; b < n; b += kSpThreads) {
            cum_s[b] = a.cum[rb + b];
            lse_s[b] = a.logits ? __ldcg(a.row_lse + rb + b) : 0.f;
        }
    if (tid == 0) {
        *f.cnt = 0;
        cnts[0] = 0;
        cnts[1] = 0;
    }
    const int total = block_sum_int(c, red_i);   // valid candidates of the request (+ a barrier)
    const int want = min(BW, total);
    uint64_t prefix = ~0ull, mask = 0;
    bool ranked = false;   // the winners were placed in rank order
    const uint64_t *keys = a.keys + (int64_t)r * a.key_cap;
    if (csr && E > a.key_cap) {
        // the key buffer overflowed: exact selection over every candidate
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
        if (want > 0 && want < total) radix_select(cand, f.rp[n], want, hist, sc, prefix, mask);
        collect(cand, f.rp[n], prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
    } else if (want > 0) {
        // tau from the heads (every head key is a real candidate)
        int c0 = 0;
        for (int i = tid; i < BW * m; i += kSpThreads) c0 += hk[i] != kNoKey;
        const int in_heads = block_sum_int(c0, red_i);
        uint64_t tau = kNoKey;
        if (total > BW && in_heads >= BW) {
            uint64_t tp, tm;
            smem_radix_select(hk, BW * m, BW, hist, scan_w, red_k, sc, tp, tm);
            tau = selected_max(hk, BW * m, tp, tm, red_k);
        }
        // survivors from the heads; beams whose whole head survived and that have
        // more entries go on the saturated list
        for (int i = tid; i < BW * m; i += kSpThreads) {
            const uint64_t key = hk[i];
            if (key == kNoKey || key > tau) continue;
            const int pos = atomicAdd(&cnts[0], 1);
            if (pos < scap) {
                sk[pos] = key;
                se[pos] = he[i];
            }
            const int b = i / m;
            if (i % m == m - 1 && f.rl[b] > m) sat[atomicAdd(&cnts[1], 1)] = b;
        }
        __syncthreads();
        const int n_sat = cnts[1];
        for (int q = 0; q < n_sat; ++q) {   // their keys beyond the head (worse than its last)
            const int b = sat[q];
            const uint64_t last = hk[b * m + m - 1];
            const int e1 = (int)min((int64_t)f.rp[b] + f.rl[b], E);
            for (int e = max(f.rp[b], 0) + tid; e < e1; e += kSpThreads) {
                const uint64_t key = __ldcg(keys + e);
                if (key == kNoKey || key > tau || key <= last) continue;
                const int pos = atomicAdd(&cnts[0], 1);
                if (pos < scap) {
                    sk[pos] = key;
                    se[pos] = e;
                }
            }
        }
        __syncthreads();
        const int ns = cnts[0];
        if (ns <= kRankDirect) {   // few survivors: each one's rank by counting
            place_by_rank(sk, se, ns, want, f);
            ranked = true;
        } else if (ns <= scap) {
            if (want < ns) smem_radix_select(sk, ns, want, hist, scan_w, red_k, sc, prefix, mask);
            collect(ListCand<false>{sk}, ns, prefix, mask, BW, [&](int64_t i) { return se[i]; }, f);
        } else {   // more survivors than the buffer: exact selection over the key buffer
            const KeyCand cand{keys, tau, f.rp, f.rl, csr ? 0 : a.row_stride, n};
            radix_select(cand, E, want, hist, sc, prefix, mask);
            collect(cand, E, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
        }
    }
    __syncthreads();
    finish_request(a, r, ranked ? want : min(*f.cnt, want), f, ranked);
}

__global__ void __launch_bounds__(kSpThreads) select_sparse_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full_bar[kSpWarps];
    __shared__ int hist[kRadixBins];
    __shared__ int scan_w[32];
    __shared__ int red_i[32];
    __shared__ uint64_t red_k[32];
    __shared__ int sc[4];
    __shared__ int last;
    const Dims dm = a.dims;
    const int C = a.sp_parts, R = a.sp_rows;
    const int r = blockIdx.x / C, part = blockIdx.x % C;
    const int warp = threadIdx.x / 32;
    const int64_t rb = (int64_t)r * dm.BW;
    const int n_live = min(max(a.n_live[r], 0), dm.BW);
    const int base = a.mask_kind == XGR_MASK_CSR ? a.row_ptr[rb] : 0;
    uint64_t *keys = a.keys + (int64_t)r * a.key_cap;
    const int b0 = part * R, b1 = min(dm.BW, part * R + R);
    // short logits rows (every warp's fits beside the others') are staged by
    // the TMA engine, one slot and one landing barrier per warp; longer ones
    // stream through registers
    const int ns = a.sp_slots;   // 0 or R
    const size_t xb = al16((size_t)dm.V * 4);
    float *xslot = reinterpret_cast<float *>(smem);
    int *wtok = reinterpret_cast<int *>(smem + ns * xb) + (size_t)warp * a.row_stride;   // NODE_BITS rows
    if (ns > 0) {
        if (threadIdx.x == 0) {
            for (int w = 0; w < ns; ++w) mbar_init(smem_u32(&full_bar[w]), 1);
            fence_mbar_init();
            for (int w = 0; w < min(ns, b1 - b0); ++w) {
                if (b0 + w >= n_live) continue;   // dead rows are not read
                mbar_expect_tx(smem_u32(&full_bar[w]), (uint32_t)dm.V * 4u);
                bulk_g2s(smem_u32(xslot + (size_t)w * (xb / 4)), a.scores + (rb + b0 + w) * dm.V,
                         (uint32_t)dm.V * 4u, smem_u32(&full_bar[w]));
            }
        }
        __syncthreads();
    }
    const int b = b0 + warp;
    if (b < b1) {
        const float *xs = nullptr;
        if (ns > 0 && b < n_live) {
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full_bar[warp]), 0, nullptr))) {
                if ((threadIdx.x & 31) == 0) set_status(a.status, XGR_DEV_TIMEOUT);
            } else {
                xs = xslot + (size_t)warp * (xb / 4);
            }
        }
        sparse_row(a, r, b, n_live, base, keys, wtok, xs);
    }
    // the request's last CTA to arrive selects
    __threadfence();   // this thread's keys and head are visible before the ticket
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&a.ticket[r], 1u) == (unsigned)(C - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    select_request(a, r, smem, hist, scan_w, red_k, sc, red_i);
    if (threadIdx.x == 0) a.ticket[r] = 0;   // zero again for the next call
}

// ------------------------------------------------------------------ dense step

// The first step: one live beam per request and the dense bitset of valid
// first tokens.  One CTA of kDnThreads per request: the beam's score row is
// staged by one bulk copy; its log-sum-exp from per-warp partials; every
// thread takes the keys of its tokens t = tid + kDnThreads * u and keeps their
// minimum -- kDnThreads real candidates at most; tau = the BW-th best of
// these (so at least BW candidates rank at or above it); the survivors at or
// above tau (each thread recomputes its keys from the staged row) are ranked
// by counting, then finish_request.
constexpr int kDnThreads = 512;
__host__ __device__ inline int dense_surv_cap(int BW) { return BW >= 512 ? 4 * BW : 2048; }
__host__ __device__ inline size_t dense_x_bytes(int V) { return al16((size_t)V * 4); }
__host__ __device__ inline size_t dense_bits_bytes(int V) { return al16((size_t)((V + 31) / 32) * 4); }

size_t dense_smem(const Dims &dm) {
    const int scap = dense_surv_cap(dm.BW);
    return dense_x_bytes(dm.V) + dense_bits_bytes(dm.V) + al16((size_t)kDnThreads * 8) +
           al16((size_t)scap * 8) + al16((size_t)scap * 4) + finish_bytes(dm.BW, 1, dm.S, (dm.V + 31) / 32) + 64;
}

__global__ void __launch_bounds__(kDnThreads) select_dense_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar_mem;
    __shared__ float red_f[2 * (kDnThreads / 32)];
    __shared__ int red_i[32];
    __shared__ int scan_w[32];
    __shared__ uint64_t red_k[32];
    __shared__ int hist[kRadixBins];
    __shared__ int sc[4];
    __shared__ int cnts[1];
    constexpr int kWarps = kDnThreads / 32;
    const Dims dm = a.dims;
    const int V = dm.V, BW = dm.BW, nw = (V + 31) / 32;
    const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rb = (int64_t)r * BW;
    const int scap = dense_surv_cap(BW);
    uint8_t *p = smem;
    float *x = reinterpret_cast<float *>(p);
    p += dense_x_bytes(V);
    uint32_t *bits = reinterpret_cast<uint32_t *>(p);
    p += dense_bits_bytes(V);
    uint64_t *mins = reinterpret_cast<uint64_t *>(p);
    p += al16((size_t)kDnThreads * 8);
    uint64_t *sk = reinterpret_cast<uint64_t *>(p);
    p += al16((size_t)scap * 8);
    int *se = reinterpret_cast<int *>(p);
    p += al16((size_t)scap * 4);
    const FinishSmem f = carve_finish(p, BW, 1, dm.S, nw);
    const float *xg = a.scores + rb * V;   // beam 0 of request r
    const uint32_t bar = smem_u32(&bar_mem);
    const bool bulk = (V & 3) == 0 && (reinterpret_cast<uintptr_t>(xg) & 15) == 0;
    const int n = min(max(a.n_live[r], 0), 1);
    if (tid == 0) {
        *f.cnt = 0;
        cnts[0] = 0;
        if (bulk && n > 0) {
            mbar_init(bar, 1);
            fence_mbar_init();
            mbar_expect_tx(bar, (uint32_t)V * 4u);
            bulk_g2s(smem_u32(x), xg, (uint32_t)V * 4u, bar);
        }
    }
    const float cum = a.cum[rb];
    // the mask with the tokens past V cleared; the valid-candidate count
    int c = 0;
    for (int w = tid; w < nw; w += kDnThreads) {
        const uint32_t v = a.bits[w] & (32 * w + 32 <= V ? ~0u : (1u << (V & 31)) - 1u);
        bits[w] = v;
        c += __popc(v);
    }
    if (a.rewire) {
        stage_rows(a, rb, n, f);
        if (a.trie.root_bits) {
            // root children: bitset and exclusive prefix popcounts (trie order =
            // token order); thread t owns words [t*wpt, t*wpt + wpt)
            const int wpt = (nw + kDnThreads - 1) / kDnThreads;
            int cw = 0;
            for (int k = 0; k < wpt; ++k) {
                const int w = tid * wpt + k;
                if (w < nw) {
                    const uint32_t v = a.trie.root_bits[w];
                    f.root[w] = v;
                    cw += __popc(v);
                }
            }
            int tot;
            int pre = block_exclusive_scan_int(cw, scan_w, &tot);
            for (int k = 0; k < wpt; ++k) {
                const int w = tid * wpt + k;
                if (w < nw) {
                    f.root[nw + w] = (uint32_t)pre;
                    pre += __popc(f.root[w]);
                }
            }
        }
    }
    if (!bulk && n > 0)
        for (int i = tid; i < V; i += kDnThreads) x[i] = xg[i];
    const int total = n > 0 ? block_sum_int(c, red_i) : 0;   // (+ a barrier)
    if (bulk && n > 0 && !mbar_wait(bar, 0, nullptr)) set_status(a.status, XGR_DEV_TIMEOUT);
    const int want = min(BW, total);
    float lse = 0.f;
    if (a.logits && want > 0) {   // per-warp (max, sum) over a slice, then combined
        const int per = (V + kWarps - 1) / kWarps;
        float mw = -INFINITY, sw = 0.f;
        bool nan = false;
        for (int i = warp * per + lane; i < min(V, warp * per + per); i += 32) {
            const float v = x[i];
            nan |= v != v;
            if (v > mw) {
                sw = mw == -INFINITY ? 0.f : sw * ex2f((mw - v) * kLog2e);
                mw = v;
            }
            if (mw != -INFINITY) sw += ex2f((v - mw) * kLog2e);
        }
        if (__any_sync(0xffffffffu, nan) && lane == 0) set_status(a.status, XGR_DEV_NAN);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, mw, o), s2 = __shfl_xor_sync(0xffffffffu, sw, o);
            lse_pair_merge(mw, sw, m2, s2);
        }
        if (lane == 0) {
            red_f[2 * warp] = mw;
            red_f[2 * warp + 1] = sw;
        }
        __syncthreads();
        float M = red_f[0], Ssum = red_f[1];
        for (int k = 1; k < kWarps; ++k) lse_pair_merge(M, Ssum, red_f[2 * k], red_f[2 * k + 1]);
        lse = M + logf(Ssum);
    }
    DenseCand cand{x, bits, cum, lse, V, a.logits, a.status};
    uint64_t prefix = ~0ull, mask = 0;
    bool ranked = false;
    if (want > 0) {
        // each thread's best key: real candidates for the threshold
        uint64_t mn = kNoKey;
        for (int t = tid; t < V; t += kDnThreads) {
            uint64_t key = kNoKey;
            if (cand(t, key) && key < mn) mn = key;
        }
        mins[tid] = mn;
        const int n_min = block_sum_int(mn != kNoKey ? 1 : 0, red_i);   // (+ a barrier)
        uint64_t tau = kNoKey;
        if (total > BW && n_min >= BW) {
            uint64_t tp, tm;
            smem_radix_select(mins, kDnThreads, BW, hist, scan_w, red_k, sc, tp, tm);
            tau = selected_max(mins, kDnThreads, tp, tm, red_k);
        }
        // survivors: every key at or above tau, recomputed from the staged row
        for (int t = tid; t < V; t += kDnThreads) {
            uint64_t key;
            if (!cand(t, key) || key > tau) continue;
            const int pos = atomicAdd(&cnts[0], 1);
            if (pos < scap) {
                sk[pos] = key;
                se[pos] = t;
            }
        }
        __syncthreads();
        const int ns = cnts[0];
        if (ns <= kRankDirect) {
            place_by_rank(sk, se, ns, want, f);
            ranked = true;
        } else if (ns <= scap) {
            if (want < ns) smem_radix_select(sk, ns, want, hist, scan_w, red_k, sc, prefix, mask);
            collect(ListCand<false>{sk}, ns, prefix, mask, BW, [&](int64_t i) { return se[i]; }, f);
        } else {   // more survivors than the buffer: exact selection over every token
            radix_select(cand, V, want, hist, sc, prefix, mask);
            collect(cand, V, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
        }
    }
    __syncthreads();
    finish_request(a, r, ranked ? want : min(*f.cnt, want), f, ranked);
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

int select_head_m(int BW) { return BW >= 1024 ? 4 : 8; }

size_t select_ticket_offset(int B, int BW) {
    const size_t rows = (size_t)B * BW, m = (size_t)select_head_m(BW);
    return 4 * al256(rows * 4) + al256(rows * m * 8) + al256(rows * m * 4);
}

size_t select_scratch_bytes(int B, int BW, int64_t key_cap) {
    return select_ticket_offset(B, BW) + al256((size_t)B * 4) + al256((size_t)B * key_cap * 8);
}

void select_scratch_carve(uint8_t *base, int B, int BW, int64_t key_cap, SelectArgs &a) {
    const size_t rows = (size_t)B * BW;
    const int m = select_head_m(BW);
    a.row_lse = reinterpret_cast<float *>(base);
    base += al256(rows * 4);
    a.row_cnt = reinterpret_cast<int32_t *>(base);
    base += al256(rows * 4);
    a.row_len = reinterpret_cast<int32_t *>(base);
    base += al256(rows * 4);
    a.row_cb = reinterpret_cast<int32_t *>(base);
    base += al256(rows * 4);
    a.head_k = reinterpret_cast<uint64_t *>(base);
    base += al256(rows * m * 8);
    a.head_e = reinterpret_cast<int32_t *>(base);
    base += al256(rows * m * 4);
    a.ticket = reinterpret_cast<uint32_t *>(base);
    base += al256((size_t)B * 4);
    a.keys = reinterpret_cast<uint64_t *>(base);
    a.key_cap = key_cap;
    a.head_m = m;
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
        select_dense_kernel<<<dm.B, kDnThreads, smem, s>>>(a);
        return cudaGetLastError();
    }
    // sparse: one launch, sp_parts CTAs per request of R beams, one per warp
    const int R = std::min(dm.BW, kSpWarps);
    a.sp_rows = R;
    a.sp_parts = (dm.BW + R - 1) / R;
    if (a.head_m < 1 || a.head_m > 32) return cudaErrorInvalidValue;
    if (a.mask_kind != XGR_MASK_CSR && a.mask_kind != XGR_MASK_TRIE_ROWS && a.mask_kind != XGR_MASK_NODE_BITS)
        return cudaErrorInvalidValue;
    if (a.mask_kind != XGR_MASK_CSR && (int64_t)dm.BW * a.row_stride > a.key_cap) return cudaErrorInvalidValue;
    const int wt = a.mask_kind == XGR_MASK_NODE_BITS ? a.row_stride : 0;
    // logits rows through the TMA engine: as many slots of a row as fit beside
    // the token lists (each CTA takes R <= 8 rows, one per warp)
    a.sp_slots = 0;
    if (a.logits && (dm.V & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0) {
        const size_t room = (200u << 10) - (size_t)kSpWarps * wt * 4;
        // only when every warp gets a slot of its own: a slot handed from warp to
        // warp would leave the later rows waiting for the earlier ones
        if (room / al16((size_t)dm.V * 4) >= (size_t)R) a.sp_slots = R;
    }
    const size_t smem = sparse_smem(dm, a.head_m, wt, a.sp_slots);
    if (smem > (220u << 10)) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem(select_sparse_kernel, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)dm.B * a.sp_parts;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    select_sparse_kernel<<<(int)grid, kSpThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace xgr

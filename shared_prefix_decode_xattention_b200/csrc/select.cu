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
//    log-sum-exp (logits); the cut comes from the threads' best keys (at
//    least BW real candidates lie at or before it), and the survivors are
//    ranked by counting.
//  * sparse masks (steps >= 1): two launches.  select_rows_kernel gives each
//    beam row a warp: its log-sum-exp (logits), the key of each of its mask
//    entries, and its head -- the beam's m best keys in order (the page's
//    ordered per-beam candidate list, cut at m).  select_pick_kernel (one CTA
//    per request) cuts at the heads (at least BW real candidates lie at or
//    before the cut, so every winner survives), gathers the survivors -- the
//    head keys, and the further keys of beams whose whole head survived --
//    and ranks them.  Both end in finish_request: the ordering, the outputs
//    and the rewiring.
//  Every kernel is launched as a programmatic dependent of the kernel before
//  it; the one-CTA-per-request kernels run a dry pass of their own code on
//  synthetic shared-memory data before they wait for that kernel, so the
//  instruction fetches of code that runs once per launch are not on the
//  critical path.
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

// Warp-wide reductions by the warp-reduce instruction (redux.sync, 32-bit
// operands): a 64-bit minimum is the minimum of the high words, then of the
// low words of the lanes that hold it -- two reduce steps instead of five
// dependent shuffle-and-compare levels.  Every lane of the warp takes part.
__device__ __forceinline__ uint64_t warp_min_u64(uint64_t v) {
    const uint32_t hi = (uint32_t)(v >> 32), lo = (uint32_t)v;
    const uint32_t mh = __reduce_min_sync(0xffffffffu, hi);
    const uint32_t ml = __reduce_min_sync(0xffffffffu, hi == mh ? lo : 0xffffffffu);
    return ((uint64_t)mh << 32) | ml;
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
    const uint32_t hi = (uint32_t)(v >> 32), lo = (uint32_t)v;
    const uint32_t mh = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t ml = __reduce_max_sync(0xffffffffu, hi == mh ? lo : 0u);
    return ((uint64_t)mh << 32) | ml;
}
__device__ __forceinline__ int warp_sum_int(int v) { return __reduce_add_sync(0xffffffffu, v); }
__device__ __forceinline__ float warp_sum_f(float v) {
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
// dry: the same instructions with every global load and store turned off (a
// warm-up pass over synthetic shared-memory data)
__device__ void finish_request(const SelectArgs &a, int r, int n_win, const FinishSmem &f,
                               bool in_rank_order, bool dry) {
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
        if (!a.rewire || a.dense || i >= n_win || dry) continue;
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
    const bool wr = !dry;   // (predicated stores: a dry pass fetches the same code)
    for (int i = threadIdx.x; i < BW; i += blockDim.x) {
        if (i < n_win) {
            const int nb = f.rank[i];
            const int64_t o = rb + nb;
            const uint64_t key = f.win_k[i];
            const uint32_t lo = (uint32_t)key;
            const int p = (int)(lo / (uint32_t)V), t = (int)(lo % (uint32_t)V);
            const float sc = desc_bits_to_score((uint32_t)(key >> 32));
            if (wr) {
                a.parent[o] = p;
                a.token[o] = t;
                a.cum_out[o] = sc;
            }
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
                if (wr) {
                    a.st.anc[o * S + j] = av;
                    a.st.seq[o * S + j] = sv;
                }
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
                } else if (wr) {
                    child = find_child(a.trie, s, node, t);
                }
            } else {
                // the mask row of parent p lists its children in trie order, so
                // the entry index located the child (checked above)
                child = f.win_e[i];
            }
            if (wr) {
                if (child < 0) set_status(a.status, XGR_DEV_MASK);
                a.st.node[o] = child;
                a.st.cum[o] = sc;
            }
        } else if (wr) {
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
    if (threadIdx.x == 0 && wr) {
        a.n_out[r] = n_win;
        if (a.rewire) a.st.n_live[r] = n_win;
    }
}

// ------------------------------------------------------------------ sparse steps

// Phase 1 (select_rows_kernel): request r gets sp_parts CTAs of 32 * sp_rows
// threads; CTA `part` takes beams [part*R, part*R + R) (R = sp_rows), one warp
// per beam, so no reduction spans more than one warp.  Per beam:
//  * logits mode: the row's log-sum-exp over the full vocabulary, streamed
//    from HBM through a ring of bulk copies (online max / sum of exponentials
//    per lane, then across the warp), while the mask lookups and the first
//    entries' scores are fetched;
//  * the key of every mask entry, written to the request's key buffer;
//  * the beam's head: its m best keys with their entries, ascending (the
//    page's per-beam ordered candidate list, cut at m).
// Phase 2 (select_pick_kernel) selects for the whole request from the heads.
constexpr int kSpThreads = 256;   // the pick kernel's CTA
constexpr int kSpWarps = kSpThreads / 32;
// The rows kernel's CTA takes kRowWarpsWide beam rows with five-stage rings
// (one CTA per SM) when the grid fits one wave, else kRowWarpsNarrow rows with
// three-stage rings (three CTAs per SM: more rows stream at once, and one
// CTA's keys and head merge overlap the others' streams).
constexpr int kRowWarpsWide = 8, kRingWide = 5;
constexpr int kRowWarpsNarrow = 4, kRingNarrow = 3;
constexpr int kSpKpc = 8;             // CSR entries per lane in one pass of the key loop (many-wave shape)
// the one-wave shape's rows (small batches, where each row's latency is the
// launch's) take half as many a pass: cheaper merge rounds over a short row;
// a longer row's later passes go through the insertion path (measured: the
// 128-beam decode 0.4-1.0 us faster; 4 for the many-wave shape's long rows
// cost the 512-beam selection 2.5%)
constexpr int kSpKpcWide = 4;
constexpr int kRingStageBytes = 4096;  // one stage of a warp's row stream
constexpr int kWtokCap = 1024;         // NODE_BITS tokens listed beside the ring before the stream
// a warp's area: its ring of `ring` stages, then its token list
__host__ __device__ inline size_t ring_warp_bytes(int ring) { return (size_t)ring * kRingStageBytes + kWtokCap * 4; }

// max that returns NaN when either operand is NaN
__device__ __forceinline__ float max_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

// Folds 32 values into a lane's running (max m, sum s of 2^((v - m) log2 e)):
// the values' maximum over eight independent chains, s rescaled when the
// maximum grows, then the exponentials into eight independent partial sums.
// A NaN value turns s into NaN (reported by the caller through the row's
// log-sum-exp).
__device__ __forceinline__ void lse_fold32(const float (&v)[32], float &m, float &s) {
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mx[e] = v[e];
#pragma unroll
    for (int e = 8; e < 32; ++e) mx[e & 7] = max_nan(mx[e & 7], v[e]);
    const float bm = max_nan(max_nan(max_nan(mx[0], mx[1]), max_nan(mx[2], mx[3])),
                             max_nan(max_nan(mx[4], mx[5]), max_nan(mx[6], mx[7])));
    if (!(bm <= m)) {   // the maximum grew (or a NaN arrived)
        s = m == -INFINITY ? 0.f : s * ex2f((m - bm) * kLog2e);
        m = bm;
    }
    if (m != -INFINITY) {
        const float mk = m * kLog2e;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = ex2f(fmaf(v[e], kLog2e, -mk));
#pragma unroll
        for (int e = 8; e < 32; ++e) acc[e & 7] += ex2f(fmaf(v[e], kLog2e, -mk));
        s += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    }
}

__device__ __forceinline__ float warp_lse_merge(float m, float s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_pair_merge(m, s, m2, s2);
    }
    return m + logf(s);
}

// A warp's score-row stream: the row's bytes go through the warp's ring of
// RING shared-memory stages by bulk copies (the TMA engine), issued
// by lane 0 and landing on one mbarrier per stage; all stages but the one the
// lanes fold are in flight.  The same warp issues, waits for and refills each
// stage in order, so a stage's barrier is never more than one phase ahead of
// its waiter (parity = use count & 1).  Needs the row 16-byte aligned and a
// multiple of 16 bytes long.
template <int RING>
struct RowStream {
    const uint8_t *src;
    int bytes, nst;
    float4 *stages;   // the warp's stage area
    uint32_t bar0;    // its RING barriers (8 bytes apart)
    __device__ void issue(int st) const {   // lane 0
        if (st >= nst) return;
        const int slot = st % RING, off = st * kRingStageBytes;
        const uint32_t n = (uint32_t)min(kRingStageBytes, bytes - off);
        const uint32_t bar = bar0 + 8u * (uint32_t)slot;
        mbar_expect_tx(bar, n);
        bulk_g2s(smem_u32(stages) + (uint32_t)(slot * kRingStageBytes), src + off, n, bar);
    }
};

// starts the stream: the first RING stages go out (barriers initialised
// by lane 0 here, before any lane waits on them)
template <int RING>
__device__ RowStream<RING> row_stream_start(const float *x, int V, float4 *ring_area, uint64_t *bars) {
    RowStream<RING> rs;
    rs.src = reinterpret_cast<const uint8_t *>(x);
    rs.bytes = V * 4;
    rs.nst = (rs.bytes + kRingStageBytes - 1) / kRingStageBytes;
    rs.stages = ring_area;
    rs.bar0 = smem_u32(bars);
    if ((threadIdx.x & 31) == 0) {
        for (int i = 0; i < RING; ++i) mbar_init(rs.bar0 + 8u * (uint32_t)i, 1);
        fence_mbar_init();
        for (int st = 0; st < min(rs.nst, RING); ++st) rs.issue(st);
    }
    __syncwarp();
    return rs;
}

// Natural-log log-sum-exp of the streamed row by its warp (every lane gets it;
// NaN when the row holds a NaN).  Each stage is folded by all lanes, then
// refilled with the stage RING ahead.  A stage that never lands (a
// bounded wait runs out) sets XGR_DEV_TIMEOUT; the copies still in flight are
// waited for (bounded) before the ring is given back.
template <int RING>
__device__ float row_stream_lse(const RowStream<RING> &rs, int32_t *status) {
    const int lane = threadIdx.x & 31;
    float m = -INFINITY, s = 0.f;
    int st = 0;
    for (; st < rs.nst; ++st) {
        const int slot = st % RING;
        const uint32_t bar = rs.bar0 + 8u * (uint32_t)slot;
        if (!__all_sync(0xffffffffu, mbar_wait(bar, (uint32_t)(st / RING) & 1u, nullptr))) break;
        const float4 *src = rs.stages + slot * (kRingStageBytes / 16);
        const int n4 = min(kRingStageBytes, rs.bytes - st * kRingStageBytes) / 16;
        float v[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = u * 32 + lane;
            const float4 q = i < n4 ? src[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            v[4 * u] = q.x;
            v[4 * u + 1] = q.y;
            v[4 * u + 2] = q.z;
            v[4 * u + 3] = q.w;
        }
        lse_fold32(v, m, s);
        __syncwarp();   // every lane has read the stage
        if (lane == 0 && st + RING < rs.nst) {
            fence_async_smem();   // those reads before the bulk copy's writes
            rs.issue(st + RING);
        }
    }
    if (st < rs.nst) {   // timed out: let the issued copies land before the ring is reused
        if (lane == 0) {
            set_status(status, XGR_DEV_TIMEOUT);
            for (int q = st; q < min(rs.nst, st + RING); ++q)
                mbar_wait(rs.bar0 + 8u * (uint32_t)(q % RING), (uint32_t)(q / RING) & 1u, nullptr);
        }
        __syncwarp();
    }
    return warp_lse_merge(m, s);
}

// the same for rows the ring cannot take (V % 4 != 0 or unaligned): plain loads
__device__ float warp_row_lse_plain(const float *x, int V) {
    const int lane = threadIdx.x & 31;
    float m = -INFINITY, s = 0.f;
    for (int i0 = 0; i0 < V; i0 += 32 * 32) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = i0 + e * 32 + lane;
            v[e] = i < V ? __ldg(x + i) : -INFINITY;
        }
        lse_fold32(v, m, s);
    }
    return warp_lse_merge(m, s);
}

// Merges the keys c[] of every lane (entries ce[]) into the warp's running
// head: afterwards lanes 0..m-1 hold the m smallest keys seen so far, in
// ascending order (kNoKey pads), with their entries.  Keys are unique.
// Only keys below the head's m-th key can enter it.  When at most
// kHeadInsertMax of them do (a sparse row, or a long row's later pass once
// its head is full), each is inserted into the lane-distributed sorted head
// (its rank by one ballot, the lanes above shifted up by one); otherwise m
// rounds of a warp minimum.  c[] is consumed.
constexpr int kHeadInsertMax = 32;
template <int KPC>
__device__ __forceinline__ void warp_head_merge(uint64_t (&c)[KPC], const int (&ce)[KPC], uint64_t &run,
                                                int &run_e, int m) {
    const int lane = threadIdx.x & 31;
    uint64_t bound = __shfl_sync(0xffffffffu, run, m - 1);   // the head's m-th key (kNoKey: not full)
    int q = 0;
#pragma unroll
    for (int u = 0; u < KPC; ++u) q += c[u] < bound;
    const int entering = __reduce_add_sync(0xffffffffu, q);
    if (entering == 0) return;
    if (entering <= kHeadInsertMax) {
#pragma unroll
        for (int u = 0; u < KPC; ++u) {
            // a key at or above the bound now cannot enter later: the bound only falls
            unsigned who = __ballot_sync(0xffffffffu, c[u] < bound);
            while (who) {
                const int src = __ffs(who) - 1;
                who &= who - 1;
                const uint64_t x = __shfl_sync(0xffffffffu, c[u], src);
                const int xe = __shfl_sync(0xffffffffu, ce[u], src);
                if (x >= bound) continue;   // (uniform) passed by keys inserted meanwhile
                const int pos = __popc(__ballot_sync(0xffffffffu, lane < m && run < x));
                const uint64_t up = __shfl_up_sync(0xffffffffu, run, 1);
                const int up_e = __shfl_up_sync(0xffffffffu, run_e, 1);
                if (lane > pos && lane < m) {
                    run = up;
                    run_e = up_e;
                }
                if (lane == pos) {
                    run = x;
                    run_e = xe;
                }
                bound = __shfl_sync(0xffffffffu, run, m - 1);
            }
        }
        return;
    }
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

// The valid tokens of a NODE_BITS row, compacted into wtok[0..) in token
// order (the node's children in trie order) by one warp; returns their count.
// first: the first pass's words, when the caller loaded them already.
__device__ int warp_bits_to_tokens(const uint32_t *wb, int nw, int *wtok, int cap,
                                   const uint32_t *first = nullptr) {
    const int lane = threadIdx.x & 31;
    int cnt = 0;
    for (int w0 = 0; w0 < nw; w0 += 32 * 8) {
        uint32_t wv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {   // up to 256 words in flight per pass
            const int w = w0 + u * 32 + lane;
            wv[u] = (w0 == 0 && first) ? first[u] : w < nw ? __ldg(wb + w) : 0u;
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
// listed in the warp's token area).
//
// row_prep runs before the kernel waits for the kernel before it: it reads
// only the beam state, which the previous selection wrote (that kernel had
// completed before the one before this kernel started), and the mask tables.
// row_run follows the wait: in logits mode the row streams through the warp's
// ring for its log-sum-exp while the first pass's scores are fetched.  area:
// the warp's ring_warp_bytes(RING) of shared memory (16-byte aligned);
// bars: its RING mbarriers.
template <int KPC>
struct RowPrep {
    bool live;
    float cum;
    int node, n_e, cb, nb_full;
    int64_t ebase;
    const int32_t *tokp;
    int tk0[KPC];   // the first pass's tokens (lane j: entries j, j + 32, ...)
};

template <int RING, int KPC>
__device__ RowPrep<KPC> row_prep(const SelectArgs &a, int r, int b, int n_live, int base, uint8_t *area) {
    const int lane = threadIdx.x & 31;
    const Dims dm = a.dims;
    const int s = a.step;
    const int64_t row = (int64_t)r * dm.BW + b;
    int *wtok = reinterpret_cast<int *>(area + (size_t)RING * kRingStageBytes);
    RowPrep<KPC> p;
    p.live = b < n_live;
    p.cum = a.cum[row];
    const bool csr = a.mask_kind == XGR_MASK_CSR;
    const int beg = csr ? a.row_ptr[row] : 0, end = csr ? a.row_ptr[row + 1] : 0;
    p.node = (csr ? (a.rewire && p.live) : p.live) ? (csr ? a.st.node[row] : a.row_node[row]) : -1;
    p.tokp = nullptr;
    p.n_e = 0;
    p.cb = -1;
    p.nb_full = 0;
    if (csr) {
        p.tokp = a.cols + beg;
        p.n_e = max(0, end - beg);
        p.ebase = beg - base;
        if (s < a.trie.levels && p.node >= 0 && p.node < a.trie.n_nodes[s]) p.cb = a.trie.ptr[s][p.node];
    } else {
        p.ebase = (int64_t)b * a.row_stride;
        if (p.node >= 0 && p.node < a.n_nodes) {
            const uint32_t *wb = a.node_bits + (int64_t)p.node * a.n_words;
            uint32_t first[8];   // the bitset's first words load beside the child range
            if (a.mask_kind == XGR_MASK_NODE_BITS)
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int w = u * 32 + lane;
                    first[u] = w < a.n_words ? __ldg(wb + w) : 0u;
                }
            const int lo = a.node_ptr[p.node], hi = a.node_ptr[p.node + 1];
            p.cb = lo;
            p.n_e = min(max(0, hi - lo), a.row_stride);
            if (a.mask_kind == XGR_MASK_TRIE_ROWS) {
                p.tokp = a.node_tok + lo;
            } else {
                p.nb_full = warp_bits_to_tokens(wb, a.n_words, wtok, kWtokCap, first);
                if (p.nb_full != hi - lo && lane == 0) set_status(a.status, XGR_DEV_MASK);   // table and trie disagree
                p.n_e = min(p.nb_full, a.row_stride);
                p.tokp = wtok;
            }
        } else if (p.live && lane == 0) {
            set_status(a.status, XGR_DEV_INDEX);
        }
    }
#pragma unroll
    for (int u = 0; u < KPC; ++u) {
        const int j = u * 32 + lane;
        p.tk0[u] = (j < p.n_e && p.live) ? p.tokp[j] : -1;
    }
    return p;
}

template <int RING, int KPC>
__device__ void row_run(const SelectArgs &a, int r, int b, const RowPrep<KPC> &p, uint64_t *keys, uint8_t *area,
                        uint64_t *bars) {
    const int lane = threadIdx.x & 31;
    const Dims dm = a.dims;
    const int V = dm.V, m = a.head_m;
    const int64_t row = (int64_t)r * dm.BW + b;
    const bool live = p.live;
    const float *x = a.scores + row * V;
    float4 *ring = reinterpret_cast<float4 *>(area);
    const bool stream = a.logits && live && (V & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0;
    RowStream<RING> rs{};
    if (stream) rs = row_stream_start<RING>(x, V, ring, bars);
    // the first pass's scores go out before the stream is folded
    float sv0[KPC];
#pragma unroll
    for (int u = 0; u < KPC; ++u) sv0[u] = (p.tk0[u] >= 0 && p.tk0[u] < V) ? __ldg(x + p.tk0[u]) : 0.f;
    float lse = 0.f;
    if (a.logits && live) {
        lse = stream ? row_stream_lse(rs, a.status) : warp_row_lse_plain(x, V);
        if (lse != lse && lane == 0) set_status(a.status, XGR_DEV_NAN);
    }
    const int32_t *tokp = p.tokp;
    if (p.nb_full > kWtokCap) {
        // a node with more children than the token area holds: list them all in
        // the ring, which the stream has given back
        int *wtok = reinterpret_cast<int *>(area);
        warp_bits_to_tokens(a.node_bits + (int64_t)p.node * a.n_words, a.n_words, wtok, a.row_stride);
        tokp = wtok;
    }
    const int n_e = p.n_e;
    uint64_t run = kNoKey;   // lane i < m: the i-th best key of the row so far
    int run_e = -1;
    int n_valid = 0;
    for (int j0 = 0; j0 < n_e; j0 += 32 * KPC) {
        uint64_t c[KPC];
        int ce[KPC];
        int tk[KPC];
        float sv[KPC];
        if (j0 == 0) {
#pragma unroll
            for (int u = 0; u < KPC; ++u) {
                tk[u] = p.tk0[u];
                sv[u] = sv0[u];
            }
        } else {
#pragma unroll
            for (int u = 0; u < KPC; ++u) {   // the entries' tokens (one round trip) ...
                const int j = j0 + u * 32 + lane;
                tk[u] = (j < n_e && live) ? tokp[j] : -1;
            }
#pragma unroll
            for (int u = 0; u < KPC; ++u)     // ... then their scores (another)
                sv[u] = (tk[u] >= 0 && tk[u] < V) ? __ldg(x + tk[u]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < KPC; ++u) {
            const int j = j0 + u * 32 + lane;
            c[u] = kNoKey;
            ce[u] = -1;
            if (j >= n_e) continue;
            const int64_t e = p.ebase + j;   // the entry, relative to the request
            uint64_t key = kNoKey;
            if (live) {
                if (tk[u] < 0 || tk[u] >= V) {
                    set_status(a.status, XGR_DEV_MASK);
                } else {
                    const float lp = a.logits ? sv[u] - lse : sv[u];
                    uint64_t k2;
                    if (make_key(p.cum, lp, b, tk[u], V, a.status, k2)) key = k2;
                }
            }
            if (e >= 0 && e < a.key_cap) keys[e] = key;
            c[u] = key;
            ce[u] = (int)e;
            n_valid += key != kNoKey;
        }
        warp_head_merge(c, ce, run, run_e, m + 1);
    }
    n_valid = warp_sum_int(n_valid);
    if (lane < m) {
        a.head_k[row * m + lane] = run;
        a.head_e[row * m + lane] = run_e;
    } else if (lane == m) {
        a.head_next[row] = run;   // the best key beyond the head
    }
    if (lane == 0) {
        a.row_cnt[row] = n_valid;
        a.row_lse[row] = lse;
        a.row_len[row] = n_e;
        a.row_cb[row] = p.cb;
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

// ---- the threshold cut
//
// The survivors of a cut are the candidates that can still be among the
// `want` best.  A binned cut maps every key's score word (key >> 32, which
// orders like the key) onto kCutBins linear bins between the smallest and
// largest score word of a reference set of real candidates (the beams' heads,
// or the threads' best keys), and finds the smallest bin B* such that at
// least `want` reference keys lie in bins <= B*.  The mapping is monotone in
// the key, so the `want` best reference keys -- and with them the `want` best
// candidates overall -- all lie in bins <= B*: "bin <= B*" keeps every winner,
// and needs one histogram pass instead of a radix select.  When every
// reference key has the same score word the cut falls back to the exact
// BW-th best reference key (tau); with fewer than `want` reference keys
// everything survives.
constexpr int kCutBins = 2048;
struct Cut {
    int mode;        // 0: everything survives; 1: binned; 2: key <= tau
    uint32_t lo;     // binned: the smallest score word
    float scale;     // binned: bins per score-word unit
    int bstar;       // binned: the last surviving bin
    uint64_t tau;    // mode 2
    __device__ __forceinline__ int bin(uint64_t key) const {
        const uint32_t d = (uint32_t)(key >> 32) - lo;
        return min(kCutBins - 1, (int)((float)d * scale));
    }
    __device__ __forceinline__ bool keep(uint64_t key) const {
        if (key == kNoKey) return false;
        return mode == 0 ? true : mode == 1 ? bin(key) <= bstar : key <= tau;
    }
};

// the request's key buffer, restricted to the survivors of the cut; with a
// row stride (node masks) only the first rl[b] slots of row b hold keys
struct KeyCand {
    const uint64_t *k;
    Cut cut;
    const int *rp, *rl;   // shared memory
    int stride, n;        // stride 0: CSR numbering (every entry written)
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        if (stride) {
            const int b = (int)(e / stride), j = (int)(e % stride);
            if (b >= n || j >= rl[b]) return false;
        }
        key = __ldcg(k + e);
        return cut.keep(key);
    }
};

// The cut over the reference keys k[0..n) (kNoKey entries are not keys), by
// the whole block (blockDim a multiple of 32, kCutBins a multiple of it).
// hist: kCutBins ints; red32: 64 words; scan_w: 32 ints; sc: 4 ints; red_k: 32
// u64 (exact fallback).
__device__ Cut make_cut(const uint64_t *k, int n, int want, int *hist, uint32_t *red32, int *scan_w, int *sc,
                        uint64_t *red_k) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    Cut c{0, 0, 0.f, 0, kNoKey};
    for (int i = tid; i < kCutBins; i += nt) hist[i] = 0;
    uint32_t lo = ~0u, hi = 0;
    int cnt = 0;
    for (int i = tid; i < n; i += nt) {
        const uint64_t key = k[i];
        if (key == kNoKey) continue;
        const uint32_t w = (uint32_t)(key >> 32);
        lo = min(lo, w);
        hi = max(hi, w);
        ++cnt;
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) {
        red32[warp] = lo;
        red32[32 + warp] = hi;
        scan_w[warp] = cnt;
    }
    __syncthreads();
    lo = ~0u;
    hi = 0;
    cnt = 0;
    for (int w = 0; w < nw; ++w) {
        lo = min(lo, red32[w]);
        hi = max(hi, red32[32 + w]);
        cnt += scan_w[w];
    }
    __syncthreads();   // red32 / scan_w are read before anyone reuses them
    if (cnt < want || want <= 0) return c;   // everything survives
    if (lo == hi) {   // one score word: the exact BW-th best key
        uint64_t tp, tm;
        smem_radix_select(k, n, want, hist, scan_w, red_k, sc, tp, tm);
        c.mode = 2;
        c.tau = selected_max(k, n, tp, tm, red_k);
        return c;
    }
    c.mode = 1;
    c.lo = lo;
    c.scale = (float)kCutBins / ((float)(hi - lo) + 1.f);
    for (int i = tid; i < n; i += nt) {
        const uint64_t key = k[i];
        if (key != kNoKey) atomicAdd(&hist[c.bin(key)], 1);
    }
    __syncthreads();
    // the bin where the running count reaches `want`: each thread scans its
    // kCutBins / nt consecutive bins
    const int bpt = kCutBins / nt;
    int sum = 0;
    for (int j = 0; j < bpt; ++j) sum += hist[tid * bpt + j];
    int total;
    int acc = block_exclusive_scan_int(sum, scan_w, &total);
    if (acc < want && acc + sum >= want) {
        for (int j = 0; j < bpt; ++j) {
            acc += hist[tid * bpt + j];
            if (acc >= want) {
                sc[0] = tid * bpt + j;
                break;
            }
        }
    }
    __syncthreads();
    c.bstar = sc[0];
    __syncthreads();   // sc is read before anyone reuses it
    return c;
}

// Global -> shared copy of `bytes` (a multiple of 4) through L2 only (the
// source may have been written by other CTAs of this launch): 16-byte
// cp.async copies when both ends are 16-byte aligned, else 4-byte loads.  The
// caller waits (cp_async_wait_all, then a barrier).
__device__ void stage_l2(void *dst, const void *src, int bytes) {
    const int tid = threadIdx.x, nt = blockDim.x;
    int i4 = 0;
    if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) == 0) {
        const int n16 = bytes >> 4;
        for (int i = tid; i < n16; i += nt)
            cp_async16(smem_u32(static_cast<uint8_t *>(dst) + 16 * i), static_cast<const uint8_t *>(src) + 16 * i);
        i4 = n16 * 4;
    }
    for (int i = i4 + tid; i < (bytes >> 2); i += nt)
        static_cast<int *>(dst)[i] = __ldcg(static_cast<const int *>(src) + i);
}

// The `want` best of the survivors sk[0..ns) (unique keys, ns >= want), placed
// in rank order: a survivor's rank is its number of better survivors (every
// thread counts for its own survivors over the whole list -- broadcast reads,
// no barrier in between), so the winners land at f.win_k[rank] directly.
constexpr int kRankDirect = 512;   // most survivors ranked by counting
__device__ void place_by_rank(const uint64_t *sk, const int *se, int ns, int want, const FinishSmem &f) {
    for (int i = threadIdx.x; i < ns; i += blockDim.x) {
        const uint64_t x = sk[i];
        int c = 0, j = 0;
        for (; j + 8 <= ns; j += 8) {   // eight broadcast reads in flight
#pragma unroll
            for (int u = 0; u < 8; ++u) c += sk[j + u] < x;
        }
        for (; j < ns; ++j) c += sk[j] < x;
        if (c < want) {
            f.win_k[c] = x;
            f.win_e[c] = se[i];
        }
    }
}

__host__ __device__ inline int sparse_cand_cap(int BW, int m) { return BW * m; }
__host__ __device__ inline int sparse_surv_cap(int BW) { return BW >= 1024 ? 4096 : (BW >= 256 ? 4 * BW : 1024); }

size_t sparse_pick_smem(const Dims &dm, int m) {
    const int cc = sparse_cand_cap(dm.BW, m), scap = sparse_surv_cap(dm.BW);
    return al16((size_t)cc * 8) + al16((size_t)cc * 4) + al16((size_t)scap * 8) + al16((size_t)scap * 4) +
           al16((size_t)(dm.BW + 1) * 4) + 2 * al16((size_t)dm.BW * 4) + al16((size_t)dm.BW * 8) +
           finish_bytes(dm.BW, dm.BW, dm.S, 0) + 64;
}
// phase 1: one ring per warp (the row stream and the NODE_BITS token list)

// Phase 2, by the request's last CTA.  The cut comes from the beams' heads
// (every head key is a real candidate, so at least BW real candidates lie at
// or before it and every winner survives).  Survivors = the head keys that
// the cut keeps, plus, for a beam whose whole head survived and that has more
// entries than its head holds, its further keys that the cut keeps (from the
// key buffer, one warp per such beam).  The survivors are ranked by counting
// (or radix-selected when there are many), then finish_request writes the
// outputs and the rewiring.  Exact fallbacks: survivors beyond the
// shared-memory buffer select from the key buffer; a request with more CSR
// entries than the key buffer holds selects from the scores.
// dry: a warm-up pass -- a synthetic request in shared memory (BW x m
// distinct head keys, no beam saturated, no trie) through the same code, with
// no global memory access.
__device__ __forceinline__ void select_request(const SelectArgs &a, int r, int n, uint8_t *smem, int *hist,
                                               int *scan_w, uint64_t *red_k, int *sc, int *red_i, uint32_t *red32,
                                               bool dry) {
    const Dims dm = a.dims;
    const int BW = dm.BW, m = a.head_m, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    uint64_t *hnext = reinterpret_cast<uint64_t *>(p);   // each beam's best key beyond its head
    p += al16((size_t)BW * 8);
    const FinishSmem f = carve_finish(p, BW, BW, dm.S, 0);
    int *cnts = reinterpret_cast<int *>(p + finish_bytes(BW, BW, dm.S, 0));   // [0] survivors, [1] saturated

    // Everything this CTA reads from phase 1 and the beam state, in one round
    // trip: the heads, each beam's entry count and first trie child, the CSR
    // row offsets and the old beam rows (rewiring) stream into shared memory
    // by cp.async while each thread loads its beams' candidate counts.  (n,
    // the live beams, is the count phase 1 read: dead beams' heads hold no
    // keys.)
    const bool csr = a.mask_kind == XGR_MASK_CSR && !dry;
    const int mshift = __ffs(m) - 1;   // m is a power of two
    int base = 0, c = 0;
    int64_t E = (int64_t)BW * (dry ? m : a.row_stride);
    if (dry) {
        n = BW;
        for (int i = tid; i < BW * m; i += kSpThreads) {
            const uint32_t h = 0xC1000000u + (((uint32_t)i * 2654435761u) >> 10);
            hk[i] = ((uint64_t)h << 32) | (uint32_t)((i >> mshift) * dm.V + (i & (m - 1)) % dm.V);
            he[i] = i;
        }
        for (int b = tid; b < BW; b += kSpThreads) {
            f.rl[b] = m;
            f.cb[b] = -1;
            f.rp[b] = b * m;
            hnext[b] = kNoKey;
        }
        if (tid == 0) f.rp[BW] = BW * m;
        c = tid == 0 ? BW * m : 0;
    } else {
        stage_l2(hk, a.head_k + rb * m, BW * m * 8);
        stage_l2(he, a.head_e + rb * m, BW * m * 4);
        stage_l2(f.rl, a.row_len + rb, BW * 4);
        stage_l2(f.cb, a.row_cb + rb, BW * 4);
        stage_l2(hnext, a.head_next + rb, BW * 8);
        if (csr) stage_l2(f.rp, a.row_ptr + rb, (BW + 1) * 4);
        if (a.rewire) {
            stage_l2(f.st_anc, a.st.anc + rb * dm.S, BW * dm.S * 4);
            stage_l2(f.st_seq, a.st.seq + rb * dm.S, BW * dm.S * 4);
            stage_l2(f.st_node, a.st.node + rb, BW * 4);
        }
        if (csr) {
            base = a.row_ptr[rb];
            E = (int64_t)a.row_ptr[rb + BW] - base;
        }
        for (int b = tid; b < n; b += kSpThreads) c += __ldcg(a.row_cnt + rb + b);
    }
    if (tid == 0) {
        *f.cnt = 0;
        cnts[0] = 0;
        cnts[1] = 0;
    }
    cp_async_wait_all();
    const int total = block_sum_int(c, red_i);   // valid candidates of the request (+ barriers)
    // the staged rows have landed: the kernel after this one (the next step's
    // attention, whose prologue prefetches the prompt K/V) may start; any
    // earlier, that traffic queued ahead of these loads
    if (!dry) griddep_launch_dependents();
    // per beam: entries relative to the request, the trie child range
    for (int b = tid; b < BW; b += kSpThreads) {
        const bool lv = b < n;
        const int len = lv ? f.rl[b] : 0, cb = lv ? f.cb[b] : -1;
        f.rl[b] = len;
        f.cb[b] = cb;
        f.ce[b] = cb >= 0 ? cb + len : -1;
        if (!dry) f.rp[b] = csr ? f.rp[b] - base : b * a.row_stride;
    }
    if (tid == 0 && !dry) f.rp[BW] = csr ? f.rp[BW] - base : BW * a.row_stride;
    if (csr && E > a.key_cap)
        for (int b = tid; b < n; b += kSpThreads) {
            cum_s[b] = a.cum[rb + b];
            lse_s[b] = a.logits ? __ldcg(a.row_lse + rb + b) : 0.f;
        }
    __syncthreads();
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
        const Cut cut = total > BW ? make_cut(hk, BW * m, BW, hist, red32, scan_w, sc, red_k) : Cut{0, 0, 0.f, 0, kNoKey};
        // survivors from the heads (one shared-memory atomic per warp); beams
        // whose whole head survived and that have more entries go on the
        // saturated list
        const unsigned lt = (1u << lane) - 1u;
        for (int i0 = 0; i0 < BW * m; i0 += kSpThreads) {
            const int i = i0 + tid;
            const uint64_t key = i < BW * m ? hk[i] : kNoKey;
            const bool keep = cut.keep(key);
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            int pos0 = 0;
            if (lane == 0 && bal) pos0 = atomicAdd(&cnts[0], __popc(bal));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            if (!keep) continue;
            const int pos = pos0 + __popc(bal & lt);
            if (pos < scap) {
                sk[pos] = key;
                se[pos] = he[i];
            }
            // (a beam whose best key beyond the head fails the cut has no
            // further survivors: its further keys are worse still)
            const int b = i >> mshift;
            if ((i & (m - 1)) == m - 1 && f.rl[b] > m && cut.keep(hnext[b])) sat[atomicAdd(&cnts[1], 1)] = b;
        }
        __syncthreads();
        const int n_sat = cnts[1];
        for (int q = warp; q < n_sat; q += kSpWarps) {   // their keys beyond the head (worse than its last)
            const int b = sat[q];
            const uint64_t last = hk[b * m + m - 1];
            const int e0 = max(f.rp[b], 0), e1 = (int)min((int64_t)f.rp[b] + f.rl[b], E);
            for (int j0 = e0; j0 < e1; j0 += 128) {   // four loads per lane in flight
                uint64_t kq[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = j0 + 32 * u + lane;
                    kq[u] = e < e1 ? __ldcg(keys + e) : kNoKey;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = j0 + 32 * u + lane;
                    const bool keep = kq[u] > last && cut.keep(kq[u]);
                    const unsigned bal = __ballot_sync(0xffffffffu, keep);
                    int pos0 = 0;
                    if (lane == 0 && bal) pos0 = atomicAdd(&cnts[0], __popc(bal));
                    pos0 = __shfl_sync(0xffffffffu, pos0, 0);
                    const int pos = pos0 + __popc(bal & lt);
                    if (keep && pos < scap) {
                        sk[pos] = kq[u];
                        se[pos] = e;
                    }
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
            const KeyCand cand{keys, cut, f.rp, f.rl, csr ? 0 : a.row_stride, n};
            radix_select(cand, E, want, hist, sc, prefix, mask);
            collect(cand, E, prefix, mask, BW, [](int64_t e) { return (int)e; }, f);
        }
    }
    __syncthreads();
    finish_request(a, r, ranked ? want : min(*f.cnt, want), f, ranked, dry);
}

// Phase 1: sp_parts CTAs per request of sp_rows (<= W) beams, one warp per
// beam, each with a ring of RING stages.
template <int W, int kMinBlocks, int RING, int KPC>
__global__ void __launch_bounds__(W * 32, kMinBlocks) select_rows_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t ring_bar[W][RING];
    const Dims dm = a.dims;
    const int C = a.sp_parts, R = a.sp_rows;
    const int r = blockIdx.x / C, part = blockIdx.x % C;
    const int warp = threadIdx.x / 32;
    const int64_t rb = (int64_t)r * dm.BW;
    const int b = part * R + warp;
    const bool has_row = warp < R && b < dm.BW;
    uint8_t *area = smem + (size_t)warp * ring_warp_bytes(RING);
    // the mask lookups (beam state and tables only) go before the wait when
    // the kernel before writes no beam state (the scores always follow it)
    RowPrep<KPC> p;
    auto prep = [&]() {
        const int n_live = min(max(a.n_live[r], 0), dm.BW);
        const int base = a.mask_kind == XGR_MASK_CSR ? a.row_ptr[rb] : 0;
        if (has_row) p = row_prep<RING, KPC>(a, r, b, n_live, base, area);
    };
    // The pick kernel (the only kernel launched after this one) may start at
    // once: before its own wait it touches no global memory, so this kernel
    // lets it in before its own wait, and the pick's warm-up overlaps phase 1.
    griddep_launch_dependents();
    if (a.prep_early) prep();
    griddep_wait();
    if (!a.prep_early) prep();
    if (has_row) row_run<RING, KPC>(a, r, b, p, a.keys + (int64_t)r * a.key_cap, area, ring_bar[warp]);
}

// Phase 2: one CTA per request.  It starts while the rows kernel runs (on the
// SMs that kernel leaves free) and first takes a dry pass of the whole pick
// over synthetic shared-memory data: the pick's code runs once per launch on
// whichever SM holds the CTA, and fetching it cold costs more than the pick
// itself, so the dry pass hides that behind phase 1.  Then it waits for the
// rows kernel and selects for real.
__global__ void __launch_bounds__(kSpThreads, 1) select_pick_kernel(const __grid_constant__ SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int hist[kRadixBins];
    __shared__ int scan_w[32];
    __shared__ int red_i[32];
    __shared__ uint32_t red32[64];
    __shared__ uint64_t red_k[32];
    __shared__ int sc[4];
    const int r = blockIdx.x;
    // Two passes through one inlined copy of the pick (a rolled loop, so the
    // dry pass fetches the very instructions the real one runs): the dry pass
    // before the wait, then the real one.
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        int n_live = 0;
        if (pass == 1) {
            griddep_wait();   // phase 1 of every request has completed
            n_live = min(max(a.n_live[r], 0), a.dims.BW);
        }
        select_request(a, r, n_live, smem, hist, scan_w, red_k, sc, red_i, red32, pass == 0);
        __syncthreads();   // the pass's shared memory is free again
    }
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

struct DenseShared {
    uint64_t bar;
    float red_f[kDnThreads / 32];
    int red_i[32];
    int scan_w[32];
    uint32_t red32[64];
    uint64_t red_k[32];
    int hist[kRadixBins];
    int sc[4];
    int cnts[1];
};

// One request's first step.  dry: a warm-up pass -- a synthetic score row,
// mask and root in shared memory through the same code, with no global
// memory access.
__device__ __forceinline__ void dense_select(const SelectArgs &a, uint8_t *smem, DenseShared &sh, bool dry) {
    float *red_f = sh.red_f;
    int *red_i = sh.red_i, *scan_w = sh.scan_w, *hist = sh.hist, *sc = sh.sc, *cnts = sh.cnts;
    uint32_t *red32 = sh.red32;
    uint64_t *red_k = sh.red_k;
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
    const uint32_t bar = smem_u32(&sh.bar);
    const bool bulk = !dry && (V & 3) == 0 && (reinterpret_cast<uintptr_t>(xg) & 15) == 0;
    const int n = dry ? 1 : min(max(a.n_live[r], 0), 1);
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
    const float cum = dry ? 0.f : a.cum[rb];
    // the mask with the tokens past V cleared; the valid-candidate count
    int c = 0;
    for (int w = tid; w < nw; w += kDnThreads) {
        const uint32_t v = (dry ? ~0u : a.bits[w]) & (32 * w + 32 <= V ? ~0u : (1u << (V & 31)) - 1u);
        bits[w] = v;
        c += __popc(v);
    }
    if (a.rewire) {
        if (!dry) stage_rows(a, rb, n, f);
        if (a.trie.root_bits) {
            // root children: bitset and exclusive prefix popcounts (trie order =
            // token order); thread t owns words [t*wpt, t*wpt + wpt)
            const int wpt = (nw + kDnThreads - 1) / kDnThreads;
            int cw = 0;
            for (int k = 0; k < wpt; ++k) {
                const int w = tid * wpt + k;
                if (w < nw) {
                    const uint32_t v = dry ? ~0u : a.trie.root_bits[w];
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
    if (dry) {
        for (int i = tid; i < V; i += kDnThreads) x[i] = -1e-3f * (float)(((uint32_t)i * 2654435761u) >> 16);
        if (a.rewire)
            for (int i = tid; i < dm.S; i += kDnThreads) {
                f.st_anc[i] = 0;
                f.st_seq[i] = 0;
            }
        if (tid == 0) f.st_node[0] = 0;
    } else if (!bulk && n > 0) {
        for (int i = tid; i < V; i += kDnThreads) x[i] = xg[i];
    }
    const int total = n > 0 ? block_sum_int(c, red_i) : 0;   // (+ a barrier)
    if (bulk && n > 0 && !mbar_wait(bar, 0, nullptr)) set_status(a.status, XGR_DEV_TIMEOUT);
    // the kernel after this one (the next step's attention) may start now: its
    // prologue prefetches the prompt K/V, and started any earlier that traffic
    // would queue ahead of this row's load
    if (!dry) griddep_launch_dependents();
    const int want = min(BW, total);
    float lse = 0.f;
    if (a.logits && want > 0) {
        // thread t folds tokens t + kDnThreads * u: the maximum over four
        // independent chains (NaN-propagating), then the sum of exponentials
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        for (int i = tid; i < V; i += 4 * kDnThreads) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = i + u * kDnThreads;
                if (t < V) mx[u] = max_nan(mx[u], x[t]);
            }
        }
        float mv = max_nan(max_nan(mx[0], mx[1]), max_nan(mx[2], mx[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mv = max_nan(mv, __shfl_xor_sync(0xffffffffu, mv, o));
        if (lane == 0) red_f[warp] = mv;
        __syncthreads();
        float M = red_f[0];
        for (int k = 1; k < kWarps; ++k) M = max_nan(M, red_f[k]);
        __syncthreads();   // red_f is read before it takes the sums
        float sv = 0.f;
        if (M != -INFINITY) {
            const float mk = M * kLog2e;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int i = tid; i < V; i += 4 * kDnThreads) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = i + u * kDnThreads;
                    if (t < V) acc[u] += ex2f(fmaf(x[t], kLog2e, -mk));
                }
            }
            sv = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        }
        sv = warp_sum_f(sv);
        if (lane == 0) red_f[warp] = sv;
        __syncthreads();
        float S = 0.f;
        for (int k = 0; k < kWarps; ++k) S += red_f[k];
        lse = M + logf(S);
        if (lse != lse && tid == 0) set_status(a.status, XGR_DEV_NAN);
    }
    DenseCand cand{x, bits, cum, lse, V, a.logits, a.status};
    uint64_t prefix = ~0ull, mask = 0;
    bool ranked = false;
    if (want > 0) {
        // each thread's best key: real candidates for the cut (four tokens in
        // flight per pass)
        uint64_t mn = kNoKey;
        for (int t0 = tid; t0 < V; t0 += 4 * kDnThreads) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = t0 + u * kDnThreads;
                uint64_t key = kNoKey;
                if (t < V && cand(t, key) && key < mn) mn = key;
            }
        }
        mins[tid] = mn;
        __syncthreads();
        const Cut cut = total > BW ? make_cut(mins, kDnThreads, BW, hist, red32, scan_w, sc, red_k)
                                   : Cut{0, 0, 0.f, 0, kNoKey};
        // survivors: every key the cut keeps, recomputed from the staged row --
        // each thread counts its own, one block scan places them, then each
        // thread writes its own (no atomics)
        // (the first kKeep of a thread's survivors wait in registers)
        constexpr int kKeep = 4;
        uint64_t kk[kKeep];
        int kt[kKeep];
        int mine = 0;
        for (int t0 = tid; t0 < V; t0 += 4 * kDnThreads) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = t0 + u * kDnThreads;
                uint64_t key;
                if (t < V && cand(t, key) && cut.keep(key)) {
#pragma unroll
                    for (int q = 0; q < kKeep; ++q)
                        if (q == mine) {
                            kk[q] = key;
                            kt[q] = t;
                        }
                    ++mine;
                }
            }
        }
        int ns;
        int pos = block_exclusive_scan_int(mine, scan_w, &ns);
        if (mine <= kKeep) {
#pragma unroll
            for (int q = 0; q < kKeep; ++q)
                if (q < mine && pos + q < scap) {
                    sk[pos + q] = kk[q];
                    se[pos + q] = kt[q];
                }
        } else {
            for (int t = tid; t < V; t += kDnThreads) {
                uint64_t key;
                if (!cand(t, key) || !cut.keep(key)) continue;
                if (pos < scap) {
                    sk[pos] = key;
                    se[pos] = t;
                }
                ++pos;
            }
        }
        __syncthreads();
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
    finish_request(a, r, ranked ? want : min(*f.cnt, want), f, ranked, dry);
}

// The first step's kernel: one CTA per request.  It starts while the kernel
// before it runs and takes a dry pass first (the code is cold on its SM),
// then waits for that kernel and selects.
__global__ void __launch_bounds__(kDnThreads) select_dense_kernel(const __grid_constant__ SelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ DenseShared sh;
    // a dry pass, then the real one, through one inlined copy (a rolled loop)
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) {
            griddep_wait();   // the scores and the beam state come from earlier kernels
        }
        dense_select(a, smem, sh, pass == 0);
        __syncthreads();   // the pass's shared memory is free again
    }
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

size_t select_scratch_bytes(int B, int BW, int64_t key_cap) {
    const size_t rows = (size_t)B * BW, m = (size_t)select_head_m(BW);
    return 4 * al256(rows * 4) + al256(rows * m * 8) + al256(rows * m * 4) + al256(rows * 8) +
           al256((size_t)B * key_cap * 8);
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
    a.head_next = reinterpret_cast<uint64_t *>(base);
    base += al256(rows * 8);
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
        return launch_pdl(select_dense_kernel, dim3(dm.B), dim3(kDnThreads), smem, s, a);
    }
    // sparse: the rows kernel (sp_parts CTAs per request of R beams, one per
    // warp), then the pick kernel (one CTA per request)
    // A NODE_BITS row's token list takes its warp's whole area once the row is
    // streamed, so a long row takes the wide shape's deeper ring.
    const int sms = a.num_sms > 0 ? a.num_sms : 148;
    const bool wide = (int64_t)dm.B * ((dm.BW + kRowWarpsWide - 1) / kRowWarpsWide) <= sms ||
                      (size_t)a.row_stride * 4 > ring_warp_bytes(kRingNarrow);
    const int R = std::min(dm.BW, wide ? kRowWarpsWide : kRowWarpsNarrow);
    a.sp_rows = R;
    a.sp_parts = (dm.BW + R - 1) / R;
    if (a.head_m < 1 || a.head_m > 16 || (a.head_m & (a.head_m - 1))) return cudaErrorInvalidValue;   // (m + 1 lanes merge)
    if (a.mask_kind != XGR_MASK_CSR && a.mask_kind != XGR_MASK_TRIE_ROWS && a.mask_kind != XGR_MASK_NODE_BITS)
        return cudaErrorInvalidValue;
    if (a.mask_kind != XGR_MASK_CSR && (int64_t)dm.BW * a.row_stride > a.key_cap) return cudaErrorInvalidValue;
    const int64_t grid = (int64_t)dm.B * a.sp_parts;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    const int ring = wide ? kRingWide : kRingNarrow;
    if (a.mask_kind == XGR_MASK_NODE_BITS && (size_t)a.row_stride * 4 > ring_warp_bytes(ring))
        return cudaErrorInvalidValue;
    const size_t rows_smem = (size_t)R * ring_warp_bytes(ring);
    const size_t pick_smem = sparse_pick_smem(dm, a.head_m);
    if (pick_smem > (220u << 10)) return cudaErrorInvalidValue;
    auto *rows_kernel = wide ? select_rows_kernel<kRowWarpsWide, 1, kRingWide, kSpKpcWide>
                             : select_rows_kernel<kRowWarpsNarrow, 3, kRingNarrow, kSpKpc>;
    cudaError_t e = ensure_smem(rows_kernel, rows_smem);
    if (e == cudaSuccess) e = ensure_smem(select_pick_kernel, pick_smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(rows_kernel, dim3((unsigned)grid), dim3((wide ? kRowWarpsWide : kRowWarpsNarrow) * 32), rows_smem,
                   s, a);
    if (e != cudaSuccess) return e;
    return launch_pdl(select_pick_kernel, dim3(dm.B), dim3(kSpThreads), pick_smem, s, a);
}

}  // namespace xgr

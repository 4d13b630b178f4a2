// beam.cu -- valid-path masks, beam top-K with early termination, and the
// in-place rewiring of the beam state.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"):
//  2.2 "Valid-path constraint": candidates come only from a pre-built
//      vocabulary of valid items (here a level-wise CSR trie).
//      "Hybrid dense/sparse storage": step 0 uses one pre-generated dense
//      bitset; later steps use sparse rows (the sorted children of each
//      beam's trie node).
//      "Early sort termination": each beam's candidates are ordered; a global
//      threshold (the page's min-heap minimum) cuts every beam's ordered list,
//      so only the few candidates above it are sorted.
//  2.1 "In-place updates": the beam state (ancestry slots, trie node, token
//      history, cumulative score) is rewritten in place; every row a new
//      beam reads is staged in shared memory before any row is written, so
//      no read sees a row already overwritten (no write-before-read hazard).
//
// Keys: a 64-bit integer whose ascending order is the rank order (higher
// fp32 score, then lower parent, then lower token), so every comparison is an
// exact integer comparison and ties are resolved identically everywhere.
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

// ------------------------------------------------------------------ begin

// Beam search starts from one live beam per request at the trie root with
// score 0.  Without a vocabulary (attention only) every beam is an
// independent live sequence whose Unshared token of step i sits at slot
// (i, b).
__global__ void begin_kernel(BeamState st, Dims dm, int Bcap, int all_live) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)Bcap * dm.BW) return;
    const int r = (int)(idx / dm.BW), b = (int)(idx % dm.BW);
    const bool live = all_live || b == 0;
    if (b == 0) st.n_live[r] = (r < dm.B) ? (all_live ? dm.BW : 1) : 0;
    st.cum[idx] = live ? 0.f : -INFINITY;
    st.node[idx] = live ? 0 : -1;
    for (int i = 0; i < dm.S; ++i) {
        st.anc[idx * dm.S + i] = all_live ? b : ((b == 0 && i == 0) ? 0 : -1);
        st.seq[idx * dm.S + i] = -1;
    }
}

// ------------------------------------------------------------------ masks

__device__ __forceinline__ int row_children(const MaskArgs &a, int64_t row) {
    const int r = (int)(row / a.dims.BW), b = (int)(row % a.dims.BW);
    if (b >= a.st.n_live[r]) return 0;
    const int node = a.st.node[row];
    if (node < 0 || node >= a.trie.n_nodes[a.step]) {
        set_status(a.st.status, XGR_DEV_INDEX);
        return 0;
    }
    return a.trie.ptr[a.step][node + 1] - a.trie.ptr[a.step][node];
}

constexpr int kScanThreads = 1024;

// One CTA: children count of every beam row, exclusive scan -> row_ptr.
__global__ void __launch_bounds__(kScanThreads) mask_scan_kernel(MaskArgs a) {
    __shared__ int64_t part[kScanThreads];
    const int64_t n_rows = (int64_t)a.dims.B * a.dims.BW;
    const int tid = threadIdx.x;
    const int64_t chunk = (n_rows + kScanThreads - 1) / kScanThreads;
    const int64_t lo = min(n_rows, tid * chunk), hi = min(n_rows, lo + chunk);
    int64_t sum = 0;
    for (int64_t row = lo; row < hi; ++row) sum += row_children(a, row);
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < kScanThreads; o <<= 1) {   // inclusive Hillis-Steele scan
        int64_t v = (tid >= o) ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int64_t off = part[tid] - sum;
    const int64_t total = part[kScanThreads - 1];
    for (int64_t row = lo; row < hi; ++row) {
        a.row_ptr[row] = (int32_t)min(off, a.cap);
        off += row_children(a, row);
    }
    if (tid == 0) {
        a.row_ptr[n_rows] = (int32_t)min(total, a.cap);
        if (total > a.cap) set_status(a.st.status, XGR_DEV_CAPACITY);
    }
}

// One warp per beam row: copy the node's sorted children into the CSR row.
__global__ void mask_fill_kernel(MaskArgs a) {
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    const int64_t n_rows = (int64_t)a.dims.B * a.dims.BW;
    if (row >= n_rows) return;
    const int beg = a.row_ptr[row], end = a.row_ptr[row + 1];
    if (end <= beg) return;
    const int node = a.st.node[row];
    const int32_t *src = a.trie.tok[a.step] + a.trie.ptr[a.step][node];
    for (int j = lane; j < end - beg; j += 32) a.cols[beg + j] = src[j];
}

// ------------------------------------------------------------------ sorting helpers

__device__ __forceinline__ int pow2_ceil(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Ascending bitonic sort of n (a power of two) keys in shared memory.
__device__ void block_sort(uint64_t *buf, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t x = buf[i], y = buf[ixj];
                    const bool up = (i & k) == 0;
                    if ((x > y) == up) {
                        buf[i] = y;
                        buf[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Exact block-wide radix select over E candidates given by `cand(e, key)`
// (returns false for a non-candidate).  Keys are unique.  On return exactly
// `want` candidates satisfy (key & mask) <= prefix (want <= number of
// candidates).  hist: 256 ints of shared memory; sc: 3 shared ints.
template <class Cand>
__device__ void radix_select(const Cand &cand, int64_t E, int want, int *hist, int *sc,
                             uint64_t &prefix, uint64_t &mask) {
    prefix = 0;
    mask = 0;
    int k_rem = want;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int64_t e = threadIdx.x; e < E; e += blockDim.x) {
            uint64_t key;
            if (cand(e, key) && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int acc = 0, d = 0;
            for (; d < 255; ++d) {
                if (acc + hist[d] >= k_rem) break;
                acc += hist[d];
            }
            sc[0] = d;
            sc[1] = hist[d] - (k_rem - acc);   // 0 <=> the whole bucket is taken
            sc[2] = k_rem - acc;
        }
        __syncthreads();
        const int d = sc[0], surplus = sc[1];
        k_rem = sc[2];
        prefix |= (uint64_t)d << shift;
        mask |= 0xFFull << shift;
        __syncthreads();
        if (surplus == 0) break;
    }
}

// ------------------------------------------------------------------ per-beam candidates

constexpr int kRowThreads = 256;
constexpr int kMaxK = 1024;

struct RowCand {
    const float *x;
    const uint32_t *bits;
    const int32_t *cols;
    int32_t *status;
    float cum, lse;
    int dense, logits, V, b;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        int t;
        if (dense) {
            t = (int)e;
            if (!((bits[t >> 5] >> (t & 31)) & 1u)) return false;
        } else {
            t = cols[e];
            if (t < 0 || t >= V) {
                set_status(status, XGR_DEV_MASK);
                return false;
            }
        }
        float lp = x[t];
        if (logits) lp = lp - lse;
        float k = cum + lp;   // one fp32 add: the score of (beam b, token t)
        if (isnan(k)) {
            set_status(status, XGR_DEV_NAN);
            return false;
        }
        if (k == 0.f) k = 0.f;   // -0.0 -> +0.0
        key = ((uint64_t)score_to_desc_bits(k) << 32) | (uint32_t)(b * V + t);
        return true;
    }
};

// One CTA per live beam row: (logits mode) the row's log-sum-exp over the
// whole vocabulary, then the beam's top-K valid candidates, sorted.
__global__ void __launch_bounds__(kRowThreads) select_row_kernel(SelectArgs a, int rows_per_req) {
    __shared__ uint64_t buf[kMaxK];
    __shared__ int hist[256];
    __shared__ int sc[4];
    __shared__ float red[kRowThreads / 32];
    const Dims dm = a.dims;
    const int r = blockIdx.x / rows_per_req, b = blockIdx.x % rows_per_req;
    const int64_t row = (int64_t)r * dm.BW + b;
    const int tid = threadIdx.x;
    if (b >= a.st.n_live[r]) {
        if (tid == 0) a.counts[row] = 0;
        return;
    }
    const float *x = a.scores + row * dm.V;
    const float cum = a.st.cum[row];

    float lse = 0.f;
    if (a.logits) {
        float mx = -INFINITY;
        int nan = 0;
        for (int t = tid; t < dm.V; t += kRowThreads) {
            const float v = x[t];
            nan |= isnan(v);
            mx = fmaxf(mx, v);
        }
        if (nan) set_status(a.st.status, XGR_DEV_NAN);
        mx = warp_max(mx);
        if (tid % 32 == 0) red[tid / 32] = mx;
        __syncthreads();
        mx = red[0];
        for (int w = 1; w < kRowThreads / 32; ++w) mx = fmaxf(mx, red[w]);
        __syncthreads();
        float sum = 0.f;
        for (int t = tid; t < dm.V; t += kRowThreads) sum += expf(x[t] - mx);
        sum = warp_sum(sum);
        if (tid % 32 == 0) red[tid / 32] = sum;
        __syncthreads();
        sum = 0.f;
        for (int w = 0; w < kRowThreads / 32; ++w) sum += red[w];
        lse = mx + logf(sum);
        if (tid == 0) a.row_lse[row] = lse;
    }

    RowCand cand;
    cand.x = x;
    cand.bits = a.bits;
    cand.status = a.st.status;
    cand.cum = cum;
    cand.lse = lse;
    cand.dense = a.dense;
    cand.logits = a.logits;
    cand.V = dm.V;
    cand.b = b;
    int64_t E;
    if (a.dense) {
        cand.cols = nullptr;
        E = dm.V;
    } else {
        const int beg = a.row_ptr[row];
        cand.cols = a.cols + beg;
        E = a.row_ptr[row + 1] - beg;
    }

    // number of valid candidates
    if (tid == 0) sc[3] = 0;
    __syncthreads();
    int mine = 0;
    for (int64_t e = tid; e < E; e += kRowThreads) {
        uint64_t key;
        mine += cand(e, key) ? 1 : 0;
    }
    atomicAdd(&sc[3], mine);
    __syncthreads();
    const int c = sc[3];
    __syncthreads();

    uint64_t prefix = ~0ull, mask = 0;
    if (c > dm.K) radix_select(cand, E, dm.K, hist, sc, prefix, mask);
    const int n_sel = min(c, dm.K);

    if (tid == 0) sc[3] = 0;
    __syncthreads();
    for (int64_t e = tid; e < E; e += kRowThreads) {
        uint64_t key;
        if (cand(e, key) && (key & mask) <= prefix) {
            const int pos = atomicAdd(&sc[3], 1);
            if (pos < kMaxK) buf[pos] = key;
        }
    }
    __syncthreads();
    const int P = pow2_ceil(max(n_sel, 1));
    for (int i = n_sel + tid; i < P; i += kRowThreads) buf[i] = kNoKey;
    __syncthreads();
    block_sort(buf, P);
    uint64_t *dst = a.lists + row * dm.K;
    for (int i = tid; i < n_sel; i += kRowThreads) dst[i] = buf[i];
    if (tid == 0) a.counts[row] = n_sel;
}

// ------------------------------------------------------------------ per-request select + rewire

constexpr int kReqThreads = 512;
constexpr int kSurvCap = 4096;

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

struct ListCand {   // the surviving prefixes of every beam's sorted list, flattened
    const uint64_t *lists;
    const int *off;   // [n+1] exclusive offsets of survivors per beam
    int n, K;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        int lo = 0, hi = n;   // beam b with off[b] <= e < off[b+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (off[mid] <= e) lo = mid; else hi = mid;
        }
        key = lists[(int64_t)lo * K + (e - off[lo])];
        return true;
    }
};

// dst[e] = the e-th entry of the concatenated heads of the beams' lists, the
// head of beam b being its first off[b+1]-off[b] entries.
__device__ void gather_flat(uint64_t *dst, const uint64_t *lists, const int *off, int n, int K,
                            int total) {
    const ListCand lc{lists, off, n, K};
    for (int e = threadIdx.x; e < total; e += blockDim.x) {
        uint64_t key;
        lc(e, key);
        dst[e] = key;
    }
}

__global__ void __launch_bounds__(kReqThreads) select_request_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const Dims dm = a.dims;
    const int BW = dm.BW, S = dm.S;
    const int sample_cap = pow2_ceil(2 * BW);
    uint64_t *sample = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *surv = sample + sample_cap;
    int *off = reinterpret_cast<int *>(surv + kSurvCap);     // [BW+1]
    int *cnt_s = off + (BW + 1);                              // [BW]
    int *st_anc = cnt_s + BW;                                 // [BW*S]
    int *st_seq = st_anc + BW * S;                            // [BW*S]
    int *st_node = st_seq + BW * S;                           // [BW]
    __shared__ int hist[256];
    __shared__ int sc[4];

    const int r = blockIdx.x;
    const int tid = threadIdx.x;
    const int n = a.st.n_live[r];
    const uint64_t *L = a.lists + (int64_t)r * BW * dm.K;
    const int32_t *cnt = a.counts + (int64_t)r * BW;

    for (int b = tid; b < BW; b += kReqThreads) cnt_s[b] = (b < n) ? cnt[b] : 0;
    __syncthreads();

    // exclusive scan helper over cnt-like values (serial on one warp; BW <= 1024)
    auto scan_into_off = [&](auto value_of) {
        if (tid < 32) {
            int carry = 0;
            for (int base = 0; base < BW; base += 32) {
                const int b = base + tid;
                int v = (b < BW) ? value_of(b) : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (tid >= o) incl += t;
                }
                if (b < BW) off[b] = carry + incl - v;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (tid == 0) off[BW] = carry;
        }
        __syncthreads();
    };

    // ---- total candidates, and a sample of the head of every beam's list
    scan_into_off([&](int b) { return cnt_s[b]; });
    const int total = off[BW];
    const int n_out = min(BW, total);
    __syncthreads();
    const int cs = n > 0 ? (BW + n - 1) / n : 0;
    scan_into_off([&](int b) { return min(cs, cnt_s[b]); });
    const int S0 = off[BW];
    gather_flat(sample, L, off, n, dm.K, S0);
    __syncthreads();
    uint64_t tau = kNoKey;
    if (S0 >= BW) {   // the BW-th best of the sample bounds the BW-th best overall
        const int P = pow2_ceil(S0);
        for (int i = S0 + tid; i < P; i += kReqThreads) sample[i] = kNoKey;
        __syncthreads();
        block_sort(sample, P);
        tau = sample[BW - 1];
    }
    __syncthreads();

    // ---- survivors: the prefix of each beam's sorted list at or above the threshold
    for (int b = tid; b < BW; b += kReqThreads) {
        int lo = 0, hi = cnt_s[b];
        const uint64_t *lb = L + (int64_t)b * dm.K;
        while (lo < hi) {   // upper bound of tau
            const int mid = (lo + hi) >> 1;
            if (lb[mid] <= tau) lo = mid + 1; else hi = mid;
        }
        st_node[b] = lo;    // temporarily: survivors of beam b
    }
    __syncthreads();
    scan_into_off([&](int b) { return st_node[b]; });
    const int T = off[BW];

    int n_sel;
    if (T <= kSurvCap) {
        gather_flat(surv, L, off, n, dm.K, T);
        n_sel = T;
    } else {   // rare: too many survivors -> exact radix select of the best BW
        ListCand lc{L, off, n, dm.K};
        uint64_t prefix, mask;
        radix_select(lc, T, n_out, hist, sc, prefix, mask);
        if (tid == 0) sc[3] = 0;
        __syncthreads();
        for (int64_t e = tid; e < T; e += kReqThreads) {
            uint64_t key;
            lc(e, key);
            if ((key & mask) <= prefix) {
                const int pos = atomicAdd(&sc[3], 1);
                if (pos < kSurvCap) surv[pos] = key;
            }
        }
        n_sel = n_out;
    }
    __syncthreads();
    {
        const int P = pow2_ceil(max(n_sel, 1));
        for (int i = n_sel + tid; i < P; i += kReqThreads) surv[i] = kNoKey;
        __syncthreads();
        block_sort(surv, P);
    }

    // ---- outputs in rank order
    for (int i = tid; i < BW; i += kReqThreads) {
        const int64_t o = (int64_t)r * BW + i;
        if (i < n_out) {
            const uint64_t key = surv[i];
            const uint32_t lo = (uint32_t)key;
            a.parent[o] = (int32_t)(lo / (uint32_t)dm.V);
            a.token[o] = (int32_t)(lo % (uint32_t)dm.V);
            a.cum_out[o] = desc_bits_to_score((uint32_t)(key >> 32));
        } else {
            a.parent[o] = -1;
            a.token[o] = -1;
            a.cum_out[o] = -INFINITY;
        }
    }
    if (tid == 0) a.n_out[r] = n_out;

    // ---- in-place rewiring: stage every old row first, then write
    const int64_t rb = (int64_t)r * BW;
    for (int i = tid; i < n * S; i += kReqThreads) {
        st_anc[i] = a.st.anc[rb * S + i];
        st_seq[i] = a.st.seq[rb * S + i];
    }
    for (int b = tid; b < n; b += kReqThreads) st_node[b] = a.st.node[rb + b];
    __syncthreads();
    const int s = a.step;
    for (int nb = tid; nb < BW; nb += kReqThreads) {
        const int64_t o = rb + nb;
        if (nb < n_out) {
            const uint64_t key = surv[nb];
            const uint32_t lo = (uint32_t)key;
            const int p = (int)(lo / (uint32_t)dm.V), t = (int)(lo % (uint32_t)dm.V);
            for (int i = 0; i < S; ++i) {
                int av = -1, sv = -1;
                if (i < s) {
                    av = st_anc[p * S + i];
                    sv = st_seq[p * S + i];
                } else if (i == s) {
                    av = p;        // the parent's own token of step s sits at slot (s, p)
                    sv = t;
                } else if (i == s + 1) {
                    av = nb;       // the new beam's token of step s+1 will sit at slot (s+1, nb)
                }
                a.st.anc[o * S + i] = av;
                a.st.seq[o * S + i] = sv;
            }
            const int child = find_child(a.trie, s, st_node[p], t);
            if (child < 0) set_status(a.st.status, XGR_DEV_MASK);
            a.st.node[o] = child;
            a.st.cum[o] = desc_bits_to_score((uint32_t)(key >> 32));
        } else {
            for (int i = 0; i < S; ++i) {
                a.st.anc[o * S + i] = -1;
                a.st.seq[o * S + i] = -1;
            }
            a.st.node[o] = -1;
            a.st.cum[o] = -INFINITY;
        }
    }
    __syncthreads();
    if (tid == 0) a.st.n_live[r] = n_out;
}

__global__ void get_sequences_kernel(BeamState st, Dims dm, int32_t *seq) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (int64_t)dm.B * dm.BW * dm.S) seq[i] = st.seq[i];
}

}  // namespace

size_t select_request_smem(const Dims &dm) {
    int sample_cap = 1;
    while (sample_cap < 2 * dm.BW) sample_cap <<= 1;
    return (size_t)(sample_cap + kSurvCap) * 8 + (size_t)(dm.BW + 1 + dm.BW) * 4 +
           (size_t)dm.BW * dm.S * 8 + (size_t)dm.BW * 4;
}

cudaError_t launch_begin(BeamState st, Dims dm, int Bcap, int all_live, cudaStream_t s) {
    const int64_t n = (int64_t)Bcap * dm.BW;
    begin_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(st, dm, Bcap, all_live);
    return cudaGetLastError();
}

cudaError_t launch_build_mask(const MaskArgs &a, cudaStream_t s) {
    mask_scan_kernel<<<1, kScanThreads, 0, s>>>(a);
    const int64_t rows = (int64_t)a.dims.B * a.dims.BW;
    mask_fill_kernel<<<(int)((rows * 32 + 255) / 256), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_beam_select(const SelectArgs &a, cudaStream_t s) {
    if (a.dims.K > kMaxK) return cudaErrorInvalidValue;
    const int rows_per_req = (a.step == 0) ? 1 : a.dims.BW;
    select_row_kernel<<<a.dims.B * rows_per_req, kRowThreads, 0, s>>>(a, rows_per_req);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = select_request_smem(a.dims);
    static size_t attr = 0;   // largest size set so far (set outside graph capture in practice)
    if (smem > attr) {
        e = cudaFuncSetAttribute(select_request_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        attr = smem;
    }
    select_request_kernel<<<a.dims.B, kReqThreads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_get_sequences(BeamState st, Dims dm, int32_t *seq, cudaStream_t s) {
    const int64_t n = (int64_t)dm.B * dm.BW * dm.S;
    if (n == 0) return cudaSuccess;
    get_sequences_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(st, dm, seq);
    return cudaGetLastError();
}

}  // namespace xgr

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

constexpr int kMaskThreads = 1024;

// block-wide exclusive scan of one value per thread (1024 threads); returns the
// exclusive prefix of this thread and writes the block total to *total
__device__ int64_t block_exclusive_scan(int64_t v, int64_t *warp_tot, int64_t *total) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int64_t w = warp_tot[lane];
        int64_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        warp_tot[lane] = wi - w;   // exclusive prefix of each warp
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    return warp_tot[warp] + incl - v;
}

// The CSR mask in two kernels.  mask_scan_kernel (one CTA): each thread owns a
// contiguous chunk of rows, loads their trie nodes and child ranges in
// independent batches, and a block scan turns the counts into row_ptr.
// mask_copy_kernel: one warp per row copies the node's sorted children.
__global__ void __launch_bounds__(kMaskThreads) mask_scan_kernel(MaskArgs a) {
    __shared__ int64_t warp_tot[32];
    __shared__ int64_t tot;
    const int64_t n_rows = (int64_t)a.dims.B * a.dims.BW;
    const int tid = threadIdx.x;
    const int64_t chunk = (n_rows + kMaskThreads - 1) / kMaskThreads;
    const int64_t lo = min(n_rows, (int64_t)tid * chunk), hi = min(n_rows, lo + chunk);
    constexpr int U = 8;
    int64_t sum = 0;
    for (int64_t r0 = lo; r0 < hi; r0 += U) {
        int c[U];
#pragma unroll
        for (int u = 0; u < U; ++u) c[u] = (r0 + u < hi) ? row_children(a, r0 + u) : 0;
#pragma unroll
        for (int u = 0; u < U; ++u) sum += c[u];
    }
    const int64_t ex = block_exclusive_scan(sum, warp_tot, &tot);
    int64_t off = ex;
    for (int64_t r0 = lo; r0 < hi; r0 += U) {
        int c[U];
#pragma unroll
        for (int u = 0; u < U; ++u) c[u] = (r0 + u < hi) ? row_children(a, r0 + u) : 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (r0 + u < hi) a.row_ptr[r0 + u] = (int32_t)min(off, a.cap);
            off += c[u];
        }
    }
    if (tid == 0) {
        a.row_ptr[n_rows] = (int32_t)min(tot, a.cap);
        if (tot > a.cap) set_status(a.st.status, XGR_DEV_CAPACITY);
    }
}

__global__ void mask_copy_kernel(MaskArgs a) {
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

// ------------------------------------------------------------------ selection
//
// Kernel 1 (row statistics): per live beam, the row log-sum-exp over the full
// vocabulary (logits mode; one online pass, 16-byte loads) and the beam's best
// kSampleK candidate keys.
// Kernel 2 (select): per request, tau = the BW-th best key of the beams'
// samples.  The samples are real candidates, so at least BW candidates rank at
// or above tau and the BW winners all do: one pass keeps the candidates at or
// above tau (usually a few hundred), sorts them and takes the first BW.  When
// the survivors overflow shared memory (or the sample is too small) an exact
// radix select over all candidates takes over.  With K >= BW the per-beam
// top-K cut never removes a winner, so the flat top-BW computed here equals
// the two-stage selection.

__device__ __forceinline__ void cswap(uint64_t &x, uint64_t &y) {
    const uint64_t lo = x < y ? x : y, hi = x < y ? y : x;
    x = lo;
    y = hi;
}

__device__ __forceinline__ void top4_insert(uint64_t (&t)[kSampleK], uint64_t key) {
    if (key >= t[3]) return;
    t[3] = key;
    cswap(t[2], t[3]);
    cswap(t[1], t[2]);
    cswap(t[0], t[1]);
}

// the 4 smallest keys of two ascending 4-lists, ascending (bitonic merge)
__device__ __forceinline__ void top4_merge(uint64_t (&t)[kSampleK], const uint64_t (&u)[kSampleK]) {
    uint64_t m0 = t[0] < u[3] ? t[0] : u[3], m1 = t[1] < u[2] ? t[1] : u[2];
    uint64_t m2 = t[2] < u[1] ? t[2] : u[1], m3 = t[3] < u[0] ? t[3] : u[0];
    cswap(m0, m2);
    cswap(m1, m3);
    cswap(m0, m1);
    cswap(m2, m3);
    t[0] = m0; t[1] = m1; t[2] = m2; t[3] = m3;
}

__device__ __forceinline__ void top4_warp(uint64_t (&t)[kSampleK]) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        uint64_t u[kSampleK];
#pragma unroll
        for (int i = 0; i < kSampleK; ++i) u[i] = __shfl_xor_sync(0xffffffffu, t[i], o);
        top4_merge(t, u);
    }
}

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// online (max, sum of 2^((x - max) log2 e)) of one value into (m, s)
__device__ __forceinline__ void lse_add(float &m, float &s, float v) {
    if (v > m) {
        s = s * ex2f((m - v) * kLog2e) + 1.f;
        m = v;
    } else if (v != -INFINITY) {
        s += ex2f((v - m) * kLog2e);
    }
}
__device__ __forceinline__ void lse_combine(float &m, float &s, float m2, float s2) {
    if (m2 > m) {
        s = s * ex2f((m - m2) * kLog2e) + s2;
        m = m2;
    } else if (m2 != -INFINITY) {
        s += s2 * ex2f((m2 - m) * kLog2e);
    }
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

constexpr int kStatThreads = 256;

// cta_per_row = 1 (dense first step): one CTA per request (its single live beam);
// otherwise one warp per beam row.
__global__ void __launch_bounds__(kStatThreads, 1) row_stats_kernel(SelectArgs a, int cta_per_row) {
    __shared__ float red_m[kStatThreads / 32], red_s[kStatThreads / 32];
    __shared__ uint64_t red_k[kStatThreads / 32][kSampleK];
    const Dims dm = a.dims;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int r, b, t0, stride;
    if (cta_per_row) {
        r = blockIdx.x;
        b = 0;
        t0 = threadIdx.x;
        stride = kStatThreads;
    } else {
        const int64_t gw = (int64_t)blockIdx.x * (kStatThreads / 32) + warp;
        if (gw >= (int64_t)dm.B * dm.BW) return;
        r = (int)(gw / dm.BW);
        b = (int)(gw % dm.BW);
        t0 = lane;
        stride = 32;
    }
    if (b >= a.n_live[r]) return;
    const int64_t row = (int64_t)r * dm.BW + b;
    const float *x = a.scores + row * dm.V;
    float lse = 0.f;
    if (a.logits) {
        float m = -INFINITY, s = 0.f;
        bool nan = false;
        if ((dm.V & 3) == 0) {
            // 16 independent 16-byte loads in flight per thread
            const float4 *x4 = reinterpret_cast<const float4 *>(x);
            const int n4 = dm.V / 4;
            constexpr int U = 16;
            for (int i0 = t0; i0 < n4; i0 += U * stride) {
                float4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + u * stride;
                    v[u] = i < n4 ? x4[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    nan |= isnan(v[u].x) | isnan(v[u].y) | isnan(v[u].z) | isnan(v[u].w);
                    const float cm = fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w));
                    if (cm > m) {
                        s *= ex2f((m - cm) * kLog2e);
                        m = cm;
                    }
                    if (cm != -INFINITY) {
                        s += ex2f((v[u].x - m) * kLog2e) + ex2f((v[u].y - m) * kLog2e) +
                             ex2f((v[u].z - m) * kLog2e) + ex2f((v[u].w - m) * kLog2e);
                    }
                }
            }
        } else {
            for (int i = t0; i < dm.V; i += stride) {
                nan |= isnan(x[i]);
                lse_add(m, s, x[i]);
            }
        }
        if (nan) set_status(a.status, XGR_DEV_NAN);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
            lse_combine(m, s, m2, s2);
        }
        if (cta_per_row) {
            if (lane == 0) {
                red_m[warp] = m;
                red_s[warp] = s;
            }
            __syncthreads();
            m = red_m[0];
            s = red_s[0];
            for (int w = 1; w < kStatThreads / 32; ++w) lse_combine(m, s, red_m[w], red_s[w]);
        }
        lse = m + logf(s);
    }
    const float cum = a.cum[row];
    uint64_t t[kSampleK] = {kNoKey, kNoKey, kNoKey, kNoKey};
    if (a.dense) {
        for (int tok = t0; tok < dm.V; tok += stride) {
            if (!((a.bits[tok >> 5] >> (tok & 31)) & 1u)) continue;
            float lp = x[tok];
            if (a.logits) lp -= lse;
            uint64_t key;
            if (make_key(cum, lp, b, tok, dm.V, a.status, key)) top4_insert(t, key);
        }
    } else {
        // batches of 8 entries per thread: the token and score loads overlap
        const int beg = a.row_ptr[row], end = a.row_ptr[row + 1];
        constexpr int U = 8;
        for (int e0 = beg + t0; e0 < end; e0 += U * stride) {
            int tk[U];
            float lv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int e = e0 + u * stride;
                tk[u] = e < end ? a.cols[e] : -1;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int e = e0 + u * stride;
                if (e < end && (tk[u] < 0 || tk[u] >= dm.V)) set_status(a.status, XGR_DEV_MASK);
                lv[u] = (tk[u] >= 0 && tk[u] < dm.V) ? x[tk[u]] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (tk[u] < 0 || tk[u] >= dm.V) continue;
                float lp = lv[u];
                if (a.logits) lp -= lse;
                uint64_t key;
                if (make_key(cum, lp, b, tk[u], dm.V, a.status, key)) top4_insert(t, key);
            }
        }
    }
    top4_warp(t);
    if (cta_per_row) {
        if (lane == 0)
            for (int i = 0; i < kSampleK; ++i) red_k[warp][i] = t[i];
        __syncthreads();
        if (warp == 0) {
            for (int i = 0; i < kSampleK; ++i) t[i] = lane < kStatThreads / 32 ? red_k[lane][i] : kNoKey;
            top4_warp(t);
        }
    }
    if ((cta_per_row ? threadIdx.x : lane) == 0) {
        for (int i = 0; i < kSampleK; ++i) a.sample[row * kSampleK + i] = t[i];
        a.row_lse[row] = lse;
    }
}

constexpr int kSelThreads = 1024;
constexpr int kSurvCap = 4096;   // survivors kept in shared memory
constexpr int kRankCap = 2048;   // sets up to this size are ordered by rank counting

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

// the candidates of one request as a flat index space: the dense first step
// enumerates tokens of beam 0; later steps enumerate the CSR entries of the
// live beams (rp = per-beam offsets relative to the request's first entry)
struct ReqCand {
    const float *x;          // scores of the request's first row
    const uint32_t *bits;
    const int32_t *cols;     // CSR entries of the request's first row
    const int *rp;           // [n+1] in shared memory
    const float *cum, *lse;  // [n] in shared memory
    int32_t *status;
    int n, dense, logits, V;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        int b, t;
        if (dense) {
            b = 0;
            t = (int)e;
            if (!((bits[t >> 5] >> (t & 31)) & 1u)) return false;
        } else {
            int lo = 0, hi = n;   // beam b with rp[b] <= e < rp[b+1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (rp[mid] <= e) lo = mid; else hi = mid;
            }
            b = lo;
            t = cols[e];
            if (t < 0 || t >= V) return false;
        }
        float lp = x[(int64_t)b * V + t];
        if (logits) lp -= lse[b];
        return make_key(cum[b], lp, b, t, V, status, key);
    }
};

// ascending bitonic sort of (key, payload) pairs, n a power of two
__device__ void block_sort_pairs(uint64_t *k, int *v, int n) {
    for (int kk = 2; kk <= n; kk <<= 1)
        for (int j = kk >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t x = k[i], y = k[ixj];
                    if ((x > y) == ((i & kk) == 0)) {
                        k[i] = y;
                        k[ixj] = x;
                        const int t = v[i];
                        v[i] = v[ixj];
                        v[ixj] = t;
                    }
                }
            }
            __syncthreads();
        }
}

size_t select_smem(const Dims &dm) {
    return (size_t)kSurvCap * 12 + (size_t)kSampleK * dm.BW * 8 + (size_t)(dm.BW + 1) * 4 +
           (size_t)dm.BW * 8 + (size_t)dm.BW * 12 + (size_t)dm.BW * dm.S * 8 + (size_t)dm.BW * 4 + 64;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const Dims dm = a.dims;
    const int BW = dm.BW, S = dm.S;
    uint64_t *surv = reinterpret_cast<uint64_t *>(smem_raw);    // [kSurvCap]
    uint64_t *samp = surv + kSurvCap;                           // [kSampleK*BW]
    uint64_t *win_k = samp + kSampleK * BW;                     // [BW]
    int *surv_e = reinterpret_cast<int *>(win_k + BW);          // [kSurvCap] entry of each survivor
    int *win_e = surv_e + kSurvCap;                             // [BW]
    int *rp = win_e + BW;                                       // [BW+1]
    float *cum_s = reinterpret_cast<float *>(rp + BW + 1);      // [BW]
    float *lse_s = cum_s + BW;                                  // [BW]
    int *st_anc = reinterpret_cast<int *>(lse_s + BW);          // [BW*S]
    int *st_seq = st_anc + BW * S;                              // [BW*S]
    int *st_node = st_seq + BW * S;                             // [BW]
    __shared__ int hist[256];
    __shared__ int sc[4];
    __shared__ int cnt;
    __shared__ unsigned long long tau_s;

    const int r = blockIdx.x, tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int64_t rb = (int64_t)r * BW;
    int n = a.n_live[r];
    if (a.dense) n = min(n, 1);   // the dense first step scores beam 0 only

    // ---- per-request tables in shared memory
    for (int b = tid; b < n; b += kSelThreads) {
        cum_s[b] = a.cum[rb + b];
        lse_s[b] = a.logits ? a.row_lse[rb + b] : 0.f;
    }
    int64_t base = 0;
    if (!a.dense) {
        base = a.row_ptr[rb];
        for (int b = tid; b <= n; b += kSelThreads) rp[b] = a.row_ptr[rb + b] - (int)base;
    }
    const int ns = n * kSampleK;
    for (int i = tid; i < ns; i += kSelThreads) samp[i] = a.sample[rb * kSampleK + i];
    if (tid == 0) {
        cnt = 0;
        tau_s = kNoKey;
    }
    __syncthreads();

    // ---- threshold: the sample key of rank BW-1 (keys are unique; padding is kNoKey)
    if (ns >= BW) {
        if (ns <= kRankCap) {
            for (int i = tid; i < ns; i += kSelThreads) {
                const uint64_t k = samp[i];
                if (k == kNoKey) continue;
                int rank = 0;
                for (int j = 0; j < ns; ++j) rank += samp[j] < k;
                if (rank == BW - 1) tau_s = k;
            }
        } else {
            int P = 1;
            while (P < ns) P <<= 1;
            // sort in the survivors buffer (P <= 4 * 1024 = kSurvCap)
            for (int i = tid; i < P; i += kSelThreads) surv[i] = i < ns ? samp[i] : kNoKey;
            __syncthreads();
            block_sort(surv, P);
            if (tid == 0) tau_s = surv[BW - 1];
        }
    }
    __syncthreads();
    const uint64_t tau = tau_s;
    const int64_t E = a.dense ? (n > 0 ? dm.V : 0) : rp[n];
    int total = 0;   // candidates of the request
    if (a.dense) {
        if (n > 0)
            for (int w = tid; w < (dm.V + 31) / 32; w += kSelThreads) total += __popc(a.bits[w]);
        atomicAdd(&cnt, total);
        __syncthreads();
        total = cnt;
        __syncthreads();
        if (tid == 0) cnt = 0;
        __syncthreads();
    } else {
        total = (int)E;
    }
    const int want = min(BW, total);
    const float *xr = a.scores + rb * dm.V;

    // ---- survivors: the candidates ranked at or above tau, with their entry index
    int T = kSurvCap + 1;
    if (tau != kNoKey || total <= kSurvCap) {
        if (a.dense) {
            for (int t = tid; t < (n > 0 ? dm.V : 0); t += kSelThreads) {
                if (!((a.bits[t >> 5] >> (t & 31)) & 1u)) continue;
                float lp = xr[t];
                if (a.logits) lp -= lse_s[0];
                uint64_t key;
                if (make_key(cum_s[0], lp, 0, t, dm.V, a.status, key) && key <= tau) {
                    const int pos = atomicAdd(&cnt, 1);
                    if (pos < kSurvCap) {
                        surv[pos] = key;
                        surv_e[pos] = t;
                    }
                }
            }
        } else {
            // one warp per beam; 4 entries per lane in flight
            const int32_t *cr = a.cols + base;
            for (int b = warp; b < n; b += kSelThreads / 32) {
                const int e_beg = rp[b], e_end = rp[b + 1];
                const float cb = cum_s[b], lb = lse_s[b];
                const float *xb = xr + (int64_t)b * dm.V;
                for (int e0 = e_beg + lane; e0 < e_end; e0 += 4 * 32) {
                    int tk[4];
                    float xv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = e0 + 32 * u;
                        tk[u] = e < e_end ? cr[e] : -1;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) xv[u] = (tk[u] >= 0 && tk[u] < dm.V) ? xb[tk[u]] : 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (tk[u] < 0 || tk[u] >= dm.V) continue;
                        float lp = xv[u];
                        if (a.logits) lp -= lb;
                        uint64_t key;
                        if (make_key(cb, lp, b, tk[u], dm.V, a.status, key) && key <= tau) {
                            const int pos = atomicAdd(&cnt, 1);
                            if (pos < kSurvCap) {
                                surv[pos] = key;
                                surv_e[pos] = e0 + 32 * u;
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();
        T = cnt;
        __syncthreads();
    }
    if (T > kSurvCap) {   // exact radix select of the best `want` over all candidates
        ReqCand cand;
        cand.x = xr;
        cand.bits = a.bits;
        cand.cols = a.dense ? nullptr : a.cols + base;
        cand.rp = rp;
        cand.cum = cum_s;
        cand.lse = lse_s;
        cand.status = a.status;
        cand.n = n;
        cand.dense = a.dense;
        cand.logits = a.logits;
        cand.V = dm.V;
        uint64_t prefix = ~0ull, mask = 0;
        if (want < total) radix_select(cand, E, want, hist, sc, prefix, mask);
        if (tid == 0) cnt = 0;
        __syncthreads();
        for (int64_t e = tid; e < E; e += kSelThreads) {
            uint64_t key;
            if (cand(e, key) && (key & mask) <= prefix) {
                const int pos = atomicAdd(&cnt, 1);
                if (pos < kSurvCap) {
                    surv[pos] = key;
                    surv_e[pos] = (int)e;
                }
            }
        }
        __syncthreads();
        T = min(cnt, kSurvCap);
        __syncthreads();
    }
    const int n_win = min(want, T);   // fewer only if some counted candidates were invalid

    // ---- the winners in rank order
    if (T <= kRankCap) {
        for (int i = tid; i < T; i += kSelThreads) {
            const uint64_t k = surv[i];
            int rank = 0;
            for (int j = 0; j < T; ++j) rank += surv[j] < k;
            if (rank < n_win) {
                win_k[rank] = k;
                win_e[rank] = surv_e[i];
            }
        }
    } else {
        int PT = 1;
        while (PT < T) PT <<= 1;
        for (int i = T + tid; i < PT; i += kSelThreads) {
            surv[i] = kNoKey;
            surv_e[i] = -1;
        }
        __syncthreads();
        block_sort_pairs(surv, surv_e, PT);
        for (int i = tid; i < n_win; i += kSelThreads) {
            win_k[i] = surv[i];
            win_e[i] = surv_e[i];
        }
    }
    __syncthreads();

    // ---- outputs in rank order
    for (int i = tid; i < BW; i += kSelThreads) {
        const int64_t o = rb + i;
        if (i < n_win) {
            const uint64_t key = win_k[i];
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
    if (tid == 0) a.n_out[r] = n_win;
    if (!a.rewire) return;

    // ---- in-place rewiring: stage every old row first, then write
    for (int i = tid; i < n * S; i += kSelThreads) {
        st_anc[i] = a.st.anc[rb * S + i];
        st_seq[i] = a.st.seq[rb * S + i];
    }
    for (int b = tid; b < n; b += kSelThreads) st_node[b] = a.st.node[rb + b];
    __syncthreads();
    const int s = a.step;
    for (int nb = tid; nb < BW; nb += kSelThreads) {
        const int64_t o = rb + nb;
        if (nb < n_win) {
            const uint64_t key = win_k[nb];
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
            // trie child: the mask row of parent p lists its children in trie
            // order, so the entry index locates the child directly
            int child = -1;
            const int node = st_node[p];
            if (a.dense) {
                child = find_child(a.trie, s, node, t);
            } else if (s < a.trie.levels && node >= 0 && node < a.trie.n_nodes[s]) {
                const int c = a.trie.ptr[s][node] + (win_e[nb] - rp[p]);
                if (c < a.trie.ptr[s][node + 1] && a.trie.tok[s][c] == t) child = c;
            }
            if (child < 0) set_status(a.status, XGR_DEV_MASK);
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
    if (tid == 0) a.st.n_live[r] = n_win;
}

__global__ void get_sequences_kernel(BeamState st, Dims dm, int32_t *seq) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (int64_t)dm.B * dm.BW * dm.S) seq[i] = st.seq[i];
}

}  // namespace

cudaError_t launch_begin(BeamState st, Dims dm, int Bcap, int all_live, cudaStream_t s) {
    const int64_t n = (int64_t)Bcap * dm.BW;
    begin_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(st, dm, Bcap, all_live);
    return cudaGetLastError();
}

cudaError_t launch_build_mask(const MaskArgs &a, cudaStream_t s) {
    const int64_t rows = (int64_t)a.dims.B * a.dims.BW;
    mask_scan_kernel<<<1, kMaskThreads, 0, s>>>(a);
    mask_copy_kernel<<<(int)((rows * 32 + 255) / 256), 256, 0, s>>>(a);
    return cudaGetLastError();
}

size_t select_sample_offset(int64_t rows) { return ((size_t)rows * 4 + 255) & ~(size_t)255; }
size_t select_scratch_bytes(int64_t rows) {
    return select_sample_offset(rows) + (size_t)rows * 8 * kSampleK;
}

cudaError_t launch_beam_select(const SelectArgs &a, cudaStream_t s) {
    if (a.dims.BW > 1024) return cudaErrorInvalidValue;
    if (a.dense) {
        row_stats_kernel<<<a.dims.B, kStatThreads, 0, s>>>(a, 1);
    } else {
        const int64_t rows = (int64_t)a.dims.B * a.dims.BW;
        const int per_cta = kStatThreads / 32;
        row_stats_kernel<<<(int)((rows + per_cta - 1) / per_cta), kStatThreads, 0, s>>>(a, 0);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = select_smem(a.dims);
    static size_t attr = 0;   // largest size set so far (set outside graph capture in practice)
    if (smem > attr) {
        e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        attr = smem;
    }
    select_kernel<<<a.dims.B, kSelThreads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_get_sequences(BeamState st, Dims dm, int32_t *seq, cudaStream_t s) {
    const int64_t n = (int64_t)dm.B * dm.BW * dm.S;
    if (n == 0) return cudaSuccess;
    get_sequences_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(st, dm, seq);
    return cudaGetLastError();
}

}  // namespace xgr

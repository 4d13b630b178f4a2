// select_noalloc.cu -- masked beam top-K for callers that cannot allocate
// device memory (xgr_beam_topk_noalloc in include/xgr.h).
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// that runs inside another framework's memory pool with no allocator hook,
// plugins whose host process forbids device allocation after start-up, or
// callers that must not add a workspace of their own.  This entry point
// computes exactly what xgr_beam_select writes to its outputs (same keys,
// same order, same tie-break), but without a context and without touching any
// beam state: the caller passes the scores, the cumulative scores, the live
// beam counts and the mask, and gets parent / token / cum / n_out back.
//
// Its scratch (each beam's sorted top-K list, the per-beam counts and the row
// log-sum-exp) lives in one file-scope device array of kScratchBytes; every
// GPU that loads the library holds that array until the process exits.  All
// calls share it, so calls that overlap on the GPU (two streams, two threads)
// race on it and must be serialised by the caller.  The array keeps the last
// call's contents; everything a call reads from it is written by that same
// call first.  Device faults (NaN scores, out-of-vocabulary mask tokens) are
// skipped as in the context path but not reported -- use the context path
// (xgr_device_status) to diagnose them.
#include <mutex>

#include "common.cuh"

namespace xgr {

namespace {

constexpr size_t kScratchBytes = 8u << 20;   // 8 MiB: lists + counts + row LSE
constexpr int kMaxDevices = 64;
constexpr int kNaRowThreads = 256;
constexpr int kNaReqThreads = 512;
constexpr int kNaMaxK = 1024;
constexpr int kNaSurvCap = 4096;

static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

struct NaArgs {
    int B, BW, K, V, step_dense, logits;
    const float *scores, *cum;
    const int32_t *n_live;
    const uint32_t *bits;
    const int32_t *row_ptr, *cols;
    int32_t *parent, *token, *n_out;
    float *cum_out;
    uint64_t *lists;   // scratch: [B][BW][K]
    int32_t *counts;   // scratch: [B][BW]
    float *row_lse;    // scratch: [B][BW]
};

__device__ __forceinline__ int na_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

__device__ void na_sort(uint64_t *buf, int n) {   // ascending bitonic sort, n a power of two
    for (int k = 2; k <= n; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t x = buf[i], y = buf[ixj];
                    if ((x > y) == ((i & k) == 0)) {
                        buf[i] = y;
                        buf[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
}

// exact radix select: afterwards exactly `want` candidates satisfy (key & mask) <= prefix
template <class Cand>
__device__ void na_select(const Cand &cand, int64_t E, int want, int *hist, int *sc,
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
            sc[1] = hist[d] - (k_rem - acc);
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

struct NaRowCand {
    const float *x;
    const uint32_t *bits;
    const int32_t *cols;
    float cum, lse;
    int dense, logits, V, b;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        int t;
        if (dense) {
            t = (int)e;
            if (!((bits[t >> 5] >> (t & 31)) & 1u)) return false;
        } else {
            t = cols[e];
            if (t < 0 || t >= V) return false;
        }
        float lp = x[t];
        if (logits) lp = lp - lse;
        float k = cum + lp;
        if (isnan(k)) return false;
        if (k == 0.f) k = 0.f;
        key = ((uint64_t)score_to_desc_bits(k) << 32) | (uint32_t)(b * V + t);
        return true;
    }
};

__global__ void __launch_bounds__(kNaRowThreads) na_row_kernel(NaArgs a, int rows_per_req) {
    __shared__ uint64_t buf[kNaMaxK];
    __shared__ int hist[256];
    __shared__ int sc[4];
    __shared__ float red[kNaRowThreads / 32];
    const int r = blockIdx.x / rows_per_req, b = blockIdx.x % rows_per_req;
    const int64_t row = (int64_t)r * a.BW + b;
    const int tid = threadIdx.x;
    if (b >= a.n_live[r]) {
        if (tid == 0) a.counts[row] = 0;
        return;
    }
    const float *x = a.scores + row * a.V;
    float lse = 0.f;
    if (a.logits) {
        float mx = -INFINITY;
        for (int t = tid; t < a.V; t += kNaRowThreads) mx = fmaxf(mx, x[t]);
        mx = warp_max(mx);
        if (tid % 32 == 0) red[tid / 32] = mx;
        __syncthreads();
        mx = red[0];
        for (int w = 1; w < kNaRowThreads / 32; ++w) mx = fmaxf(mx, red[w]);
        __syncthreads();
        float sum = 0.f;
        for (int t = tid; t < a.V; t += kNaRowThreads) sum += expf(x[t] - mx);
        sum = warp_sum(sum);
        if (tid % 32 == 0) red[tid / 32] = sum;
        __syncthreads();
        sum = 0.f;
        for (int w = 0; w < kNaRowThreads / 32; ++w) sum += red[w];
        lse = mx + logf(sum);
        if (tid == 0) a.row_lse[row] = lse;
    }
    NaRowCand cand{x, a.bits, nullptr, a.cum[row], lse, a.step_dense, a.logits, a.V, b};
    int64_t E = a.V;
    if (!a.step_dense) {
        const int beg = a.row_ptr[row];
        cand.cols = a.cols + beg;
        E = a.row_ptr[row + 1] - beg;
    }
    if (tid == 0) sc[3] = 0;
    __syncthreads();
    int mine = 0;
    for (int64_t e = tid; e < E; e += kNaRowThreads) {
        uint64_t key;
        mine += cand(e, key) ? 1 : 0;
    }
    atomicAdd(&sc[3], mine);
    __syncthreads();
    const int c = sc[3];
    __syncthreads();
    uint64_t prefix = ~0ull, mask = 0;
    if (c > a.K) na_select(cand, E, a.K, hist, sc, prefix, mask);
    const int n_sel = min(c, a.K);
    if (tid == 0) sc[3] = 0;
    __syncthreads();
    for (int64_t e = tid; e < E; e += kNaRowThreads) {
        uint64_t key;
        if (cand(e, key) && (key & mask) <= prefix) {
            const int pos = atomicAdd(&sc[3], 1);
            if (pos < kNaMaxK) buf[pos] = key;
        }
    }
    __syncthreads();
    const int P = na_pow2(max(n_sel, 1));
    for (int i = n_sel + tid; i < P; i += kNaRowThreads) buf[i] = kNoKey;
    __syncthreads();
    na_sort(buf, P);
    for (int i = tid; i < n_sel; i += kNaRowThreads) a.lists[row * a.K + i] = buf[i];
    if (tid == 0) a.counts[row] = n_sel;
}

struct NaListCand {
    const uint64_t *lists;
    const int *off;
    int n, K;
    __device__ bool operator()(int64_t e, uint64_t &key) const {
        int lo = 0, hi = n;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (off[mid] <= e) lo = mid; else hi = mid;
        }
        key = lists[(int64_t)lo * K + (e - off[lo])];
        return true;
    }
};

__global__ void __launch_bounds__(kNaReqThreads) na_request_kernel(NaArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int BW = a.BW;
    const int sample_cap = na_pow2(2 * BW);
    uint64_t *sample = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *surv = sample + sample_cap;
    int *off = reinterpret_cast<int *>(surv + kNaSurvCap);   // [BW+1]
    int *cnt_s = off + (BW + 1);                               // [BW]
    int *tmp = cnt_s + BW;                                     // [BW]
    __shared__ int hist[256];
    __shared__ int sc[4];
    const int r = blockIdx.x, tid = threadIdx.x;
    // with the dense first-step mask only beam 0 was scored by the row kernel
    const int n = a.step_dense ? min(a.n_live[r], 1) : a.n_live[r];
    const uint64_t *L = a.lists + (int64_t)r * BW * a.K;
    for (int b = tid; b < BW; b += kNaReqThreads) cnt_s[b] = (b < n) ? a.counts[(int64_t)r * BW + b] : 0;
    __syncthreads();
    auto scan = [&](auto value_of) {   // exclusive scan into off[0..BW]
        if (tid < 32) {
            int carry = 0;
            for (int base = 0; base < BW; base += 32) {
                const int b = base + tid;
                const int v = (b < BW) ? value_of(b) : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (tid >= o) incl += t;
                }
                if (b < BW) off[b] = carry + incl - v;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (tid == 0) off[BW] = carry;
        }
        __syncthreads();
    };
    auto gather = [&](uint64_t *dst, int total) {
        const NaListCand lc{L, off, n, a.K};
        for (int e = tid; e < total; e += kNaReqThreads) {
            uint64_t key;
            lc(e, key);
            dst[e] = key;
        }
    };
    scan([&](int b) { return cnt_s[b]; });
    const int total = off[BW];
    const int n_out = min(BW, total);
    __syncthreads();
    const int cs = n > 0 ? (BW + n - 1) / n : 0;
    scan([&](int b) { return min(cs, cnt_s[b]); });
    const int S0 = off[BW];
    gather(sample, S0);
    __syncthreads();
    uint64_t tau = kNoKey;
    if (S0 >= BW) {
        const int P = na_pow2(S0);
        for (int i = S0 + tid; i < P; i += kNaReqThreads) sample[i] = kNoKey;
        __syncthreads();
        na_sort(sample, P);
        tau = sample[BW - 1];
    }
    __syncthreads();
    for (int b = tid; b < BW; b += kNaReqThreads) {
        int lo = 0, hi = cnt_s[b];
        const uint64_t *lb = L + (int64_t)b * a.K;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (lb[mid] <= tau) lo = mid + 1; else hi = mid;
        }
        tmp[b] = lo;
    }
    __syncthreads();
    scan([&](int b) { return tmp[b]; });
    const int T = off[BW];
    int n_sel;
    if (T <= kNaSurvCap) {
        gather(surv, T);
        n_sel = T;
    } else {
        const NaListCand lc{L, off, n, a.K};
        uint64_t prefix, mask;
        na_select(lc, T, n_out, hist, sc, prefix, mask);
        if (tid == 0) sc[3] = 0;
        __syncthreads();
        for (int64_t e = tid; e < T; e += kNaReqThreads) {
            uint64_t key;
            lc(e, key);
            if ((key & mask) <= prefix) {
                const int pos = atomicAdd(&sc[3], 1);
                if (pos < kNaSurvCap) surv[pos] = key;
            }
        }
        n_sel = n_out;
    }
    __syncthreads();
    const int P = na_pow2(max(n_sel, 1));
    for (int i = n_sel + tid; i < P; i += kNaReqThreads) surv[i] = kNoKey;
    __syncthreads();
    na_sort(surv, P);
    for (int i = tid; i < BW; i += kNaReqThreads) {
        const int64_t o = (int64_t)r * BW + i;
        if (i < n_out) {
            const uint64_t key = surv[i];
            const uint32_t lo = (uint32_t)key;
            a.parent[o] = (int32_t)(lo / (uint32_t)a.V);
            a.token[o] = (int32_t)(lo % (uint32_t)a.V);
            a.cum_out[o] = desc_bits_to_score((uint32_t)(key >> 32));
        } else {
            a.parent[o] = -1;
            a.token[o] = -1;
            a.cum_out[o] = -INFINITY;
        }
    }
    if (tid == 0) a.n_out[r] = n_out;
}

size_t na_request_smem(int BW) {
    int sample_cap = 1;
    while (sample_cap < 2 * BW) sample_cap <<= 1;
    return (size_t)(sample_cap + kNaSurvCap) * 8 + (size_t)(3 * BW + 1) * 4;
}

// Device address of the scratch array, looked up once per device (with that
// device current) and cached; host code must never pass g_scratch itself.
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

cudaError_t scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(na_request_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)na_request_smem(1024));
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool al16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

}  // namespace xgr

extern "C" xgr_status xgr_beam_topk_noalloc(int32_t n_requests, int32_t beam_width, int32_t top_k,
                                            int32_t vocab, const float *d_scores, int32_t flags,
                                            const float *d_cum, const int32_t *d_n_live,
                                            const uint32_t *d_bits, const int32_t *d_row_ptr,
                                            const int32_t *d_cols, int32_t *d_parent,
                                            int32_t *d_token, float *d_cum_out, int32_t *d_n_out,
                                            xgr_stream_t stream) {
    using namespace xgr;
    if (flags != XGR_SCORES_LOGPROB && flags != XGR_SCORES_LOGITS) return XGR_ERR_ARG;
    if (!al16(d_scores) || !al16(d_cum) || !al16(d_n_live) || !al16(d_parent) || !al16(d_token) ||
        !al16(d_cum_out) || !al16(d_n_out))
        return XGR_ERR_ARG;
    const bool dense = d_bits != nullptr;
    if (!dense && (!al16(d_row_ptr) || !al16(d_cols))) return XGR_ERR_ARG;
    if (n_requests < 1 || beam_width < 1 || beam_width > 1024 || top_k < beam_width ||
        top_k > kNaMaxK || vocab < 1 || (int64_t)beam_width * vocab >= (1ll << 32))
        return XGR_ERR_SHAPE;
    const int64_t rows = (int64_t)n_requests * beam_width;
    const size_t lists_bytes = (size_t)rows * top_k * 8;
    const size_t need = lists_bytes + (size_t)rows * 8;
    if (need > kScratchBytes) return XGR_ERR_CAPACITY;   // beyond the fixed 8 MiB scratch
    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return XGR_ERR_CUDA;
    NaArgs a;
    a.B = n_requests;
    a.BW = beam_width;
    a.K = top_k;
    a.V = vocab;
    a.step_dense = dense;
    a.logits = flags == XGR_SCORES_LOGITS;
    a.scores = d_scores;
    a.cum = d_cum;
    a.n_live = d_n_live;
    a.bits = d_bits;
    a.row_ptr = d_row_ptr;
    a.cols = d_cols;
    a.parent = d_parent;
    a.token = d_token;
    a.cum_out = d_cum_out;
    a.n_out = d_n_out;
    a.lists = static_cast<uint64_t *>(scratch);
    a.counts = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(scratch) + lists_bytes);
    a.row_lse = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + lists_bytes + rows * 4);
    const cudaStream_t s = (cudaStream_t)stream;
    // dense mask: only beam 0 of each request can be live (the first step)
    const int rows_per_req = dense ? 1 : beam_width;
    na_row_kernel<<<n_requests * rows_per_req, kNaRowThreads, 0, s>>>(a, rows_per_req);
    if (cudaGetLastError() != cudaSuccess) return XGR_ERR_CUDA;
    na_request_kernel<<<n_requests, kNaReqThreads, na_request_smem(beam_width), s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return XGR_ERR_CUDA;
    return XGR_OK;
}

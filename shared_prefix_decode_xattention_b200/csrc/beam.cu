// beam.cu -- beam-state start, valid-path masks, and the sequences read-out.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"):
//  2.2 "Valid-path constraint": candidates come only from a pre-built
//      vocabulary of valid items (here a level-wise CSR trie).
//      "Hybrid dense/sparse storage": step 0 uses one pre-generated dense
//      bitset; later steps use sparse rows (the sorted children of each
//      beam's trie node).  The selection itself is in select.cu.
#include <algorithm>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

// ------------------------------------------------------------------ begin

// Beam search starts from one live beam per request at the trie root with
// score 0.  Without a vocabulary (attention only) every beam is an
// independent live sequence whose Unshared token of step i sits at slot
// (i, b).
__global__ void begin_kernel(BeamState st, Dims dm, int Bcap, int all_live, uint64_t *mask_sync) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (mask_sync && idx <= Bcap) mask_sync[idx] = 0;   // mask look-back words and ticket
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

constexpr int kMaskThreads = 1024;
constexpr int kMaskRows = 1024 / kMaskThreads;   // rows per thread (BW <= 1024)

// block-wide exclusive scan of one value per thread; returns the exclusive
// prefix of this thread and writes the block total to *total
__device__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < nw) warp_tot[lane] = wi - w;   // exclusive prefix of each warp
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    const int ex = warp_tot[warp] + incl - v;
    __syncthreads();
    return ex;
}

// The CSR mask of one step in one kernel: parts x B CTAs.  Every CTA of
// request r reads the trie nodes of the request's live beams and their child
// ranges, and scans the counts into the request's local row offsets.  Part 0
// publishes the request's total; every part then adds up the totals of the
// requests before r (each read once, all in parallel: a look-back over
// published values whose waits are bounded), part 0 writes the request's
// row_ptr, and each part copies its share of the request's children (the
// sorted child tokens of each node, contiguous in the trie level).  The last
// CTA to finish clears the published totals for the next call.
__global__ void __launch_bounds__(kMaskThreads) mask_kernel(MaskArgs a) {
    __shared__ int off_s[1024 + 1];   // local offset of each row of the request; [BW] = total
    __shared__ int src_s[1024];       // first child of each row in the trie level
    __shared__ int warp_tot[32];
    __shared__ int total_s;
    __shared__ long long pre_w[32];
    __shared__ int last;
    __shared__ int order;
    const Dims dm = a.dims;
    const int BW = dm.BW, s = a.step;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    // logical (part, request) in the order the CTAs started: a CTA only waits for
    // requests whose part 0 took its number earlier, so is already running
    if (tid == 0) order = (int)atomicAdd(a.ticket + 1, 1u);
    __syncthreads();
    const int parts = gridDim.x, part = order % parts, r = order / parts;
    const int64_t rb = (int64_t)r * BW;
    // the trie nodes (all loads independent of n_live), then the child ranges
    const int n = a.st.n_live[r];
    int node[kMaskRows];
#pragma unroll
    for (int i = 0; i < kMaskRows; ++i) {
        const int b = tid * kMaskRows + i;
        node[i] = b < BW ? a.st.node[rb + b] : -1;
    }
    int cnt[kMaskRows], src[kMaskRows], sum = 0;
#pragma unroll
    for (int i = 0; i < kMaskRows; ++i) {
        const int b = tid * kMaskRows + i;
        cnt[i] = 0;
        src[i] = 0;
        if (b >= BW || b >= n) continue;
        if (node[i] < 0 || node[i] >= a.trie.n_nodes[s]) {
            if (part == 0) set_status(a.st.status, XGR_DEV_INDEX);
            continue;
        }
        src[i] = a.trie.ptr[s][node[i]];
        cnt[i] = a.trie.ptr[s][node[i] + 1] - src[i];
        sum += cnt[i];
    }
    int off = block_exclusive_scan(sum, warp_tot, &total_s);
    const int total = total_s;
#pragma unroll
    for (int i = 0; i < kMaskRows; ++i) {
        const int b = tid * kMaskRows + i;
        if (b < BW) {
            off_s[b] = off;
            src_s[b] = src[i];
        }
        off += cnt[i];
    }
    if (tid == 0) {
        off_s[BW] = total;
        if (part == 0)   // publish the request's total (bit 32: present)
            atomicExch(reinterpret_cast<unsigned long long *>(a.flags + r),
                       (1ull << 32) | (uint32_t)total);
    }
    // entries before this request: the published totals of requests 0..r-1
    long long pre = 0;
    for (int r2 = tid; r2 < r; r2 += kMaskThreads) {
        uint64_t f = 0;
        for (uint32_t it = 0; it < kSpinLimit; ++it) {
            f = *reinterpret_cast<volatile uint64_t *>(a.flags + r2);
            if (f >> 32) break;
        }
        if (!(f >> 32)) set_status(a.st.status, XGR_DEV_TIMEOUT);
        pre += (uint32_t)f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, o);
    if (lane == 0) pre_w[warp] = pre;
    __syncthreads();
    pre = 0;
    for (int w = 0; w < kMaskThreads / 32; ++w) pre += pre_w[w];
    if (part == 0) {
#pragma unroll
        for (int i = 0; i < kMaskRows; ++i) {
            const int b = tid * kMaskRows + i;
            if (b < BW) a.row_ptr[rb + b] = (int32_t)min(pre + off_s[b], (long long)a.cap);
        }
        if (tid == 0 && r == dm.B - 1) {
            a.row_ptr[(int64_t)dm.B * BW] = (int32_t)min(pre + total, (long long)a.cap);
            if (pre + total > a.cap) set_status(a.st.status, XGR_DEV_CAPACITY);
        }
    }
    // copy: this part's share of the request's entries; entry e belongs to the
    // row b with off_s[b] <= e < off_s[b+1] (binary search, 8 entries in flight)
    const int per = (total + parts - 1) / parts;
    const int lo = part * per, hi = min(total, lo + per);
    const int32_t *tok = a.trie.tok[s];
    constexpr int U = 8;
    for (int e0 = lo + tid; e0 < hi; e0 += U * kMaskThreads) {
        int v[U];
        long long g[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * kMaskThreads;
            g[u] = -1;
            if (e >= hi) continue;
            int l = 0, h = BW;   // largest b with off_s[b] <= e
            while (h - l > 1) {
                const int m = (l + h) >> 1;
                if (off_s[m] <= e) l = m; else h = m;
            }
            g[u] = pre + e;
            v[u] = tok[src_s[l] + (e - off_s[l])];
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (g[u] >= 0 && g[u] < a.cap) a.cols[g[u]] = v[u];
    }
    // the last CTA clears the published totals for the next call
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        last = atomicAdd(a.ticket, 1u) == (unsigned)(parts * dm.B - 1);
    }
    __syncthreads();
    if (last) {
        for (int r2 = tid; r2 < dm.B; r2 += kMaskThreads) a.flags[r2] = 0;
        if (tid == 0) {
            a.ticket[0] = 0;
            a.ticket[1] = 0;
        }
    }
}

__global__ void get_sequences_kernel(BeamState st, Dims dm, int32_t *seq) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (int64_t)dm.B * dm.BW * dm.S) seq[i] = st.seq[i];
}

}  // namespace

cudaError_t launch_begin(BeamState st, Dims dm, int Bcap, int all_live, uint64_t *mask_sync,
                         cudaStream_t s) {
    const int64_t n = (int64_t)Bcap * dm.BW + 1;
    begin_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(st, dm, Bcap, all_live, mask_sync);
    return cudaGetLastError();
}

cudaError_t launch_build_mask(const MaskArgs &a, int parts, cudaStream_t s) {
    if (a.dims.BW > 1024 || a.dims.B < 1) return cudaErrorInvalidValue;
    mask_kernel<<<dim3(std::max(1, parts), a.dims.B), kMaskThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_get_sequences(BeamState st, Dims dm, int32_t *seq, cudaStream_t s) {
    const int64_t n = (int64_t)dm.B * dm.BW * dm.S;
    if (n == 0) return cudaSuccess;
    get_sequences_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(st, dm, seq);
    return cudaGetLastError();
}

}  // namespace xgr

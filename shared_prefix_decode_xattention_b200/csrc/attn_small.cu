// attn_small.cu -- Shared-stage partial attention for work items with few
// query rows (<= 16): step 0 (one live beam per request), the private suffix
// of a prefix-group request, tiny head counts.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"),
// 2.1 "Staged computation": the Shared stage produces, for each query row,
// local scores over a range of prompt keys together with their max and
// sum-of-exponentials; the Merging stage combines such partials.  Here one
// CTA handles one work item (a kv head, <= 16 rows, a key range) and writes
// one partial (O unnormalised, m, l) per row.  The rows are few, so the kernel
// is bound by streaming K/V from HBM; keys are staged through shared memory
// by 16-byte cp.async copies (a whole tile in flight), 128 keys per tile.
#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr int kThreads = 128;
constexpr int kTileKeys = 128;

template <int D>
struct SmallSmem {
    static constexpr int kRow = D + 8;                 // bf16 per staged row (16 B pad)
    __nv_bfloat16 k[kTileKeys * kRow];
    __nv_bfloat16 v[kTileKeys * kRow];
    float q[kSmallRows * D];
    float p[kSmallRows * kTileKeys];
    float m[kSmallRows], l[kSmallRows], alpha[kSmallRows];
    int64_t gid[kSmallRows];
    int live[kSmallRows];
};

template <int D>
__global__ void __launch_bounds__(kThreads) attn_small_kernel(SmallArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    SmallSmem<D> &sm = *reinterpret_cast<SmallSmem<D> *>(smem_raw);
    constexpr int kRow = SmallSmem<D>::kRow;
    constexpr int kRowGroups = kThreads / D;           // threads per dim
    constexpr int kRowsPerThread = kSmallRows / kRowGroups;

    const WorkItem it = a.items[blockIdx.x];   // (the plan is written before any decode kernel)
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x;
    const Dims dm = a.dims;
    const int G = dm.G;
    const int n_rows = it.n_rows;
    const float scale_log2 = kLog2e * rsqrtf((float)D);

    // ---- query rows of this item
    if (tid < kSmallRows) {
        int live = 0;
        int64_t gid = -1;
        if (tid < n_rows) {
            const int i = it.row_begin + tid;
            const int member = i / (a.nb * G);
            const int b = (i / G) % a.nb;
            const int hg = i % G;
            const int r = a.members[it.member_off + member];
            const int h = it.g * G + hg;
            gid = ((int64_t)r * dm.BW + b) * dm.Hq + h;
            live = b < a.n_live[r];
        }
        sm.gid[tid] = gid;
        sm.live[tid] = live;
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.f;
    }
    __syncthreads();
    int any_live = 0;
    for (int r = 0; r < n_rows; ++r) any_live |= sm.live[r];
    if (!any_live) return;   // every row of the item belongs to a dead beam

    for (int idx = tid; idx < kSmallRows * D / 8; idx += kThreads) {
        const int r = idx / (D / 8), c = idx % (D / 8);
        float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (r < n_rows && sm.live[r]) {
            const uint4 u = *reinterpret_cast<const uint4 *>(a.q + sm.gid[r] * D + c * 8);
            unpack8(u, f);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.q[r * D + c * 8 + e] = f[e];
    }

    // ---- per-thread output accumulators: dim d, rows rg, rg + kRowGroups, ...
    const int d = tid % D;
    const int rg = tid / D;
    float acc[kRowsPerThread];
#pragma unroll
    for (int j = 0; j < kRowsPerThread; ++j) acc[j] = 0.f;

    const int64_t head_row0 = (int64_t)it.g * a.kv_tokens + it.kv_off;
    for (int kb = it.key_begin; kb < it.key_end; kb += kTileKeys) {
        const int nk = min(kTileKeys, it.key_end - kb);
        __syncthreads();   // previous tile fully consumed
        // the tile's K and V rows, every 16-byte piece in flight at once
        for (int idx = tid; idx < nk * (D / 8); idx += kThreads) {
            const int j = idx / (D / 8), c = idx % (D / 8);
            const int64_t src = (head_row0 + kb + j) * D + c * 8;
            cp_async16(smem_u32(&sm.k[j * kRow + c * 8]), a.kstore + src);
            cp_async16(smem_u32(&sm.v[j * kRow + c * 8]), a.vstore + src);
        }
        cp_async_wait_all();
        __syncthreads();

        // scores: thread tid <-> key j of the tile, all rows
        {
            const int j = tid;
            float s[kSmallRows];
#pragma unroll
            for (int r = 0; r < kSmallRows; ++r) s[r] = 0.f;
            if (j < nk) {
                for (int c = 0; c < D / 8; ++c) {
                    float kf[8];
                    unpack8(*reinterpret_cast<const uint4 *>(&sm.k[j * kRow + c * 8]), kf);
#pragma unroll
                    for (int r = 0; r < kSmallRows; ++r) {
                        if (r < n_rows) {
                            const float4 q0 = *reinterpret_cast<const float4 *>(&sm.q[r * D + c * 8]);
                            const float4 q1 = *reinterpret_cast<const float4 *>(&sm.q[r * D + c * 8 + 4]);
                            s[r] += q0.x * kf[0] + q0.y * kf[1] + q0.z * kf[2] + q0.w * kf[3] +
                                    q1.x * kf[4] + q1.y * kf[5] + q1.z * kf[6] + q1.w * kf[7];
                        }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kSmallRows; ++r)
                if (r < n_rows) sm.p[r * kTileKeys + j] = (j < nk) ? s[r] * scale_log2 : -INFINITY;
        }
        __syncthreads();

        // running max / sum per row: warp w takes rows w, w+4, ...
        {
            const int w = tid / 32, lane = tid % 32;
            for (int r = w; r < n_rows; r += kThreads / 32) {
                float x[kTileKeys / 32];
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < kTileKeys / 32; ++c) {
                    x[c] = sm.p[r * kTileKeys + lane + 32 * c];
                    mx = fmaxf(mx, x[c]);
                }
                mx = warp_max(mx);
                const float m_old = sm.m[r];
                const float m_new = fmaxf(m_old, mx);
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < kTileKeys / 32; ++c) {
                    const float pv = exp2f(x[c] - m_new);
                    sm.p[r * kTileKeys + lane + 32 * c] = pv;
                    sum += pv;
                }
                sum = warp_sum(sum);
                if (lane == 0) {
                    const float al = exp2f(m_old - m_new);
                    sm.alpha[r] = al;
                    sm.l[r] = sm.l[r] * al + sum;
                    sm.m[r] = m_new;
                }
            }
        }
        __syncthreads();

        // O += P V for this thread's dim and rows
#pragma unroll
        for (int jr = 0; jr < kRowsPerThread; ++jr) {
            const int r = rg + jr * kRowGroups;
            if (r < n_rows) acc[jr] *= sm.alpha[r];
        }
        for (int j = 0; j < nk; ++j) {
            const float vj = bf2f(sm.v[j * kRow + d]);
#pragma unroll
            for (int jr = 0; jr < kRowsPerThread; ++jr) {
                const int r = rg + jr * kRowGroups;
                if (r < n_rows) acc[jr] += sm.p[r * kTileKeys + j] * vj;
            }
        }
    }
    __syncthreads();

    // ---- write the partials of live rows
    const int64_t rows = a.part.rows;
#pragma unroll
    for (int jr = 0; jr < kRowsPerThread; ++jr) {
        const int r = rg + jr * kRowGroups;
        if (r < n_rows && sm.live[r]) {
            a.part.o[((int64_t)it.slot * rows + sm.gid[r]) * D + d] = acc[jr];
            if (d == 0) a.part.ml[(int64_t)it.slot * rows + sm.gid[r]] = make_float2(sm.m[r], sm.l[r]);
        }
    }
}

template <int D>
cudaError_t launch_small_impl(const SmallArgs &a, int n_items, cudaStream_t st) {
    const size_t smem = sizeof(SmallSmem<D>);
    static bool attr = false;   // set once, on the first (uncaptured) launch
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(attn_small_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    return launch_pdl(attn_small_kernel<D>, dim3(n_items), dim3(kThreads), smem, st, a);
}

}  // namespace

cudaError_t launch_attn_small(const SmallArgs &a, int n_items, cudaStream_t st) {
    if (n_items <= 0) return cudaSuccess;
    if (a.dims.D == 128) return launch_small_impl<128>(a, n_items, st);
    if (a.dims.D == 64) return launch_small_impl<64>(a, n_items, st);
    return cudaErrorInvalidValue;
}

}  // namespace xgr

// attn_per_beam.cu -- the per-beam comparison path (not the product path).
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"), 1
// "Problem definition", memory inefficiency: serving systems built around
// PagedAttention treat each beam as an independent sequence, so every beam
// reloads the shared prompt KV, and forking beams copies KV blocks.  Section 4
// ("Kernel efficiency") measures the staged kernel against that baseline.
// This file builds the baseline so the ratio can be measured on B200:
//  * fork_copy_kernel: each live beam owns one block of kPerBeamBlock tokens
//    for its generated tokens (double-buffered by step parity); at step s >= 1
//    a beam copies its parent's whole block (the parent is its ancestry slot
//    of step s-1), then appends this step's k / v at position s;
//  * per_beam_attn_kernel: one CTA per (request, beam, kv head) streams the
//    request's whole prompt (+ suffix) from the KV store and the beam's own
//    block on the CUDA cores (eight warps over contiguous key ranges, one key
//    per lane for the scores, one head-dim quad per lane for the weighted
//    values, online softmax in base 2), then merges the warps.
// Results equal xgr_decode_step's within rounding (the same oracle checks
// both); the context's Unshared pool is not touched.
#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr int kPbThreads = 256;
constexpr int kPbWarps = kPbThreads / 32;
constexpr int kPbMaxG = 8;   // query heads per kv head

__device__ __forceinline__ int64_t block_off(const PerBeamArgs &a, int parity, int64_t r, int b, int g) {
    // [parity][B][BW][Hkv][kPerBeamBlock][D]
    return ((((int64_t)parity * a.Bcap + r) * a.dims.BW + b) * a.dims.Hkv + g) * kPerBeamBlock * a.dims.D;
}

__global__ void __launch_bounds__(kPbThreads) fork_copy_kernel(PerBeamArgs a) {
    const Dims dm = a.dims;
    const int64_t u = blockIdx.x;   // (request, beam, kv head)
    const int g = (int)(u % dm.Hkv), b = (int)((u / dm.Hkv) % dm.BW), r = (int)(u / ((int64_t)dm.Hkv * dm.BW));
    griddep_wait();
    griddep_launch_dependents();
    if (b >= a.n_live[r]) return;
    const int s = a.step, par = s & 1;
    const int64_t dst = block_off(a, par, r, b, g);
    const int n16 = kPerBeamBlock * dm.D / 8;   // 16-byte pieces of one block
    if (s > 0) {
        const int p = a.st.anc[((int64_t)r * dm.BW + b) * dm.S + (s - 1)];   // the parent beam
        if (p < 0 || p >= dm.BW) {
            if (threadIdx.x == 0) set_status(a.status, XGR_DEV_INDEX);
            return;
        }
        const int64_t src = block_off(a, par ^ 1, r, p, g);
        for (int i = threadIdx.x; i < n16; i += kPbThreads) {   // the whole block, as a block copy does
            reinterpret_cast<uint4 *>(a.blk_k + dst)[i] = reinterpret_cast<const uint4 *>(a.blk_k + src)[i];
            reinterpret_cast<uint4 *>(a.blk_v + dst)[i] = reinterpret_cast<const uint4 *>(a.blk_v + src)[i];
        }
        __syncthreads();   // the copy lands before the append overwrites position s
    }
    const int64_t src_new = (((int64_t)r * dm.BW + b) * dm.Hkv + g) * dm.D;
    for (int i = threadIdx.x; i < dm.D / 8; i += kPbThreads) {
        reinterpret_cast<uint4 *>(a.blk_k + dst + (int64_t)s * dm.D)[i] = reinterpret_cast<const uint4 *>(a.k_new + src_new)[i];
        reinterpret_cast<uint4 *>(a.blk_v + dst + (int64_t)s * dm.D)[i] = reinterpret_cast<const uint4 *>(a.v_new + src_new)[i];
    }
}

// key i of (request r, kv head g, beam block) in [prompt | suffix | own tokens]
__device__ __forceinline__ const __nv_bfloat16 *key_row(const __nv_bfloat16 *store, const __nv_bfloat16 *blk,
                                                        const int32_t (&seg)[4], int64_t head_off, int i,
                                                        int D) {
    if (i < seg[1]) return store + head_off + ((int64_t)seg[0] + i) * D;
    i -= seg[1];
    if (i < seg[3]) return store + head_off + ((int64_t)seg[2] + i) * D;
    return blk + (int64_t)(i - seg[3]) * D;
}

template <int G>
__global__ void __launch_bounds__(kPbThreads) per_beam_attn_kernel(PerBeamArgs a) {
    constexpr int D = 128;
    __shared__ float qs[G][D];
    __shared__ float wm[kPbWarps][G], wl[kPbWarps][G];
    __shared__ float wo[kPbWarps][G][D];
    const Dims dm = a.dims;
    const int64_t u = blockIdx.x;
    const int g = (int)(u % dm.Hkv), b = (int)((u / dm.Hkv) % dm.BW), r = (int)(u / ((int64_t)dm.Hkv * dm.BW));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    griddep_wait();
    griddep_launch_dependents();
    const int64_t row0 = ((int64_t)r * dm.BW + b) * dm.Hq + (int64_t)g * G;   // first query row
    if (b >= a.n_live[r]) {   // dead beam: O = 0, LSE = -inf
        for (int i = threadIdx.x; i < G * D; i += kPbThreads) a.out[row0 * D + i] = __float2bfloat16(0.f);
        if (threadIdx.x < G) a.lse[row0 + threadIdx.x] = -INFINITY;
        return;
    }
    const float scale = kLog2e * rsqrtf((float)D);
    for (int i = threadIdx.x; i < G * D; i += kPbThreads) qs[i / D][i % D] = __bfloat162float(a.q[row0 * D + i]) * scale;
    int32_t seg[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) seg[k] = a.req_seg[(int64_t)r * 4 + k];
    const int64_t head_off = (int64_t)g * a.kv_tokens * D;
    const __nv_bfloat16 *blk_k = a.blk_k + block_off(a, a.step & 1, r, b, g);
    const __nv_bfloat16 *blk_v = a.blk_v + block_off(a, a.step & 1, r, b, g);
    const int n = seg[1] + seg[3] + a.step + 1;
    __syncthreads();
    // this warp's keys [k0, k1)
    const int per = (n + kPbWarps - 1) / kPbWarps;
    const int k0 = min(n, warp * per), k1 = min(n, k0 + per);
    float m[G], l[G], o[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) o[h][e] = 0.f;
    }
    for (int c0 = k0; c0 < k1; c0 += 32) {
        // scores: lane = key
        const int i = c0 + lane;
        float sc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) sc[h] = -INFINITY;
        if (i < k1) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(key_row(a.kstore, blk_k, seg, head_off, i, D));
#pragma unroll
            for (int h = 0; h < G; ++h) sc[h] = 0.f;
#pragma unroll 8
            for (int c = 0; c < D / 8; ++c) {
                const uint4 w = __ldg(kr + c);
                const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
                float kv[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(p2[e]);
                    kv[2 * e] = f.x;
                    kv[2 * e + 1] = f.y;
                }
#pragma unroll
                for (int h = 0; h < G; ++h)
#pragma unroll
                    for (int e = 0; e < 8; ++e) sc[h] = fmaf(qs[h][8 * c + e], kv[e], sc[h]);
            }
        }
        // online softmax per head over the chunk
        float pr[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float cm = sc[h];
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o2));
            const float mn = fmaxf(m[h], cm);
            const float alpha = m[h] == -INFINITY ? 0.f : exp2f(m[h] - mn);
            pr[h] = sc[h] == -INFINITY ? 0.f : exp2f(sc[h] - mn);
            float ps = pr[h];
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
            l[h] = l[h] * alpha + ps;
            m[h] = mn;
#pragma unroll
            for (int e = 0; e < 4; ++e) o[h][e] *= alpha;
        }
        // weighted values: lane = head-dim quad; eight keys' rows in flight at a time
        const int nk = min(32, k1 - c0);
        for (int j0 = 0; j0 < nk; j0 += 8) {
            uint2 vw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                vw[u] = j0 + u < nk
                            ? __ldg(reinterpret_cast<const uint2 *>(key_row(a.vstore, blk_v, seg, head_off, c0 + j0 + u, D)) + lane)
                            : make_uint2(0u, 0u);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&vw[u]);
                const float2 v01 = __bfloat1622float2(p2[0]), v23 = __bfloat1622float2(p2[1]);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float p = __shfl_sync(0xffffffffu, pr[h], j0 + u);   // 0 past the chunk's keys
                    o[h][0] = fmaf(p, v01.x, o[h][0]);
                    o[h][1] = fmaf(p, v01.y, o[h][1]);
                    o[h][2] = fmaf(p, v23.x, o[h][2]);
                    o[h][3] = fmaf(p, v23.y, o[h][3]);
                }
            }
        }
    }
    // merge the warps
#pragma unroll
    for (int h = 0; h < G; ++h) {
        if (lane == 0) {
            wm[warp][h] = m[h];
            wl[warp][h] = l[h];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) wo[warp][h][4 * lane + e] = o[h][e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += kPbThreads) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
        for (int w = 0; w < kPbWarps; ++w) M = fmaxf(M, wm[w][h]);
        float L = 0.f, O = 0.f;
        for (int w = 0; w < kPbWarps; ++w) {
            if (wm[w][h] == -INFINITY) continue;
            const float f = exp2f(wm[w][h] - M);
            L += wl[w][h] * f;
            O += wo[w][h][d] * f;
        }
        a.out[(row0 + h) * D + d] = __float2bfloat16(O / L);
        if (d == 0) a.lse[row0 + h] = (M + log2f(L)) * kLn2;
    }
}

}  // namespace

cudaError_t launch_per_beam(const PerBeamArgs &a, cudaStream_t st) {
    const Dims &dm = a.dims;
    if (dm.D != 128 || dm.G < 1 || dm.G > kPbMaxG || a.step + 1 > kPerBeamBlock) return cudaErrorInvalidValue;
    const int64_t units = (int64_t)dm.B * dm.BW * dm.Hkv;
    if (units <= 0) return cudaSuccess;
    if (units > 0x7fffffff) return cudaErrorInvalidValue;
    cudaError_t e = launch_pdl(fork_copy_kernel, dim3((unsigned)units), dim3(kPbThreads), 0, st, a);
    if (e != cudaSuccess) return e;
    switch (dm.G) {
        case 1: return launch_pdl(per_beam_attn_kernel<1>, dim3((unsigned)units), dim3(kPbThreads), 0, st, a);
        case 2: return launch_pdl(per_beam_attn_kernel<2>, dim3((unsigned)units), dim3(kPbThreads), 0, st, a);
        case 4: return launch_pdl(per_beam_attn_kernel<4>, dim3((unsigned)units), dim3(kPbThreads), 0, st, a);
        case 8: return launch_pdl(per_beam_attn_kernel<8>, dim3((unsigned)units), dim3(kPbThreads), 0, st, a);
        default: return cudaErrorInvalidValue;
    }
}

size_t per_beam_block_bytes(int Bcap, int BW, int Hkv, int D) {
    return (size_t)2 * 2 * Bcap * BW * Hkv * kPerBeamBlock * D * 2;   // K and V, two parities, bf16
}

}  // namespace xgr

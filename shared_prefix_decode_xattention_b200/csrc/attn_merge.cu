// attn_merge.cu -- Unshared stage and Merging stage of the staged attention,
// with the append of this step's k/v into the token-granular Unshared pool.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"), 2.1:
//  * "Token-granular management": the Unshared cache holds one entry per
//    generated token, so a beam's history is a list of direct indices
//    (ancestry slots) into per-step token slots -- no block padding and no
//    block copy when beams fork.
//  * "Staged computation": the Unshared stage computes local scores with their
//    max/sum statistics independently of the Shared stage; the Merging stage
//    combines all partials by online softmax.
// One warp per (request, beam, kv head): its G query rows share the gathered
// k/v of the beam's step+1 tokens (16-byte vector loads, one 2*D-byte vector
// per token), then fold in the Shared-stage partials and write O (bf16) and
// LSE (fp32, natural log).
#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr int kWarps = 4;

template <int D>
struct LaneVec {
    static constexpr int N = D / 32;   // dims per lane (4 or 2)
};

template <int D>
__device__ __forceinline__ void load_lane(const __nv_bfloat16 *p, int lane, float *f) {
    constexpr int N = LaneVec<D>::N;
    if constexpr (N == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p + lane * 4);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
        float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
        f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p + lane * 2);
        float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
        f[0] = a.x; f[1] = a.y;
    }
}

template <int D>
__device__ __forceinline__ void copy_lane(const __nv_bfloat16 *src, __nv_bfloat16 *dst, int lane) {
    constexpr int N = LaneVec<D>::N;
    if constexpr (N == 4) {
        *reinterpret_cast<uint2 *>(dst + lane * 4) = *reinterpret_cast<const uint2 *>(src + lane * 4);
    } else {
        *reinterpret_cast<uint32_t *>(dst + lane * 2) =
            *reinterpret_cast<const uint32_t *>(src + lane * 2);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kWarps * 32) attn_merge_kernel(MergeArgs a) {
    constexpr int N = LaneVec<D>::N;
    const Dims dm = a.dims;
    const int lane = threadIdx.x % 32;
    const int64_t wid = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
    const int64_t n_units = (int64_t)dm.B * dm.BW * dm.Hkv;
    griddep_wait();   // the partials come from the attention kernels before
    griddep_launch_dependents();
    if (wid >= n_units) return;
    const int g = (int)(wid % dm.Hkv);
    const int b = (int)((wid / dm.Hkv) % dm.BW);
    const int r = (int)(wid / ((int64_t)dm.Hkv * dm.BW));
    const int s = a.step;
    const int64_t beam_row = (int64_t)r * dm.BW + b;
    const int64_t gid0 = beam_row * dm.Hq + (int64_t)g * G;   // row of query head g*G
    if (b >= a.st.n_live[r]) {   // dead beam: O = 0, LSE = -inf
#pragma unroll
        for (int hg = 0; hg < G; ++hg) {
#pragma unroll
            for (int e = 0; e < N; ++e) a.out[(gid0 + hg) * D + lane * N + e] = __float2bfloat16(0.f);
            if (lane == 0) a.lse[gid0 + hg] = -INFINITY;
        }
        return;
    }
    const int n_slots = a.n_slots[r];
    if (n_slots < 0) return;   // the tensor-core kernel already finished this live beam

    // append this step's token of the beam at Unshared slot (s, b)
    const int64_t kv_off = (beam_row * dm.Hkv + g) * D;
    const __nv_bfloat16 *kn = a.k_new + kv_off;
    const __nv_bfloat16 *vn = a.v_new + kv_off;
    const int64_t pool_step = (int64_t)a.Bcap * dm.BW * dm.Hkv * D;
    const int64_t pool_beam = ((int64_t)r * dm.BW * dm.Hkv) * D;
    copy_lane<D>(kn, a.pool_k + s * pool_step + pool_beam + ((int64_t)b * dm.Hkv + g) * D, lane);
    copy_lane<D>(vn, a.pool_v + s * pool_step + pool_beam + ((int64_t)b * dm.Hkv + g) * D, lane);

    // Every load below that does not depend on another goes out at once (the
    // beam's ancestry slots, then all its k and v rows, and the partials four
    // slots at a time), so the warp waits a few round trips, not one per token
    // and per partial.
    float q[G][N];
#pragma unroll
    for (int hg = 0; hg < G; ++hg) load_lane<D>(a.q + (gid0 + hg) * D, lane, q[hg]);
    int slot[kMaxSteps];
#pragma unroll
    for (int i = 0; i < kMaxSteps; ++i) slot[i] = i < s ? a.st.anc[beam_row * dm.S + i] : b;

    // ---- Unshared stage: the beam's own tokens of steps 0..s
    const float scale_log2 = kLog2e * rsqrtf((float)D);
    float kf[kMaxSteps][N], vf[kMaxSteps][N];
    bool tok_ok[kMaxSteps];
#pragma unroll
    for (int i = 0; i < kMaxSteps; ++i) {
        tok_ok[i] = i <= s && slot[i] >= 0 && slot[i] < dm.BW;
        if (i <= s && !tok_ok[i] && lane == 0) set_status(a.st.status, XGR_DEV_INDEX);   // corrupt ancestry
        const int64_t off = i * pool_step + pool_beam + ((int64_t)slot[i] * dm.Hkv + g) * D;
        const __nv_bfloat16 *kp = i == s ? kn : a.pool_k + off;
        const __nv_bfloat16 *vp = i == s ? vn : a.pool_v + off;
#pragma unroll
        for (int e = 0; e < N; ++e) kf[i][e] = vf[i][e] = 0.f;
        if (tok_ok[i]) {
            load_lane<D>(kp, lane, kf[i]);
            load_lane<D>(vp, lane, vf[i]);
        }
    }
    float m[G], l[G], o[G][N];
#pragma unroll
    for (int hg = 0; hg < G; ++hg) {
        float sc[kMaxSteps];
        m[hg] = -INFINITY;
#pragma unroll
        for (int i = 0; i < kMaxSteps; ++i) {
            float t = 0.f;
#pragma unroll
            for (int e = 0; e < N; ++e) t += q[hg][e] * kf[i][e];
            sc[i] = tok_ok[i] ? warp_sum(t) * scale_log2 : -INFINITY;
            m[hg] = fmaxf(m[hg], sc[i]);
        }
        l[hg] = 0.f;
#pragma unroll
        for (int e = 0; e < N; ++e) o[hg][e] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxSteps; ++i) {
            if (!tok_ok[i]) continue;
            const float p = exp2f(sc[i] - m[hg]);
            l[hg] += p;
#pragma unroll
            for (int e = 0; e < N; ++e) o[hg][e] += p * vf[i][e];
        }
    }

    // ---- Merging stage: fold in every Shared-stage partial (online softmax),
    // loading four slots at a time
    for (int p0 = 0; p0 < n_slots; p0 += 4) {
        float2 ml[4][G];
        float po[4][G][N];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int hg = 0; hg < G; ++hg) {
                const int64_t prow = (int64_t)(p0 + u) * a.part.rows + gid0 + hg;
                const bool in = p0 + u < n_slots;
                ml[u][hg] = in ? a.part.ml[prow] : make_float2(-INFINITY, 0.f);
                if constexpr (N == 4) {
                    const float4 t = in ? *reinterpret_cast<const float4 *>(a.part.o + prow * D + lane * 4)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    po[u][hg][0] = t.x; po[u][hg][1] = t.y; po[u][hg][2] = t.z; po[u][hg][3] = t.w;
                } else {
                    const float2 t = in ? *reinterpret_cast<const float2 *>(a.part.o + prow * D + lane * 2)
                                        : make_float2(0.f, 0.f);
                    po[u][hg][0] = t.x; po[u][hg][1] = t.y;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (p0 + u >= n_slots) break;
#pragma unroll
            for (int hg = 0; hg < G; ++hg) {
                const float m_new = fmaxf(m[hg], ml[u][hg].x);
                const float a1 = exp2f(m[hg] - m_new), a2 = exp2f(ml[u][hg].x - m_new);
                l[hg] = l[hg] * a1 + ml[u][hg].y * a2;
#pragma unroll
                for (int e = 0; e < N; ++e) o[hg][e] = o[hg][e] * a1 + po[u][hg][e] * a2;
                m[hg] = m_new;
            }
        }
    }

    // ---- write O (bf16) and LSE (natural log)
#pragma unroll
    for (int hg = 0; hg < G; ++hg) {
        const float inv = 1.f / l[hg];
        __nv_bfloat16 *dst = a.out + (gid0 + hg) * D + lane * N;
        if constexpr (N == 4) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(o[hg][0] * inv, o[hg][1] * inv);
            __nv_bfloat162 hi = __floats2bfloat162_rn(o[hg][2] * inv, o[hg][3] * inv);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t *>(&lo);
            u.y = *reinterpret_cast<uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(dst) = u;
        } else {
            __nv_bfloat162 lo = __floats2bfloat162_rn(o[hg][0] * inv, o[hg][1] * inv);
            *reinterpret_cast<__nv_bfloat162 *>(dst) = lo;
        }
        if (lane == 0) a.lse[gid0 + hg] = (m[hg] + log2f(l[hg])) * kLn2;
    }
}

template <int D>
cudaError_t launch_d(const MergeArgs &a, cudaStream_t st) {
    const int64_t units = (int64_t)a.dims.B * a.dims.BW * a.dims.Hkv;
    const int blocks = (int)((units + kWarps - 1) / kWarps);
    if (blocks == 0) return cudaSuccess;
    switch (a.dims.G) {
        case 1: return launch_pdl(attn_merge_kernel<D, 1>, dim3(blocks), dim3(kWarps * 32), 0, st, a);
        case 2: return launch_pdl(attn_merge_kernel<D, 2>, dim3(blocks), dim3(kWarps * 32), 0, st, a);
        case 4: return launch_pdl(attn_merge_kernel<D, 4>, dim3(blocks), dim3(kWarps * 32), 0, st, a);
        case 8: return launch_pdl(attn_merge_kernel<D, 8>, dim3(blocks), dim3(kWarps * 32), 0, st, a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_attn_merge(const MergeArgs &a, cudaStream_t st) {
    if (a.dims.D == 128) return launch_d<128>(a, st);
    if (a.dims.D == 64) return launch_d<64>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace xgr

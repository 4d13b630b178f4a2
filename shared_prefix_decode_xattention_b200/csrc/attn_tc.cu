// attn_tc.cu -- Shared-stage attention on the 5th-generation tensor cores.
//
// xGR page ("xGR: Efficient Generative Recommendation Serving at Scale"), 2.1
// "Separate KV cache" / "Staged computation": the prompt KV is read ONCE per
// request for all beams, and the Shared stage produces local scores with
// their max / sum-of-exponentials for the Merging stage.  Reading the prompt
// once for all beams turns the stage into a dense contraction: the query rows
// of all beams x the query heads of one kv head (128 rows per tile) against
// the prompt keys -- S = Q K^T, then O = softmax-weights(S) V.  The page notes
// the kernel turns memory-bound into compute-bound; at 128+ beams it runs on
// the tensor cores here.
//
// One CTA per work item (kv head, 128-row tile, key range):
//   warp 0      TMA producer: K and V chunks of 128 keys (two 64-column
//               128-byte-swizzled boxes each), double-buffered, K and V on
//               separate barriers so the next K streams in while P V runs;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_j = Q K_j^T into one of two TMEM buffers, then
//               O += P_{j-1} V_{j-1} into the TMEM O accumulator;
//   warps 2-5   one query row per thread: read S_j from TMEM, running max
//               (lazy rescaling: O is rescaled only when the max grows by more
//               than 2^8), exponentials, row sums, P_j (bf16) into shared
//               memory in the canonical 128-byte-swizzled K-major layout;
//               finally read O from TMEM and write the partial (O, m, l).
// Every wait on an mbarrier is bounded; on time-out the CTA records
// XGR_DEV_TIMEOUT in the status word and unwinds (no trap, no hang).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr int kTcThreads = 192;
constexpr int kBlockN = 128;                 // keys per chunk
constexpr uint32_t kHalf = 16384;            // one 128-row x 64-column bf16 sub-tile
constexpr uint32_t kTile = 2 * kHalf;        // 128 x 128 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTile;            // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;
constexpr uint32_t kOffP = kOffV + 2 * kTile;  // 2 buffers
constexpr uint32_t kOffBar = kOffP + 2 * kTile;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;   // barriers + alignment slack
constexpr uint32_t kTmemCols = 512;          // S0 [0,128) S1 [128,256) O [256,384)
constexpr uint32_t kSpinLimit = 1u << 22;

// barrier slots (8 bytes each) after kOffBar
enum { B_KFULL = 0, B_VFULL = 2, B_KEMPTY = 4, B_VEMPTY = 6, B_SFULL = 8, B_PFULL = 10,
       B_PVDONE = 12, B_QFULL = 14, B_DRAIN = 15, B_COUNT = 16 };

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Bounded wait for the completion of the phase with the given parity.  Gives
// up early when another role has aborted (abort != nullptr and set); on its
// own time-out it sets the abort flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort) {
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
        if (abort && (it & 255) == 255 && *abort) return false;
    }
    if (abort) *abort = 1;
    return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: version 1).
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// byte offset of 16-byte chunk c (0..15) of row `row` in a 128-row tile stored
// as two 128-byte-swizzled 64-column halves (the TMA / UMMA canonical layout)
__device__ __forceinline__ uint32_t sw128_off(int row, int c) {
    return (uint32_t)(c >> 3) * kHalf + (uint32_t)row * 128u + (uint32_t)(((c & 7) ^ (row & 7)) << 4);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_holder;
    __shared__ int abort_flag;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sb = smem_u32(base);
    const uint32_t bar0 = sb + kOffBar;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };

    const WorkItem it = a.items[blockIdx.x];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n_keys = it.key_end - it.key_begin;
    const int nchunks = (n_keys + kBlockN - 1) / kBlockN;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_KFULL + s), 1);
            mbar_init(bar(B_VFULL + s), 1);
            mbar_init(bar(B_KEMPTY + s), 1);
            mbar_init(bar(B_VEMPTY + s), 1);
            mbar_init(bar(B_SFULL + s), 1);
            mbar_init(bar(B_PFULL + s), 128);
            mbar_init(bar(B_PVDONE + s), 1);
        }
        mbar_init(bar(B_QFULL), 128);
        mbar_init(bar(B_DRAIN), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_holder;
    volatile int *abort = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int y0 = it.g * (int)a.kv_tokens + it.kv_off + it.key_begin;
            int nk[2] = {0, 0}, nv[2] = {0, 0};   // loads issued per stage
            for (int j = 0; j < nchunks; ++j) {
                const int st = j & 1;
                const int y = y0 + j * kBlockN;
                if (j >= 2 && !mbar_wait(bar(B_KEMPTY + st), ((j - 2) >> 1) & 1, abort)) break;
                mbar_expect_tx(bar(B_KFULL + st), kTile);
                tma_load_2d(sb + kOffK + st * kTile, &tmk, 0, y, bar(B_KFULL + st));
                tma_load_2d(sb + kOffK + st * kTile + kHalf, &tmk, 64, y, bar(B_KFULL + st));
                ++nk[st];
                if (j >= 2 && !mbar_wait(bar(B_VEMPTY + st), ((j - 2) >> 1) & 1, abort)) break;
                mbar_expect_tx(bar(B_VFULL + st), kTile);
                tma_load_2d(sb + kOffV + st * kTile, &tmv, 0, y, bar(B_VFULL + st));
                tma_load_2d(sb + kOffV + st * kTile + kHalf, &tmv, 64, y, bar(B_VFULL + st));
                ++nv[st];
            }
            if (*abort) {   // let the copies in flight land before the CTA exits
                for (int st = 0; st < 2; ++st) {
                    if (nk[st]) mbar_wait(bar(B_KFULL + st), (nk[st] - 1) & 1, nullptr);
                    if (nv[st]) mbar_wait(bar(B_VFULL + st), (nv[st] - 1) & 1, nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
            bool ok = mbar_wait(bar(B_QFULL), 0, abort);
            for (int j = 0; ok && j <= nchunks; ++j) {
                if (j < nchunks) {
                    const int st = j & 1;
                    if (!mbar_wait(bar(B_KFULL + st), (j >> 1) & 1, abort)) break;
                    fence_after_sync();
                    const uint32_t kq = sb + kOffQ, kk = sb + kOffK + st * kTile;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (uint32_t)(k >> 2) * kHalf + (uint32_t)(k & 3) * 32u;
                        umma_bf16(tmem + (uint32_t)st * 128u, umma_desc(kq + off, 16, 1024),
                                  umma_desc(kk + off, 16, 1024), idS, k > 0);
                    }
                    umma_commit(bar(B_SFULL + st));
                    umma_commit(bar(B_KEMPTY + st));
                }
                if (j >= 1) {
                    const int jp = j - 1, sp = jp & 1;
                    if (!mbar_wait(bar(B_PFULL + sp), (jp >> 1) & 1, abort)) break;
                    if (!mbar_wait(bar(B_VFULL + sp), (jp >> 1) & 1, abort)) break;
                    fence_after_sync();
                    const uint32_t kp = sb + kOffP + sp * kTile, kv = sb + kOffV + sp * kTile;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t offp = (uint32_t)(k >> 2) * kHalf + (uint32_t)(k & 3) * 32u;
                        umma_bf16(tmem + 256u, umma_desc(kp + offp, 16, 1024),
                                  umma_desc(kv + (uint32_t)k * 2048u, kHalf, 1024), idPV,
                                  (jp > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(bar(B_PVDONE + sp));
                    umma_commit(bar(B_VEMPTY + sp));
                }
            }
            if (*abort) {   // every MMA issued so far must finish before TMEM is freed
                umma_commit(bar(B_DRAIN));
                mbar_wait(bar(B_DRAIN), 0, nullptr);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax rows
        const int row = 32 * (warp & 3) + lane;
        const Dims dm = a.dims;
        const int G = dm.G;
        int64_t gid = -1;
        bool live = false;
        if (row < it.n_rows) {
            const int i = it.row_begin + row;
            const int member = i / (a.nb * G);
            const int b = (i / G) % a.nb;
            const int hg = i % G;
            const int r = a.members[it.member_off + member];
            gid = ((int64_t)r * dm.BW + b) * dm.Hq + it.g * G + hg;
            live = b < a.n_live[r];
        }
        // Q row -> shared memory (canonical swizzled K-major layout)
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.q + (live ? gid : 0) * 128);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                uint4 u = live ? src[c] : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(base + kOffQ + sw128_off(row, c)) = u;
            }
            fence_async_smem();
            mbar_arrive(bar(B_QFULL));
        }
        const float cscale = kLog2e * rsqrtf(128.f);
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nchunks && ok; ++j) {
            const int sbuf = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + sbuf), (j >> 1) & 1, abort));
            if (!ok) break;
            fence_after_sync();
            float s[128];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tmem + lane_base + sbuf * 128 + q4 * 32, s + q4 * 32);
            tmem_wait_ld();
            const int nvalid = min(kBlockN, n_keys - j * kBlockN);
            // row max over the raw scores (the scale is positive), 8 independent chains
            float mxp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxp[e] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                if (c >= nvalid) s[c] = -INFINITY;
                mxp[c & 7] = fmaxf(mxp[c & 7], s[c]);
            }
            const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                                   fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) * cscale;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_used + 8.f) {
                alpha = exp2f(m_used - mx);
                rescale = j > 0;
                m_used = mx;
            }
            const float neg_m = -m_used;
            float sp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) sp[e] = 0.f;
            uint32_t packed[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = exp2f(fmaf(s[2 * c], cscale, neg_m));
                const float p1 = exp2f(fmaf(s[2 * c + 1], cscale, neg_m));
                sp[c & 7] += p0 + p1;
                __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                packed[c] = *reinterpret_cast<uint32_t *>(&h);
            }
            const float sum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
            l = l * alpha + sum;
            if (j >= 2) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + sbuf), ((j - 2) >> 1) & 1, abort));
                if (!ok) break;
            }
            if (__any_sync(0xffffffffu, rescale)) {
                // O must hold every P V product up to chunk j-1 before it is rescaled
                const int jp = j - 1;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + (jp & 1)), (jp >> 1) & 1, abort));
                if (!ok) break;
                fence_after_sync();
                const float f = rescale ? alpha : 1.f;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + 256 + q4 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= f;
                    tmem_st32(tmem + lane_base + 256 + q4 * 32, o);
                }
                tmem_wait_st();
            }
            uint8_t *pb = base + kOffP + sbuf * kTile;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<uint4 *>(pb + sw128_off(row, c)) =
                    make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
            fence_async_smem();
            fence_before_sync();
            mbar_arrive(bar(B_PFULL + sbuf));
        }
        if (ok && nchunks > 0) {
            const int jl = nchunks - 1;
            if (__all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + (jl & 1)), (jl >> 1) & 1, abort))) {
                fence_after_sync();
                float *dst = a.part.o + ((int64_t)it.slot * a.part.rows + (live ? gid : 0)) * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + 256 + q4 * 32, o);
                    tmem_wait_ld();
                    if (live) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(dst + q4 * 32 + e) =
                                make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
                    }
                }
                if (live) a.part.ml[(int64_t)it.slot * a.part.rows + gid] = make_float2(m_used, l);
            }
        }
    }

    fence_before_sync();
    __syncthreads();
    if (*abort && tid == 0) set_status(a.status, XGR_DEV_TIMEOUT);
    if (warp == 1) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

cudaError_t make_kv_tensor_map(CUtensorMap *map, const void *base, int64_t rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_attn_tc(const CUtensorMap &tmk, const CUtensorMap &tmv, const TcArgs &a,
                           int n_items, cudaStream_t st) {
    if (n_items <= 0) return cudaSuccess;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    attn_tc_kernel<<<n_items, kTcThreads, kSmemBytes, st>>>(tmk, tmv, a);
    return cudaGetLastError();
}

}  // namespace xgr

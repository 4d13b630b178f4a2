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
//   warp 0      TMA producer: Q, then K and V chunks of 128 keys (two 64-column
//               128-byte-swizzled boxes each) on separate two-stage rings;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_j = Q K_j^T into TMEM buffer j % 2, O_{j%2} += P_j V_j with
//               P_j read from tensor memory;
//   warp 10     gathers the Unshared chunks (see below);
//   warps 2-9   two softmax warpgroups; warpgroup h owns the chunks j with
//               j % 2 == h, one query row per thread: it reads S_j from TMEM,
//               keeps the running max and sum of its own accumulator O_h (lazy
//               rescaling: O_h is rescaled only when the max grows by more than
//               2^8), and writes P_j (bf16 pairs) over the first half of S_j's
//               TMEM buffer, so no shared memory goes to P (it holds the
//               Unshared staging area instead).  The two warpgroups never wait for each other
//               inside the loop, so one's exponentials overlap the other's row
//               maxima and TMEM traffic; at the end they swap (m, l) and merge
//               O_0 and O_1 into the partial (O, m, l) or, for a request's only
//               segment, the output.
// In a request's only KV segment ("final" items) the Unshared and Merging
// stages run here too.  The Unshared stage is one more key chunk of the same
// loop (or a few, when the tile's beams x tokens pass 128): a gather warp
// collects the tile's beams' own k / v rows of steps 0..s (direct
// indices into the token-granular pool; this step's from k_new / v_new) into
// the U area at kernel start, so the gather overlaps the Shared loop, and
// append this step's k / v to the pool.  Row u of that chunk is token u % T of
// the tile's beam u / T (T = s + 1 tokens per beam): the chunk is block-
// diagonal, and each query row keeps only its own beam's valid tokens (the
// rest of the chunk's scores are masked to -inf before the exponentials).
// The online softmax then merges the Shared and Unshared stages as it goes.
// Zero-fill items (step 0) only write the rows of the beams that are not live
// yet.
// Every wait on an mbarrier is bounded; on time-out the CTA records
// XGR_DEV_TIMEOUT in the status word and unwinds (no trap, no hang).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr int kTcThreads = 352;              // producer warp, MMA warp, 2 softmax warpgroups, gather warp
constexpr int kGatherWarp = 10;              // gathers the Unshared chunks (and appends this step's k / v)
constexpr int kSoftmaxThreads = 256;
constexpr int kGroupThreads = 128;           // one softmax warpgroup: one query row per thread
constexpr int kBlockN = 128;                 // keys per chunk
constexpr int kKStages = 2;                  // K chunks in flight
constexpr int kVStages = 2;                  // V chunks in flight
constexpr uint32_t kHalf = 16384;            // one 128-row x 64-column bf16 sub-tile
constexpr uint32_t kTile = 2 * kHalf;        // 128 x 128 bf16
constexpr uint32_t kUBytes = 65536;          // U area: the Unshared chunk's K and V tiles
constexpr int kGatherLanes = 32;             // the gather warp's lanes
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTile;
constexpr uint32_t kOffV = kOffK + kKStages * kTile;
constexpr uint32_t kOffU = kOffV + kVStages * kTile;
constexpr uint32_t kOffBar = kOffU + kUBytes;
constexpr uint32_t kOffMisc = kOffBar + 256;  // TMEM address, abort flag
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = 232448;       // the sm_100 per-block maximum
constexpr uint32_t kSmemSpare = kSmemBytes - kSmemUsed;   // room to realign the window
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P_j (bf16, two
// per column) overwrites the first 64 columns of S_j's buffer once S_j is read
constexpr uint32_t kTmemCols = 512;

// barrier slots (8 bytes each) after kOffBar; SFULL, PFULL, PVDONE and XCH have one
// slot per warpgroup
enum { B_KFULL = 0, B_KEMPTY = B_KFULL + kKStages, B_VFULL = B_KEMPTY + kKStages,
       B_VEMPTY = B_VFULL + kVStages, B_SFULL = B_VEMPTY + kVStages, B_PFULL = B_SFULL + 2,
       B_PVDONE = B_PFULL + 2, B_QFULL = B_PVDONE + 2, B_DONE = B_QFULL + 1, B_XCH = B_DONE + 1,
       B_UFULL = B_XCH + 2, B_UEMPTY = B_UFULL + 1, B_COUNT = B_UEMPTY + 1 };
// B_PVDONE: P_j V_j has completed (S_j's TMEM buffer, which held P_j, may take
// S_{j+2}); B_DONE: every MMA has completed; B_XCH: the warpgroups' (m, l) exchange;
// B_UFULL: an Unshared chunk is gathered into the U area; B_UEMPTY: its MMAs have
// completed (the U area may take the next one)
static_assert(B_COUNT * 8 <= 256, "barrier area");

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
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

// the same with A in tensor memory (rows in lanes, two bf16 per 32-bit column)
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate)
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

// wait for this thread's TMEM loads; v (their destination) is tied to the wait,
// so no use of it can be scheduled before
__device__ __forceinline__ void tmem_wait_ld_into(float *v) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
                   "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]),
                   "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]), "+f"(v[18]),
                   "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]), "+f"(v[24]),
                   "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]), "+f"(v[30]),
                   "+f"(v[31])
                 :
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

__device__ __forceinline__ float ex2(float x) {   // 2^x, one MUFU op; tiny results flush to 0
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pair a * b + c (one instruction for two lanes of arithmetic on
// sm_100), each element rounded as the scalar fmaf rounds it.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// query row `row` of a work item -> (request, beam, query head, global row, live)
struct RowInfo {
    int r, b, hg;
    int64_t gid;
    bool valid, live;
};
__device__ __forceinline__ RowInfo row_info(const TcArgs &a, const WorkItem &it, int row) {
    RowInfo ri{0, 0, 0, 0, false, false};
    if (row < it.n_rows) {
        const int G = a.dims.G;
        const int i = it.row_begin + row;
        const int member = i / (a.nb * G);
        ri.b = (i / G) % a.nb;
        ri.hg = i % G;
        ri.r = it.n_members == 1 ? it.r0 : a.members[it.member_off + member];
        ri.gid = ((int64_t)ri.r * a.dims.BW + ri.b) * a.dims.Hq + it.g * G + ri.hg;
        ri.valid = true;
    }
    return ri;
}

// 11 warps: the register file is split over the 4 schedulers (16K registers each) and 3
// warps share each of three of them, so a thread may use at most 168 registers.  One instance
// serves every step (the code is warm in the caches after the first launch).
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   const __grid_constant__ CUtensorMap tmq, TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > kSmemSpare) {   // the dynamic window is expected 1024-aligned; never trap
        if (threadIdx.x == 0) set_status(a.status, XGR_DEV_TIMEOUT);
        return;
    }
    uint8_t *base = smem_raw + pad;
    const uint32_t sb = smem_u32(base);
    const uint32_t bar0 = sb + kOffBar;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + kOffMisc);
    int *abort_flag = reinterpret_cast<int *>(base + kOffMisc + 4);

    const WorkItem it = a.items[blockIdx.x];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    if (it.flags & 4) {   // zero-fill item: these CTAs run beside the attention on idle SMs
        griddep_wait();
        griddep_launch_dependents();
        const int64_t row0 = ((int64_t)it.r0 * a.dims.BW + it.row_begin) * a.dims.Hq;   // first query row
        const int64_t n = (int64_t)it.n_rows * a.dims.Hq;
        uint4 *o = reinterpret_cast<uint4 *>(a.out + row0 * 128);
        for (int64_t u = tid; u < n * 16; u += kTcThreads) o[u] = make_uint4(0, 0, 0, 0);
        for (int64_t u = tid; u < n; u += kTcThreads) a.lse[row0 + u] = -INFINITY;
        return;
    }
    const int n_keys = it.key_end - it.key_begin;
    const int nchunks = (n_keys + kBlockN - 1) / kBlockN;   // Shared-stage chunks
    const bool final_item = (it.flags & 1) != 0;
    // Unshared chunks (final items): the tile's beams x (s + 1) tokens, 128 rows each
    const int T = a.step + 1;
    const int lb0 = it.row_begin / a.dims.G;
    const int nbeam = (it.row_begin + it.n_rows - 1) / a.dims.G - lb0 + 1;
    const int n_u = final_item ? (nbeam * T + kBlockN - 1) / kBlockN : 0;
    const int nall = nchunks + n_u;
    const bool q_tma = (it.flags & 2) != 0;   // the Q tile is one TMA box
    volatile int *abort = abort_flag;
    const int y0 = it.g * (int)a.kv_tokens + it.kv_off + it.key_begin;
    // producer lanes: lane 0 streams K chunks, lane 1 V chunks, each on its own ring
    auto issue_k = [&](int j) {
        const int st = j % kKStages;
        mbar_expect_tx(bar(B_KFULL + st), kTile);
        tma_load_2d(sb + kOffK + st * kTile, &tmk, 0, y0 + j * kBlockN, bar(B_KFULL + st));
        tma_load_2d(sb + kOffK + st * kTile + kHalf, &tmk, 64, y0 + j * kBlockN, bar(B_KFULL + st));
    };
    auto issue_v = [&](int j) {
        const int st = j % kVStages;
        mbar_expect_tx(bar(B_VFULL + st), kTile);
        tma_load_2d(sb + kOffV + st * kTile, &tmv, 0, y0 + j * kBlockN, bar(B_VFULL + st));
        tma_load_2d(sb + kOffV + st * kTile + kHalf, &tmv, 64, y0 + j * kBlockN, bar(B_VFULL + st));
    };

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < kKStages; ++s) {
                mbar_init(bar(B_KFULL + s), 1);
                mbar_init(bar(B_KEMPTY + s), 1);
            }
            for (int s = 0; s < kVStages; ++s) {
                mbar_init(bar(B_VFULL + s), 1);
                mbar_init(bar(B_VEMPTY + s), 1);
            }
            for (int h = 0; h < 2; ++h) {
                mbar_init(bar(B_SFULL + h), 1);
                mbar_init(bar(B_PFULL + h), kGroupThreads);
                mbar_init(bar(B_PVDONE + h), 1);
                mbar_init(bar(B_XCH + h), kGroupThreads);
            }
            mbar_init(bar(B_QFULL), q_tma ? 1 : kSoftmaxThreads);
            mbar_init(bar(B_DONE), 1);
            mbar_init(bar(B_UFULL), kGatherLanes);
            mbar_init(bar(B_UEMPTY), 1);
            *abort_flag = 0;
            fence_mbar_init();
        }
        __syncwarp();
        // The prompt's first K / V chunks stream in while the kernel before this
        // one finishes: the prompt (and suffix) KV store is written only by the
        // prefill copies, which completed before any decode kernel started.
        if (lane == 0)
            for (int j = 0; j < min(nchunks, kKStages); ++j) issue_k(j);
        if (lane == 1)
            for (int j = 0; j < min(nchunks, kVStages); ++j) issue_v(j);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Everything above touches only this CTA's shared and tensor memory, the
    // plan (written before any decode kernel) and the prompt KV store; from
    // here on the kernel reads what the kernels before it wrote (the beam
    // state, this step's inputs).
    griddep_wait();
    griddep_launch_dependents();
    if (warp == 0 && lane == 0 && q_tma) {   // Q streams in before the block-wide setup barrier
        const int G = a.dims.G;
        const int z = it.r0 * a.dims.BW + it.row_begin / G;
        mbar_expect_tx(bar(B_QFULL), kTile);
        tma_load_3d(sb + kOffQ, &tmq, 0, it.g * G, z, bar(B_QFULL));
        tma_load_3d(sb + kOffQ + kHalf, &tmq, 64, it.g * G, z, bar(B_QFULL));
    }
    // softmax threads stage the Q tile meanwhile: 16 consecutive threads read one
    // 256-byte row (coalesced) and write it in the swizzled K-major layout
    if (warp >= 2 && warp < kGatherWarp && !q_tma) {
        const int ts = tid - 64;
        uint4 qv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = ts + kSoftmaxThreads * k;
            const RowInfo qi = row_info(a, it, idx >> 4);
            qv[k] = qi.valid ? reinterpret_cast<const uint4 *>(a.q + qi.gid * 128)[idx & 15]
                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = ts + kSoftmaxThreads * k;
            *reinterpret_cast<uint4 *>(base + kOffQ + sw128_off(idx >> 4, idx & 15)) = qv[k];
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producers
        if (lane == 0) {
            int n_issued = min(nchunks, kKStages);
            for (int j = kKStages; j < nchunks && n_issued == j; ++j) {
                if (!mbar_wait(bar(B_KEMPTY + j % kKStages), ((j / kKStages) - 1) & 1, abort)) break;
                issue_k(j);
                ++n_issued;
            }
            if (*abort)   // let the copies in flight land before the CTA exits
                for (int j = max(0, n_issued - kKStages); j < n_issued; ++j)
                    mbar_wait(bar(B_KFULL + j % kKStages), (j / kKStages) & 1, nullptr);
        } else if (lane == 1) {
            int n_issued = min(nchunks, kVStages);
            for (int j = kVStages; j < nchunks && n_issued == j; ++j) {
                if (!mbar_wait(bar(B_VEMPTY + j % kVStages), ((j / kVStages) - 1) & 1, abort)) break;
                issue_v(j);
                ++n_issued;
            }
            if (*abort)
                for (int j = max(0, n_issued - kVStages); j < n_issued; ++j)
                    mbar_wait(bar(B_VFULL + j % kVStages), (j / kVStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Chunk j belongs to warpgroup h = j % 2: S_j goes to TMEM buffer h, P_j
        // comes from P buffer h, and P_j V_j accumulates into O_h.  Order of
        // issue: S_0, S_1, then for each j: S_{j+2} as soon as warpgroup h has
        // read S_j, then P_j V_j once P_j is written.
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
            // chunk j < nchunks: a Shared chunk in the K / V rings; j >= nchunks: an
            // Unshared chunk in the U area (its K and V land together on B_UFULL)
            auto k_ready = [&](int j, bool block) -> bool {
                const uint32_t b = j < nchunks ? bar(B_KFULL + j % kKStages) : bar(B_UFULL);
                const uint32_t ph = j < nchunks ? (j / kKStages) & 1 : (j - nchunks) & 1;
                return block ? mbar_wait(b, ph, abort) : mbar_test(b, ph);
            };
            auto issue_s = [&](int j) {   // S_j = Q K_j^T into TMEM buffer j % 2
                fence_after_sync();
                const uint32_t kq = sb + kOffQ;
                const uint32_t kk = j < nchunks ? sb + kOffK + (j % kKStages) * kTile : sb + kOffU;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (uint32_t)(k >> 2) * kHalf + (uint32_t)(k & 3) * 32u;
                    umma_bf16(tmem + (uint32_t)(j & 1) * 128u, umma_desc(kq + off, 16, 1024),
                              umma_desc(kk + off, 16, 1024), idS, k > 0);
                }
                umma_commit(bar(B_SFULL + (j & 1)));
                if (j < nchunks) umma_commit(bar(B_KEMPTY + j % kKStages));
            };
            bool ok = mbar_wait(bar(B_QFULL), 0, abort);
            int ns = 0;   // the next S to issue
            for (; ok && ns < min(nall, 2); ++ns) {
                ok = k_ready(ns, true);
                if (ok) issue_s(ns);
            }
            // Then whichever is ready first: S_ns (P_{ns-2} V_{ns-2}, which read its
            // TMEM buffer, complete and K_ns landed) or O_h += P_j V_j (P_j written,
            // V_j landed).  Every phase polled here is at most one behind the
            // barrier's current one, so the parity tests are exact.
            uint32_t idle = 0;
            for (int j = 0; ok && j < nall;) {
                bool progress = false;
                if (ns < nall && mbar_test(bar(B_PVDONE + (ns & 1)), ((ns - 2) >> 1) & 1) &&
                    k_ready(ns, false)) {
                    issue_s(ns++);
                    progress = true;
                }
                const int h = j & 1, sv = j % kVStages;
                const bool v_ready = j < nchunks ? mbar_test(bar(B_VFULL + sv), (j / kVStages) & 1)
                                                 : mbar_test(bar(B_UFULL), (j - nchunks) & 1);
                if (!(mbar_test(bar(B_PFULL + h), (j >> 1) & 1) && v_ready)) {
                    if (progress) {
                        idle = 0;
                    } else if (++idle >= kSpinLimit) {
                        *abort = 1;
                        ok = false;
                    } else if ((idle & 255) == 0 && *abort) {
                        ok = false;
                    }
                    continue;
                }
                idle = 0;
                fence_after_sync();
                const uint32_t kv = j < nchunks ? sb + kOffV + sv * kTile : sb + kOffU + kTile;
#pragma unroll
                for (int k = 0; k < 8; ++k)   // P_j: 16 keys = 8 TMEM columns per MMA
                    umma_bf16_ts(tmem + 256u + (uint32_t)h * 128u, tmem + (uint32_t)h * 128u + 8u * k,
                                 umma_desc(kv + (uint32_t)k * 2048u, kHalf, 1024), idPV,
                                 (k > 0 || j >= 2) ? 1u : 0u);
                umma_commit(bar(B_PVDONE + h));
                umma_commit(j < nchunks ? bar(B_VEMPTY + sv) : bar(B_UEMPTY));
                ++j;
            }
            // arrives once every MMA issued above has completed (TMEM final / free)
            umma_commit(bar(B_DONE));
            if (*abort) mbar_wait(bar(B_DONE), 0, nullptr);
        }
    } else if (warp < kGatherWarp) {
        // ------------------------------------------------------------ softmax
        // Warpgroup `half` owns the chunks j with j % 2 == half, whole rows: thread
        // `row` reads TMEM lane `row` of S buffer `half`, keeps the running max and
        // sum of accumulator O_half and writes row `row` of P_j over it.  The
        // two warpgroups never wait for each other inside the loop; their
        // (m, l, O) are merged at the end, where thread (row, half) handles
        // head-dim columns [64*half, 64*half + 64).
        const int half = (warp - 2) >> 2;
        const int row = 32 * (warp & 3) + lane;
        bool ok = true;
        if (!q_tma) {
            fence_async_smem();
            mbar_arrive(bar(B_QFULL));
        }

        const RowInfo ri = row_info(a, it, row);
        const float cscale = kLog2e * rsqrtf(128.f);
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t col0 = (uint32_t)(64 * half);
        float m_used = -INFINITY, l = 0.f;   // running max / sum of O_half
        const Dims dm = a.dims;
        const bool live = ri.valid && ri.b < a.n_live[ri.r];
        // Unshared chunks: this row keeps columns [u_lo, u_lo + T) of the block-
        // diagonal U rows -- its beam's tokens -- where the token's slot is valid
        // (bit i of vmask; this step's own token when the beam is live)
        uint32_t vmask = 0;
        const int u_lo = ((it.row_begin + row) / dm.G - lb0) * T;
        if (final_item && live) {
            const int64_t beam_row = (int64_t)ri.r * dm.BW + ri.b;
            vmask = 1u << a.step;
            for (int i = 0; i < a.step; ++i) {
                const int sl = a.st.anc[beam_row * dm.S + i];
                if (sl >= 0 && sl < dm.BW) vmask |= 1u << i;
                else if (ri.hg == 0 && half == 0) set_status(a.status, XGR_DEV_INDEX);
            }
        }
        const uint32_t s_col = (uint32_t)half * 128u;          // S buffer of this warpgroup
        const uint32_t o_col = 256u + (uint32_t)half * 128u;   // its O accumulator
        for (int j = half, jj = 0; ok && j < nall; j += 2, ++jj) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + half), jj & 1, abort));
            if (!ok) break;
            fence_after_sync();
            const int nvalid = n_keys - j * kBlockN;   // keys of the chunk inside the range
            const bool is_u = j >= nchunks;            // an Unshared chunk
            const int c0 = u_lo - kBlockN * (j - nchunks);   // (is_u) the row's first column in it
            // Masked chunks (an Unshared chunk: only this row's own tokens count;
            // the range's last chunk: keys past its end do not) keep the
            // columns of a 32-bit mask per 32-column piece
            const bool masked = is_u || nvalid < kBlockN;
            auto piece_mask = [&](int q2) -> uint32_t {
                if (is_u) {   // the row's valid tokens (vmask) start at column c0
                    const int off = c0 - 32 * q2;
                    return off >= 32 || off <= -32 ? 0u : off >= 0 ? vmask << off : vmask >> -off;
                }
                const int nv = nvalid - 32 * q2;
                return nv >= 32 ? ~0u : nv <= 0 ? 0u : (1u << nv) - 1u;
            };
            // the chunk's 128 scores in one TMEM read (P_j then overwrites them)
            float sv[128];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) tmem_ld32(tmem + lane_base + s_col + 32 * q2, sv + 32 * q2);
            tmem_wait_ld();
            if (masked) {
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const uint32_t pm = piece_mask(q2);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((pm >> e) & 1u)) sv[32 * q2 + e] = -INFINITY;
                }
            }
            // row maximum: eight chains of three-input maxima
            float mxp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxp[e] = fmaxf(sv[e], sv[8 + e]);
#pragma unroll
            for (int c = 16; c < 128; c += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) mxp[e] = fmax3(mxp[e], sv[c + e], sv[c + 8 + e]);
            const float mx = fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmax3(mxp[3], mxp[4], mxp[5]),
                                   fmaxf(mxp[6], mxp[7])) * cscale;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_used + 8.f) {   // lazy rescaling: keep the old max unless it grew by 2^8
                alpha = ex2(m_used - mx);
                rescale = jj > 0;   // O_half already holds data
                m_used = mx;
            }
            // (S_j was issued after P_{j-2} V_{j-2} completed: O_half is current and
            // this TMEM buffer no longer holds P_{j-2})
            // exponentials, row sum and P (bf16 pairs) into the first 64 columns of
            // the S buffer, from the scores already in registers (masked ones are
            // -inf): piece q's 16 P columns land on scores already read
            // x = s * scale - m in packed pairs; sums in eight chains
            const float2 sc2 = make_float2(cscale, cscale), nm2 = make_float2(-m_used, -m_used);
            float sp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) sp[e] = 0.f;
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                float pw[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 x = ffma2(make_float2(sv[32 * q2 + 2 * e], sv[32 * q2 + 2 * e + 1]), sc2, nm2);
                    const float2 p = make_float2(ex2(x.x), ex2(x.y));
                    sp[(2 * e) & 7] += p.x;
                    sp[(2 * e + 1) & 7] += p.y;
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p.x, p.y);
                    pw[e] = __uint_as_float(*reinterpret_cast<uint32_t *>(&h2));
                }
                tmem_st16(tmem + lane_base + s_col + 16 * q2, pw);
            }
            if (__any_sync(0xffffffffu, rescale)) {   // O_half *= alpha before P_j V_j adds in
                fence_after_sync();
                const float f = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int q2 = 0; q2 < 4; ++q2) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + o_col + q2 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= f;
                    tmem_st32(tmem + lane_base + o_col + q2 * 32, o);
                }
                tmem_wait_st();
            }
            l = l * alpha + (((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7])));
            tmem_wait_st();   // P_j (and a rescaled O_half) in TMEM before the MMA warp reads them
            fence_before_sync();
            mbar_arrive(bar(B_PFULL + half));
        }
        // every MMA done: O_0 and O_1 are final, the P buffers free
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0, abort));
        if (ok) {
            fence_after_sync();
            // the warpgroups swap (m, l); thread (row, half) then merges head-dim
            // columns [64*half, 64*half + 64) of O_0 and O_1
            float2 *xl = reinterpret_cast<float2 *>(base + kOffV);   // [2][128]; V is consumed
            xl[half * 128 + row] = make_float2(m_used, l);
            mbar_arrive(bar(B_XCH + half));
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_XCH + (half ^ 1)), 0, abort));
            const float2 other = xl[(half ^ 1) * 128 + row];
            const float m0 = half == 0 ? m_used : other.x, l0 = half == 0 ? l : other.y;
            const float m1 = half == 0 ? other.x : m_used, l1 = half == 0 ? other.y : l;
            const float M = fmaxf(m0, m1);
            // an accumulator that never received a chunk (m = -inf) holds no data
            const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
            const float f1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
            const float l_row = l0 * f0 + l1 * f1;
            if (ok) {
#pragma unroll 1
                for (int q2 = 0; q2 < 2; ++q2) {
                    float o[32], o1[32];
                    tmem_ld32(tmem + lane_base + 256 + col0 + 32 * q2, o);
                    tmem_ld32(tmem + lane_base + 384 + col0 + 32 * q2, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = (f0 != 0.f ? o[e] * f0 : 0.f) + (f1 != 0.f ? o1[e] * f1 : 0.f);
                    const uint32_t c0 = col0 + 32 * q2;
                    if (!final_item) {
                        if (live) {
                            float *dst = a.part.o + ((int64_t)it.slot * a.part.rows + ri.gid) * 128 + c0;
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *reinterpret_cast<float4 *>(dst + e) =
                                    make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
                        }
                    } else if (ri.valid) {
                        // final: O / l in bf16; dead rows 0
                        const float inv = live ? 1.f / l_row : 0.f;
                        uint4 *dst = reinterpret_cast<uint4 *>(a.out + ri.gid * 128 + c0);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t w4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float v0 = live ? o[8 * c + 2 * e] * inv : 0.f;
                                const float v1 = live ? o[8 * c + 2 * e + 1] * inv : 0.f;
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                                w4[e] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
                if (half == 0) {
                    if (!final_item) {
                        if (live) a.part.ml[(int64_t)it.slot * a.part.rows + ri.gid] = make_float2(M, l_row);
                    } else if (ri.valid) {   // LSE = m + log2(l) in natural log; dead rows -inf
                        a.lse[ri.gid] = live ? (M + __log2f(l_row)) * kLn2 : -INFINITY;
                    }
                }
            }
        }
    } else if (n_u > 0) {
        // ------------------------------------------------------------ gather
        {
            // ---- Unshared stage: gather the tile's beams' own k / v rows of steps
            // 0..s into the U area, one 128-row chunk at a time (row u: token u % T
            // of tile beam u / T), in the canonical swizzled layout; rows of dead
            // beams, bad slots and the tail are zero.  This step's rows are also
            // appended to the pool at slot (s, b).
            const int gl = lane;
            const Dims dm = a.dims;
            const int s_now = a.step;
            const int64_t pool_step = (int64_t)a.Bcap * dm.BW * dm.Hkv * 128;
            for (int q = 0; q < n_u; ++q) {
                if (q > 0 && !mbar_wait(bar(B_UEMPTY), (q - 1) & 1, abort)) break;
                // this lane's rows u = gl + k * kGatherLanes: their request and beam,
                // then every index they need, then the copies -- each stage's loads
                // all in flight together
                constexpr int kRowsPerLane = (kBlockN + kGatherLanes - 1) / kGatherLanes;
                int rr[kRowsPerLane], bb[kRowsPerLane], ii[kRowsPerLane];
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    const int u = gl + k * kGatherLanes, ug = kBlockN * q + u, lb = ug / T;
                    ii[k] = ug % T;
                    rr[k] = -1;
                    bb[k] = -1;
                    if (u < kBlockN && lb < nbeam) {
                        const int lbs = lb0 + lb;   // beam index within the segment's rows / G
                        bb[k] = lbs % a.nb;
                        rr[k] = it.n_members == 1 ? it.r0 : a.members[it.member_off + lbs / a.nb];
                    }
                }
                int nl[kRowsPerLane], sl[kRowsPerLane];
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    nl[k] = rr[k] >= 0 ? a.n_live[rr[k]] : 0;
                    sl[k] = (rr[k] >= 0 && ii[k] < s_now)
                                ? a.st.anc[((int64_t)rr[k] * dm.BW + bb[k]) * dm.S + ii[k]] : -1;
                }
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    const int u = gl + k * kGatherLanes;
                    if (u >= kBlockN) continue;
                    const __nv_bfloat16 *sk = nullptr, *sv = nullptr;
                    if (rr[k] >= 0 && bb[k] < nl[k]) {
                        const int64_t brow = (int64_t)rr[k] * dm.BW + bb[k];
                        if (ii[k] == s_now) {
                            sk = a.k_new + (brow * dm.Hkv + it.g) * 128;
                            sv = a.v_new + (brow * dm.Hkv + it.g) * 128;
                        } else if (sl[k] >= 0 && sl[k] < dm.BW) {
                            const int64_t prow = (brow - bb[k] + sl[k]) * dm.Hkv + it.g;
                            sk = a.pool_k + ii[k] * pool_step + prow * 128;
                            sv = a.pool_v + ii[k] * pool_step + prow * 128;
                        }
                    }
                    const uint32_t dk = sb + kOffU, dv = sb + kOffU + kTile;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        if (sk) {
                            cp_async16(dk + sw128_off(u, c), sk + 8 * c);
                            cp_async16(dv + sw128_off(u, c), sv + 8 * c);
                        } else {
                            *reinterpret_cast<uint4 *>(base + kOffU + sw128_off(u, c)) = make_uint4(0, 0, 0, 0);
                            *reinterpret_cast<uint4 *>(base + kOffU + kTile + sw128_off(u, c)) =
                                make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                cp_async_wait_all();
                // this step's k / v of the gathered live beams -> pool slot (s, b)
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    const int u = gl + k * kGatherLanes;
                    if (u >= kBlockN || rr[k] < 0 || ii[k] != s_now || bb[k] >= nl[k]) continue;
                    const int64_t orow = ((int64_t)rr[k] * dm.BW + bb[k]) * dm.Hkv + it.g;
                    uint4 *pk = reinterpret_cast<uint4 *>(a.pool_k + s_now * pool_step + orow * 128);
                    uint4 *pv = reinterpret_cast<uint4 *>(a.pool_v + s_now * pool_step + orow * 128);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        pk[c] = *reinterpret_cast<const uint4 *>(base + kOffU + sw128_off(u, c));
                        pv[c] = *reinterpret_cast<const uint4 *>(base + kOffU + kTile + sw128_off(u, c));
                    }
                }
                fence_async_smem();   // the gathered rows are visible to the tensor cores
                mbar_arrive(bar(B_UFULL));
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


// ---------------------------------------------------------------- one-O variant
// For short items (a few key chunks each) both softmax warpgroups add into one O:
// that frees TMEM for a third S buffer, so S_{j+3} waits for P_j V_j, issued a
// whole chunk earlier, and the tensor pipe does not drain between chunks.  A row
// then has one reference maximum (shared memory), raised lazily -- only when a
// chunk's max passes it by more than 2^8 -- by the warpgroup that sees that
// chunk; the other warpgroup takes the new reference (B_DEC) before its next
// chunk's P, and O is rescaled between the two products.  Long items keep
// attn_tc_kernel, whose warpgroups never wait for each other.
namespace one_o {

constexpr uint32_t kOffMref = kOffMisc + 16;  // [128] each row's reference maximum (log2 units)
constexpr uint32_t kSmemUsed = kOffMref + 512;
constexpr uint32_t kSmemSpare = kSmemBytes - kSmemUsed;   // room to realign the window
// TMEM columns: S0 [0,128) S1 [128,256) S2 [256,384) O [384,512); S_j goes to
// buffer j % 3, and P_j (bf16, two per column) overwrites its first 64 columns
// once S_j is read.
constexpr int kSBufs = 3;
constexpr uint32_t kOCol = 384;
// P_j written and P_j V_j complete: barriers j % 4.  (With three S buffers a
// warpgroup may finish chunk j+2 before P_j V_j is issued -- S_{j+2} waits only
// for P_{j-1} V_{j-1} -- but not chunk j+4, whose S waits for P_{j+1} V_{j+1};
// and P_{j+4} V_{j+4} cannot complete before S_{j+4}, issued once P_{j+1} V_{j+1}
// was seen complete: four barriers of each keep every phase polled at most one
// behind the barrier's current one, so the parity tests are exact.)
constexpr int kPBars = 4;
// S_j complete: barrier j % 6, so that each barrier serves one warpgroup and
// its phases are consumed in order without relying on commit order
constexpr int kSBars = 6;

// barrier slots (8 bytes each) after kOffBar
enum { B_KFULL = 0, B_KEMPTY = B_KFULL + kKStages, B_VFULL = B_KEMPTY + kKStages,
       B_VEMPTY = B_VFULL + kVStages, B_SFULL = B_VEMPTY + kVStages, B_PFULL = B_SFULL + kSBars,
       B_PVDONE = B_PFULL + kPBars, B_QFULL = B_PVDONE + kPBars, B_DONE = B_QFULL + 1, B_XCH = B_DONE + 1,
       B_UFULL = B_XCH + 2, B_UEMPTY = B_UFULL + 1, B_DEC = B_UEMPTY + 1, B_COUNT = B_DEC + 2 };
// B_SFULL: one per chunk index mod 6; B_PFULL, B_PVDONE: one per chunk index
// mod 4; B_DEC: one per chunk parity (= warpgroup).  B_PVDONE: P_j V_j has completed (O holds every product up to
// chunk j; S_j's buffer, which held P_j, may take S_{j+3}); B_DEC: chunk j's
// warpgroup has settled the rows' reference maxima for chunk j (the other
// warpgroup reads them for chunk j+1); B_DONE: every MMA has completed; B_XCH: the warpgroups' l exchange;
// B_UFULL: an Unshared chunk is gathered into the U area; B_UEMPTY: its MMAs have
// completed (the U area may take the next one)
static_assert(B_COUNT * 8 <= 256, "barrier area");

// The one-O variant (same warps, shared memory and registers as attn_tc_kernel).
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_one_o_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   const __grid_constant__ CUtensorMap tmq, TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > kSmemSpare) {   // the dynamic window is expected 1024-aligned; never trap
        if (threadIdx.x == 0) set_status(a.status, XGR_DEV_TIMEOUT);
        return;
    }
    uint8_t *base = smem_raw + pad;
    const uint32_t sb = smem_u32(base);
    const uint32_t bar0 = sb + kOffBar;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + kOffMisc);
    int *abort_flag = reinterpret_cast<int *>(base + kOffMisc + 4);

    const WorkItem it = a.items[blockIdx.x];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    if (it.flags & 4) {   // zero-fill item: these CTAs run beside the attention on idle SMs
        griddep_wait();
        griddep_launch_dependents();
        const int64_t row0 = ((int64_t)it.r0 * a.dims.BW + it.row_begin) * a.dims.Hq;   // first query row
        const int64_t n = (int64_t)it.n_rows * a.dims.Hq;
        uint4 *o = reinterpret_cast<uint4 *>(a.out + row0 * 128);
        for (int64_t u = tid; u < n * 16; u += kTcThreads) o[u] = make_uint4(0, 0, 0, 0);
        for (int64_t u = tid; u < n; u += kTcThreads) a.lse[row0 + u] = -INFINITY;
        return;
    }
    const int n_keys = it.key_end - it.key_begin;
    const int nchunks = (n_keys + kBlockN - 1) / kBlockN;   // Shared-stage chunks
    const bool final_item = (it.flags & 1) != 0;
    // Unshared chunks (final items): the tile's beams x (s + 1) tokens, 128 rows each
    const int T = a.step + 1;
    const int lb0 = it.row_begin / a.dims.G;
    const int nbeam = (it.row_begin + it.n_rows - 1) / a.dims.G - lb0 + 1;
    const int n_u = final_item ? (nbeam * T + kBlockN - 1) / kBlockN : 0;
    const int nall = nchunks + n_u;
    const bool q_tma = (it.flags & 2) != 0;   // the Q tile is one TMA box
    volatile int *abort = abort_flag;
    const int y0 = it.g * (int)a.kv_tokens + it.kv_off + it.key_begin;
    // producer lanes: lane 0 streams K chunks, lane 1 V chunks, each on its own ring
    auto issue_k = [&](int j) {
        const int st = j % kKStages;
        mbar_expect_tx(bar(B_KFULL + st), kTile);
        tma_load_2d(sb + kOffK + st * kTile, &tmk, 0, y0 + j * kBlockN, bar(B_KFULL + st));
        tma_load_2d(sb + kOffK + st * kTile + kHalf, &tmk, 64, y0 + j * kBlockN, bar(B_KFULL + st));
    };
    auto issue_v = [&](int j) {
        const int st = j % kVStages;
        mbar_expect_tx(bar(B_VFULL + st), kTile);
        tma_load_2d(sb + kOffV + st * kTile, &tmv, 0, y0 + j * kBlockN, bar(B_VFULL + st));
        tma_load_2d(sb + kOffV + st * kTile + kHalf, &tmv, 64, y0 + j * kBlockN, bar(B_VFULL + st));
    };

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < kKStages; ++s) {
                mbar_init(bar(B_KFULL + s), 1);
                mbar_init(bar(B_KEMPTY + s), 1);
            }
            for (int s = 0; s < kVStages; ++s) {
                mbar_init(bar(B_VFULL + s), 1);
                mbar_init(bar(B_VEMPTY + s), 1);
            }
            for (int h = 0; h < kPBars; ++h) {
                mbar_init(bar(B_PFULL + h), kGroupThreads);
                mbar_init(bar(B_PVDONE + h), 1);
            }
            for (int h = 0; h < 2; ++h) {
                mbar_init(bar(B_XCH + h), kGroupThreads);
                mbar_init(bar(B_DEC + h), kGroupThreads);
            }
            for (int b = 0; b < kSBars; ++b) mbar_init(bar(B_SFULL + b), 1);
            mbar_init(bar(B_QFULL), q_tma ? 1 : kSoftmaxThreads);
            mbar_init(bar(B_DONE), 1);
            mbar_init(bar(B_UFULL), kGatherLanes);
            mbar_init(bar(B_UEMPTY), 1);
            *abort_flag = 0;
            fence_mbar_init();
        }
        __syncwarp();
        // The prompt's first K / V chunks stream in while the kernel before this
        // one finishes: the prompt (and suffix) KV store is written only by the
        // prefill copies, which completed before any decode kernel started.
        if (lane == 0)
            for (int j = 0; j < min(nchunks, kKStages); ++j) issue_k(j);
        if (lane == 1)
            for (int j = 0; j < min(nchunks, kVStages); ++j) issue_v(j);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Everything above touches only this CTA's shared and tensor memory, the
    // plan (written before any decode kernel) and the prompt KV store; from
    // here on the kernel reads what the kernels before it wrote (the beam
    // state, this step's inputs).
    griddep_wait();
    griddep_launch_dependents();
    if (warp == 0 && lane == 0 && q_tma) {   // Q streams in before the block-wide setup barrier
        const int G = a.dims.G;
        const int z = it.r0 * a.dims.BW + it.row_begin / G;
        mbar_expect_tx(bar(B_QFULL), kTile);
        tma_load_3d(sb + kOffQ, &tmq, 0, it.g * G, z, bar(B_QFULL));
        tma_load_3d(sb + kOffQ + kHalf, &tmq, 64, it.g * G, z, bar(B_QFULL));
    }
    // softmax threads stage the Q tile meanwhile: 16 consecutive threads read one
    // 256-byte row (coalesced) and write it in the swizzled K-major layout
    if (warp >= 2 && warp < kGatherWarp && !q_tma) {
        const int ts = tid - 64;
        uint4 qv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = ts + kSoftmaxThreads * k;
            const RowInfo qi = row_info(a, it, idx >> 4);
            qv[k] = qi.valid ? reinterpret_cast<const uint4 *>(a.q + qi.gid * 128)[idx & 15]
                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = ts + kSoftmaxThreads * k;
            *reinterpret_cast<uint4 *>(base + kOffQ + sw128_off(idx >> 4, idx & 15)) = qv[k];
        }
    }
    if (warp >= 2 && warp < 6) reinterpret_cast<float *>(base + kOffMref)[tid - 64] = -INFINITY;
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producers
        if (lane == 0) {
            int n_issued = min(nchunks, kKStages);
            for (int j = kKStages; j < nchunks && n_issued == j; ++j) {
                if (!mbar_wait(bar(B_KEMPTY + j % kKStages), ((j / kKStages) - 1) & 1, abort)) break;
                issue_k(j);
                ++n_issued;
            }
            if (*abort)   // let the copies in flight land before the CTA exits
                for (int j = max(0, n_issued - kKStages); j < n_issued; ++j)
                    mbar_wait(bar(B_KFULL + j % kKStages), (j / kKStages) & 1, nullptr);
        } else if (lane == 1) {
            int n_issued = min(nchunks, kVStages);
            for (int j = kVStages; j < nchunks && n_issued == j; ++j) {
                if (!mbar_wait(bar(B_VEMPTY + j % kVStages), ((j / kVStages) - 1) & 1, abort)) break;
                issue_v(j);
                ++n_issued;
            }
            if (*abort)
                for (int j = max(0, n_issued - kVStages); j < n_issued; ++j)
                    mbar_wait(bar(B_VFULL + j % kVStages), (j / kVStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Chunk j belongs to warpgroup h = j % 2: S_j goes to TMEM buffer j % 3,
        // P_j is read from that buffer, and every P_j V_j accumulates into O in
        // chunk order.  Order of issue: S_0 .. S_2, then whichever is ready:
        // S_ns (P_{ns-3} V_{ns-3}, which read its buffer, complete and K_ns
        // landed) or P_j V_j (P_j written, V_j landed).
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
            // chunk j < nchunks: a Shared chunk in the K / V rings; j >= nchunks: an
            // Unshared chunk in the U area (its K and V land together on B_UFULL)
            auto k_ready = [&](int j, bool block) -> bool {
                const uint32_t b = j < nchunks ? bar(B_KFULL + j % kKStages) : bar(B_UFULL);
                const uint32_t ph = j < nchunks ? (j / kKStages) & 1 : (j - nchunks) & 1;
                return block ? mbar_wait(b, ph, abort) : mbar_test(b, ph);
            };
            auto issue_s = [&](int j) {   // S_j = Q K_j^T into TMEM buffer j % 3
                fence_after_sync();
                const uint32_t kq = sb + kOffQ;
                const uint32_t kk = j < nchunks ? sb + kOffK + (j % kKStages) * kTile : sb + kOffU;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (uint32_t)(k >> 2) * kHalf + (uint32_t)(k & 3) * 32u;
                    umma_bf16(tmem + (uint32_t)(j % kSBufs) * 128u, umma_desc(kq + off, 16, 1024),
                              umma_desc(kk + off, 16, 1024), idS, k > 0);
                }
                umma_commit(bar(B_SFULL + j % kSBars));
                if (j < nchunks) umma_commit(bar(B_KEMPTY + j % kKStages));
            };
            bool ok = mbar_wait(bar(B_QFULL), 0, abort);
            int ns = 0;   // the next S to issue
            for (; ok && ns < min(nall, kSBufs); ++ns) {
                ok = k_ready(ns, true);
                if (ok) issue_s(ns);
            }
            uint32_t idle = 0;
            for (int j = 0; ok && j < nall;) {
                bool progress = false;
                if (ns < nall && mbar_test(bar(B_PVDONE + (ns - kSBufs) % kPBars), ((ns - kSBufs) / kPBars) & 1) &&
                    k_ready(ns, false)) {
                    issue_s(ns++);
                    progress = true;
                }
                const int sv = j % kVStages;
                const bool v_ready = j < nchunks ? mbar_test(bar(B_VFULL + sv), (j / kVStages) & 1)
                                                 : mbar_test(bar(B_UFULL), (j - nchunks) & 1);
                if (!(mbar_test(bar(B_PFULL + j % kPBars), (j / kPBars) & 1) && v_ready)) {
                    if (progress) {
                        idle = 0;
                    } else if (++idle >= kSpinLimit) {
                        *abort = 1;
                        ok = false;
                    } else if ((idle & 255) == 0 && *abort) {
                        ok = false;
                    }
                    continue;
                }
                idle = 0;
                fence_after_sync();
                const uint32_t kv = j < nchunks ? sb + kOffV + sv * kTile : sb + kOffU + kTile;
                const uint32_t pcol = (uint32_t)(j % kSBufs) * 128u;
#pragma unroll
                for (int k = 0; k < 8; ++k)   // P_j: 16 keys = 8 TMEM columns per MMA
                    umma_bf16_ts(tmem + kOCol, tmem + pcol + 8u * k, umma_desc(kv + (uint32_t)k * 2048u, kHalf, 1024),
                                 idPV, (k > 0 || j > 0) ? 1u : 0u);
                umma_commit(bar(B_PVDONE + j % kPBars));
                umma_commit(j < nchunks ? bar(B_VEMPTY + sv) : bar(B_UEMPTY));
                ++j;
            }
            // arrives once every MMA issued above has completed (TMEM final / free)
            umma_commit(bar(B_DONE));
            if (*abort) mbar_wait(bar(B_DONE), 0, nullptr);
        }
    } else if (warp < kGatherWarp) {
        // ------------------------------------------------------------ softmax
        // Warpgroup `half` owns the chunks j with j % 2 == half, whole rows: thread
        // `row` reads TMEM lane `row` of S_j's buffer and writes row `row` of P_j
        // over it.  Both warpgroups' P_j V_j add into the one O, so each row has
        // one reference maximum (shared memory), raised lazily -- only when a
        // chunk's max passes it by 2^8 -- by the warpgroup that sees the chunk;
        // the other warpgroup waits for that decision (B_DEC) before its next
        // chunk's P, and O is rescaled between P_{j-1} V_{j-1} and P_j V_j.
        // Each warpgroup keeps its own row sum l relative to the reference it
        // last used; at the end the two sums meet, and thread (row, half)
        // handles head-dim columns [64*half, 64*half + 64).
        const int half = (warp - 2) >> 2;
        const int row = 32 * (warp & 3) + lane;
        bool ok = true;
        if (!q_tma) {
            fence_async_smem();
            mbar_arrive(bar(B_QFULL));
        }

        const RowInfo ri = row_info(a, it, row);
        const float cscale = kLog2e * rsqrtf(128.f);
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t col0 = (uint32_t)(64 * half);
        float my_ref = -INFINITY, l = 0.f;   // the reference l is relative to; this warpgroup's row sum
        float *mref = reinterpret_cast<float *>(base + kOffMref);   // [128] the rows' shared references
        const Dims dm = a.dims;
        const bool live = ri.valid && ri.b < a.n_live[ri.r];
        // Unshared chunks: this row keeps columns [u_lo, u_lo + T) of the block-
        // diagonal U rows -- its beam's tokens -- where the token's slot is valid
        // (bit i of vmask; this step's own token when the beam is live)
        uint32_t vmask = 0;
        const int u_lo = ((it.row_begin + row) / dm.G - lb0) * T;
        if (final_item && live) {
            const int64_t beam_row = (int64_t)ri.r * dm.BW + ri.b;
            vmask = 1u << a.step;
            for (int i = 0; i < a.step; ++i) {
                const int sl = a.st.anc[beam_row * dm.S + i];
                if (sl >= 0 && sl < dm.BW) vmask |= 1u << i;
                else if (ri.hg == 0 && half == 0) set_status(a.status, XGR_DEV_INDEX);
            }
        }
        for (int j = half; ok && j < nall; j += 2) {
            const uint32_t s_col = (uint32_t)(j % kSBufs) * 128u;   // S_j's buffer
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + j % kSBars), (j / kSBars) & 1, abort));
            if (!ok) break;
            fence_after_sync();
            const int nvalid = n_keys - j * kBlockN;   // keys of the chunk inside the range
            const bool is_u = j >= nchunks;            // an Unshared chunk
            const int c0 = u_lo - kBlockN * (j - nchunks);   // (is_u) the row's first column in it
            // Masked chunks (an Unshared chunk: only this row's own tokens count;
            // the range's last chunk: keys past its end do not) keep the
            // columns of a 32-bit mask per 32-column piece
            const bool masked = is_u || nvalid < kBlockN;
            auto piece_mask = [&](int q2) -> uint32_t {
                if (is_u) {   // the row's valid tokens (vmask) start at column c0
                    const int off = c0 - 32 * q2;
                    return off >= 32 || off <= -32 ? 0u : off >= 0 ? vmask << off : vmask >> -off;
                }
                const int nv = nvalid - 32 * q2;
                return nv >= 32 ? ~0u : nv <= 0 ? 0u : (1u << nv) - 1u;
            };
            // the chunk's 128 scores in one TMEM read (P_j then overwrites them)
            float sv[128];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) tmem_ld32(tmem + lane_base + s_col + 32 * q2, sv + 32 * q2);
            tmem_wait_ld();
            if (masked) {
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const uint32_t pm = piece_mask(q2);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((pm >> e) & 1u)) sv[32 * q2 + e] = -INFINITY;
                }
            }
            // row maximum: eight chains of three-input maxima
            float mxp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxp[e] = fmaxf(sv[e], sv[8 + e]);
#pragma unroll
            for (int c = 16; c < 128; c += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) mxp[e] = fmax3(mxp[e], sv[c + e], sv[c + 8 + e]);
            const float mx = fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmax3(mxp[3], mxp[4], mxp[5]),
                                   fmaxf(mxp[6], mxp[7])) * cscale;
            // the rows' references as chunk j-1's warpgroup left them
            if (j > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DEC + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort));
            if (!ok) break;
            const float ref = mref[row];
            if (ref != my_ref) {   // raised by the other warpgroup: l follows (l is 0 while my_ref is -inf)
                l *= ex2(my_ref - ref);
                my_ref = ref;
            }
            const bool grow = mx > my_ref + 8.f;   // lazy: a new reference only when the max grew by 2^8
            const float alpha = grow ? ex2(my_ref - mx) : 1.f;
            if (grow) {
                my_ref = mx;
                mref[row] = mx;
            }
            mbar_arrive(bar(B_DEC + (j & 1)));   // (releases the reference for chunk j+1)
            // exponentials, row sum and P (bf16 pairs) into the first 64 columns of
            // the S buffer, from the scores already in registers (masked ones are
            // -inf; a row masked in every chunk so far has a -inf reference and P 0):
            // piece q's 16 P columns land on scores already read
            const float nm = my_ref == -INFINITY ? 0.f : -my_ref;
            // x = s * scale - m in packed pairs; sums in eight chains
            const float2 sc2 = make_float2(cscale, cscale), nm2 = make_float2(nm, nm);
            float sp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) sp[e] = 0.f;
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                float pw[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 x = ffma2(make_float2(sv[32 * q2 + 2 * e], sv[32 * q2 + 2 * e + 1]), sc2, nm2);
                    const float2 p = make_float2(ex2(x.x), ex2(x.y));
                    sp[(2 * e) & 7] += p.x;
                    sp[(2 * e + 1) & 7] += p.y;
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p.x, p.y);
                    pw[e] = __uint_as_float(*reinterpret_cast<uint32_t *>(&h2));
                }
                tmem_st16(tmem + lane_base + s_col + 16 * q2, pw);
            }
            if (__any_sync(0xffffffffu, grow && j > 0)) {
                // O *= alpha on the rows whose reference rose, once every product
                // of the old reference (up to P_{j-1} V_{j-1}) is in O and before
                // P_j V_j adds in
                ok = __all_sync(0xffffffffu,
                                mbar_wait(bar(B_PVDONE + (j - 1) % kPBars), ((j - 1) / kPBars) & 1, abort));
                if (!ok) break;
                fence_after_sync();
                const float f = grow ? alpha : 1.f;
#pragma unroll 1
                for (int q2 = 0; q2 < 4; ++q2) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + kOCol + q2 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= f;
                    tmem_st32(tmem + lane_base + kOCol + q2 * 32, o);
                }
            }
            l = l * alpha + (((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7])));
            tmem_wait_st();   // P_j (and a rescaled O) in TMEM before the MMA warp reads them
            fence_before_sync();
            mbar_arrive(bar(B_PFULL + j % kPBars));
        }
        // every MMA done: O is final, the S buffers free
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0, abort));
        if (ok) {
            fence_after_sync();
            // the warpgroups swap (reference, l): the larger reference is the row's
            // last, the one O is relative to; thread (row, half) then writes
            // head-dim columns [64*half, 64*half + 64) of O
            float2 *xl = reinterpret_cast<float2 *>(base + kOffV);   // [2][128]; V is consumed
            xl[half * 128 + row] = make_float2(my_ref, l);
            mbar_arrive(bar(B_XCH + half));
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_XCH + (half ^ 1)), 0, abort));
            const float2 other = xl[(half ^ 1) * 128 + row];
            const float m0 = half == 0 ? my_ref : other.x, l0 = half == 0 ? l : other.y;
            const float m1 = half == 0 ? other.x : my_ref, l1 = half == 0 ? other.y : l;
            const float M = fmaxf(m0, m1);
            // a sum relative to a -inf reference is 0 (no chunk of the row had a key)
            const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
            const float f1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
            const float l_row = l0 * f0 + l1 * f1;
            if (ok) {
#pragma unroll 1
                for (int q2 = 0; q2 < 2; ++q2) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + kOCol + col0 + 32 * q2, o);
                    tmem_wait_ld();
                    const uint32_t c0 = col0 + 32 * q2;
                    if (!final_item) {
                        if (live) {
                            float *dst = a.part.o + ((int64_t)it.slot * a.part.rows + ri.gid) * 128 + c0;
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *reinterpret_cast<float4 *>(dst + e) =
                                    make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
                        }
                    } else if (ri.valid) {
                        // final: O / l in bf16; dead rows 0
                        const float inv = live ? 1.f / l_row : 0.f;
                        uint4 *dst = reinterpret_cast<uint4 *>(a.out + ri.gid * 128 + c0);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t w4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float v0 = live ? o[8 * c + 2 * e] * inv : 0.f;
                                const float v1 = live ? o[8 * c + 2 * e + 1] * inv : 0.f;
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                                w4[e] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
                if (half == 0) {
                    if (!final_item) {
                        if (live) a.part.ml[(int64_t)it.slot * a.part.rows + ri.gid] = make_float2(M, l_row);
                    } else if (ri.valid) {   // LSE = m + log2(l) in natural log; dead rows -inf
                        a.lse[ri.gid] = live ? (M + __log2f(l_row)) * kLn2 : -INFINITY;
                    }
                }
            }
        }
    } else if (n_u > 0) {
        // ------------------------------------------------------------ gather
        {
            // ---- Unshared stage: gather the tile's beams' own k / v rows of steps
            // 0..s into the U area, one 128-row chunk at a time (row u: token u % T
            // of tile beam u / T), in the canonical swizzled layout; rows of dead
            // beams, bad slots and the tail are zero.  This step's rows are also
            // appended to the pool at slot (s, b).
            const int gl = lane;
            const Dims dm = a.dims;
            const int s_now = a.step;
            const int64_t pool_step = (int64_t)a.Bcap * dm.BW * dm.Hkv * 128;
            for (int q = 0; q < n_u; ++q) {
                if (q > 0 && !mbar_wait(bar(B_UEMPTY), (q - 1) & 1, abort)) break;
                // this lane's rows u = gl + k * kGatherLanes: their request and beam,
                // then every index they need, then the copies -- each stage's loads
                // all in flight together
                constexpr int kRowsPerLane = (kBlockN + kGatherLanes - 1) / kGatherLanes;
                int rr[kRowsPerLane], bb[kRowsPerLane], ii[kRowsPerLane];
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    const int u = gl + k * kGatherLanes, ug = kBlockN * q + u, lb = ug / T;
                    ii[k] = ug % T;
                    rr[k] = -1;
                    bb[k] = -1;
                    if (u < kBlockN && lb < nbeam) {
                        const int lbs = lb0 + lb;   // beam index within the segment's rows / G
                        bb[k] = lbs % a.nb;
                        rr[k] = it.n_members == 1 ? it.r0 : a.members[it.member_off + lbs / a.nb];
                    }
                }
                int nl[kRowsPerLane], sl[kRowsPerLane];
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    nl[k] = rr[k] >= 0 ? a.n_live[rr[k]] : 0;
                    sl[k] = (rr[k] >= 0 && ii[k] < s_now)
                                ? a.st.anc[((int64_t)rr[k] * dm.BW + bb[k]) * dm.S + ii[k]] : -1;
                }
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    const int u = gl + k * kGatherLanes;
                    if (u >= kBlockN) continue;
                    const __nv_bfloat16 *sk = nullptr, *sv = nullptr;
                    if (rr[k] >= 0 && bb[k] < nl[k]) {
                        const int64_t brow = (int64_t)rr[k] * dm.BW + bb[k];
                        if (ii[k] == s_now) {
                            sk = a.k_new + (brow * dm.Hkv + it.g) * 128;
                            sv = a.v_new + (brow * dm.Hkv + it.g) * 128;
                        } else if (sl[k] >= 0 && sl[k] < dm.BW) {
                            const int64_t prow = (brow - bb[k] + sl[k]) * dm.Hkv + it.g;
                            sk = a.pool_k + ii[k] * pool_step + prow * 128;
                            sv = a.pool_v + ii[k] * pool_step + prow * 128;
                        }
                    }
                    const uint32_t dk = sb + kOffU, dv = sb + kOffU + kTile;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        if (sk) {
                            cp_async16(dk + sw128_off(u, c), sk + 8 * c);
                            cp_async16(dv + sw128_off(u, c), sv + 8 * c);
                        } else {
                            *reinterpret_cast<uint4 *>(base + kOffU + sw128_off(u, c)) = make_uint4(0, 0, 0, 0);
                            *reinterpret_cast<uint4 *>(base + kOffU + kTile + sw128_off(u, c)) =
                                make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                cp_async_wait_all();
                // this step's k / v of the gathered live beams -> pool slot (s, b)
#pragma unroll
                for (int k = 0; k < kRowsPerLane; ++k) {
                    const int u = gl + k * kGatherLanes;
                    if (u >= kBlockN || rr[k] < 0 || ii[k] != s_now || bb[k] >= nl[k]) continue;
                    const int64_t orow = ((int64_t)rr[k] * dm.BW + bb[k]) * dm.Hkv + it.g;
                    uint4 *pk = reinterpret_cast<uint4 *>(a.pool_k + s_now * pool_step + orow * 128);
                    uint4 *pv = reinterpret_cast<uint4 *>(a.pool_v + s_now * pool_step + orow * 128);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        pk[c] = *reinterpret_cast<const uint4 *>(base + kOffU + sw128_off(u, c));
                        pv[c] = *reinterpret_cast<const uint4 *>(base + kOffU + kTile + sw128_off(u, c));
                    }
                }
                fence_async_smem();   // the gathered rows are visible to the tensor cores
                mbar_arrive(bar(B_UFULL));
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

}  // namespace one_o

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return nullptr;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    return encode;
}

cudaError_t make_kv_tensor_map(CUtensorMap *map, const void *base, int64_t rows) {
    auto encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_q_tensor_map(CUtensorMap *map, const void *q, int64_t beam_rows, int Hq, int G) {
    auto encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {128, (cuuint64_t)Hq, (cuuint64_t)beam_rows};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)Hq * 128 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(128 / G)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

template <class K>
cudaError_t launch_tc(K kernel, bool &attr, const CUtensorMap &tmk, const CUtensorMap &tmv, const CUtensorMap &tmq,
                      const TcArgs &a, int n_items, cudaStream_t st) {
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return e;
        if (fa.maxThreadsPerBlock < kTcThreads) {
            debug_log("attn_tc: %d registers/thread allow only %d threads per block", fa.numRegs,
                      fa.maxThreadsPerBlock);
            return cudaErrorLaunchOutOfResources;
        }
        attr = true;
    }
    return launch_pdl(kernel, dim3(n_items), dim3(kTcThreads), kSmemBytes, st, tmk, tmv, tmq, a);
}

}  // namespace

cudaError_t launch_attn_tc(const CUtensorMap &tmk, const CUtensorMap &tmv, const CUtensorMap &tmq,
                           const TcArgs &a, int n_items, cudaStream_t st) {
    if (n_items <= 0) return cudaSuccess;
    if (a.step + 1 > kMaxSteps) return cudaErrorInvalidValue;   // Unshared tokens of a beam
    static bool attr_two = false, attr_one = false;
    return a.shared_o ? launch_tc(one_o::attn_tc_one_o_kernel, attr_one, tmk, tmv, tmq, a, n_items, st)
                      : launch_tc(attn_tc_kernel, attr_two, tmk, tmv, tmq, a, n_items, st);
}

}  // namespace xgr

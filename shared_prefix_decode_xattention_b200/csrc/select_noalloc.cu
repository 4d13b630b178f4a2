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
// It runs the very same selection kernels as xgr_beam_select (without the
// rewiring).  Their scratch (each beam's row log-sum-exp, candidate count and
// head of best keys, each request's ticket and key buffer) lives in one
// file-scope device array of
// kScratchBytes; every GPU that loads the library holds that array until the
// process exits.  All
// calls share it, so calls that overlap on the GPU (two streams, two threads)
// race on it and must be serialised by the caller.  The array keeps the last
// call's contents; everything a call reads from it is written by that same
// call first.  Device faults (NaN scores, out-of-vocabulary mask tokens) are
// skipped as in the context path but not reported -- use the context path
// (xgr_device_status) to diagnose them.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace xgr {

namespace {

constexpr size_t kScratchBytes = 8u << 20;   // 8 MiB: status word + selection scratch
constexpr size_t kStatusBytes = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

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
        top_k > 1024 || vocab < 1 || (int64_t)beam_width * vocab >= (1ll << 32))
        return XGR_ERR_SHAPE;
    if (vocab > kSelectMaxVocab) return XGR_ERR_UNIMPLEMENTED;
    // what the fixed array leaves after the per-row scratch goes to the key
    // buffer (8 bytes a CSR entry)
    const size_t fixed = kStatusBytes + select_scratch_bytes(n_requests, beam_width, 0) + 1024;
    if (fixed >= kScratchBytes) return XGR_ERR_CAPACITY;
    const int64_t key_cap = (int64_t)((kScratchBytes - fixed) / ((size_t)n_requests * 8)) & ~31ll;
    const int64_t need = std::max<int64_t>({(int64_t)vocab, 8ll * beam_width, 4096});
    if (key_cap < need ||
        kStatusBytes + select_scratch_bytes(n_requests, beam_width, key_cap) > kScratchBytes)
        return XGR_ERR_CAPACITY;   // beyond the fixed 8 MiB scratch
    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return XGR_ERR_CUDA;
    uint8_t *sc = static_cast<uint8_t *>(scratch);
    SelectArgs a{};
    a.cum = d_cum;
    a.n_live = d_n_live;
    a.status = reinterpret_cast<int32_t *>(sc);   // faults are skipped, not reported here
    a.rewire = 0;
    a.dims = Dims{n_requests, beam_width, top_k, 1, 1, 1, 128, vocab, 1};
    a.step = dense ? 0 : 1;
    a.logits = flags == XGR_SCORES_LOGITS;
    a.scores = d_scores;
    a.dense = dense;
    a.prep_early = 0;   // nothing is known about the kernel before
    a.mask_kind = dense ? XGR_MASK_DENSE : XGR_MASK_CSR;
    a.bits = d_bits;
    a.row_ptr = d_row_ptr;
    a.cols = d_cols;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&a.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return XGR_ERR_CUDA;
    select_scratch_carve(sc + kStatusBytes, n_requests, beam_width, key_cap, a);
    a.parent = d_parent;
    a.token = d_token;
    a.cum_out = d_cum_out;
    a.n_out = d_n_out;
    if (launch_beam_select(a, (cudaStream_t)stream) != cudaSuccess) return XGR_ERR_CUDA;
    return XGR_OK;
}

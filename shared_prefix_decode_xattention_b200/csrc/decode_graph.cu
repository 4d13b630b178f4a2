// decode_graph.cu -- a whole decode of one or more request groups as one CUDA
// graph (declared in include/xgr.h).  xGR page, 2.3 xSchedule, "Graph-based
// execution" and "Dynamic batching and multi-stream": the decode's kernels are
// captured once and dispatched in one go, each request group's chain on a
// stream of its own so that independent groups overlap.  Host code only: the
// graph holds exactly the kernels the step calls launch.
#include <new>
#include <vector>

#include "common.cuh"

struct xgr_decode_graph {
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    int32_t n_kernels = 0;
};

namespace {

constexpr int kMaxGroups = 64;

// one group's decode on stream st, through the public calls
xgr_status enqueue_group(const xgr_decode_group &g, int32_t steps, cudaStream_t st) {
    const xgr_stream_t s = (xgr_stream_t)st;
    xgr_status e = xgr_begin(g.ctx, g.n_requests, s);
    for (int32_t k = 0; e == XGR_OK && k < steps; ++k) {
        xgr_mask m;
        e = xgr_build_mask(g.ctx, k, &m, s);
        if (e == XGR_OK) e = xgr_decode_step(g.ctx, k, g.d_q[k], g.d_k_new[k], g.d_v_new[k], g.d_out, g.d_lse, s);
        if (e == XGR_OK)
            e = xgr_beam_select(g.ctx, k, g.d_scores[k], g.score_flags, &m, g.d_parent, g.d_token, g.d_cum,
                                g.d_n_out, s);
    }
    return e;
}

// streams and events of the fork / join around the groups' chains
struct Fork {
    cudaStream_t origin = nullptr;
    std::vector<cudaStream_t> st;
    std::vector<cudaEvent_t> ev;   // [0]: fork; [1 + g]: group g done
    bool ok = true;
    explicit Fork(int n) : st(n, nullptr), ev(n + 1, nullptr) {
        ok = cudaStreamCreateWithFlags(&origin, cudaStreamNonBlocking) == cudaSuccess;
        for (auto &s : st) ok = ok && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess;
        for (auto &e : ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    }
    ~Fork() {
        for (auto e : ev)
            if (e) cudaEventDestroy(e);
        for (auto s : st)
            if (s) cudaStreamDestroy(s);
        if (origin) cudaStreamDestroy(origin);
    }
    xgr_status enqueue(const xgr_decode_group *groups, int32_t steps) {
        if (cudaEventRecord(ev[0], origin) != cudaSuccess) return XGR_ERR_CUDA;
        for (size_t g = 0; g < st.size(); ++g) {
            if (cudaStreamWaitEvent(st[g], ev[0], 0) != cudaSuccess) return XGR_ERR_CUDA;
            const xgr_status e = enqueue_group(groups[g], steps, st[g]);
            if (e != XGR_OK) return e;
            if (cudaEventRecord(ev[1 + g], st[g]) != cudaSuccess ||
                cudaStreamWaitEvent(origin, ev[1 + g], 0) != cudaSuccess)
                return XGR_ERR_CUDA;
        }
        return XGR_OK;
    }
};

int32_t count_kernels(cudaGraph_t graph) {
    size_t n = 0;
    if (cudaGraphGetNodes(graph, nullptr, &n) != cudaSuccess) return -1;
    std::vector<cudaGraphNode_t> nodes(n);
    if (n && cudaGraphGetNodes(graph, nodes.data(), &n) != cudaSuccess) return -1;
    int32_t k = 0;
    for (auto nd : nodes) {
        cudaGraphNodeType t;
        if (cudaGraphNodeGetType(nd, &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++k;
    }
    return k;
}

}  // namespace

extern "C" {

xgr_status xgr_decode_graph_create(const xgr_decode_group *groups, int32_t n_groups, int32_t steps,
                                   xgr_decode_graph **out) {
    if (!out) return XGR_ERR_ARG;
    *out = nullptr;
    if (!groups || n_groups < 1 || n_groups > kMaxGroups || steps < 1) return XGR_ERR_ARG;
    for (int32_t g = 0; g < n_groups; ++g) {
        const xgr_decode_group &x = groups[g];
        if (!x.ctx || !x.d_q || !x.d_k_new || !x.d_v_new || !x.d_scores) return XGR_ERR_ARG;
        for (int32_t h = 0; h < g; ++h)
            if (groups[h].ctx == x.ctx) return XGR_ERR_ARG;   // one context's state per chain
    }
    Fork f(n_groups);
    if (!f.ok) return XGR_ERR_CUDA;
    // eager decode: plans, launch attributes and tensor maps, and the calls'
    // own argument checks, all before the capture
    xgr_status e = f.enqueue(groups, steps);
    if (e != XGR_OK) return e;
    if (cudaStreamSynchronize(f.origin) != cudaSuccess) return XGR_ERR_CUDA;
    if (cudaStreamBeginCapture(f.origin, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return XGR_ERR_CUDA;
    e = f.enqueue(groups, steps);
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(f.origin, &graph);
    if (e != XGR_OK || ce != cudaSuccess || !graph) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();   // (an invalidated capture leaves its error behind)
        return e != XGR_OK ? e : XGR_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    if (cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
        cudaGraphDestroy(graph);
        return XGR_ERR_CUDA;
    }
    xgr_decode_graph *dg = new (std::nothrow) xgr_decode_graph;
    if (!dg) {
        cudaGraphExecDestroy(exec);
        cudaGraphDestroy(graph);
        return XGR_ERR_CAPACITY;
    }
    dg->graph = graph;
    dg->exec = exec;
    dg->n_kernels = count_kernels(graph);
    *out = dg;
    return XGR_OK;
}

xgr_status xgr_decode_graph_launch(xgr_decode_graph *g, xgr_stream_t stream) {
    if (!g) return XGR_ERR_ARG;
    return cudaGraphLaunch(g->exec, (cudaStream_t)stream) == cudaSuccess ? XGR_OK : XGR_ERR_CUDA;
}

xgr_status xgr_decode_graph_kernels(const xgr_decode_graph *g, int32_t *n_kernels) {
    if (!g || !n_kernels) return XGR_ERR_ARG;
    *n_kernels = g->n_kernels;
    return XGR_OK;
}

xgr_status xgr_decode_graph_destroy(xgr_decode_graph *g) {
    if (!g) return XGR_ERR_ARG;
    cudaGraphExecDestroy(g->exec);
    cudaGraphDestroy(g->graph);
    delete g;
    return XGR_OK;
}

}  // extern "C"

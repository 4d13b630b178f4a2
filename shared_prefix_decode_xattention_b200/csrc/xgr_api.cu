// xgr_api.cu -- the C ABI of libxgr.so (declared in include/xgr.h): argument
// validation, the carving of the caller's workspace, the host-side trie
// build, the prompt KV store, the Shared-stage work planner and the launches.
#include <algorithm>
#include <cstring>
#include <new>
#include <numeric>
#include <vector>

#include "common.cuh"
#include "kernels.h"

using namespace xgr;

namespace {

constexpr size_t kAlign = 256;
// the largest pre-generated table of per-node bitsets (dense masks of step 1)
constexpr size_t kNodeBitsMax = size_t(256) << 20;
// a level takes dense masks when its nodes have at least V / 256 children on
// average (many candidates per beam) and at most kNodeBitsStride children each
// (the selection compacts a row's bits into a per-warp list of that size)
constexpr int kNodeBitsStride = 2048;
constexpr int kMinChunk = 256;     // fewest keys per split-K work item
// the separate merge kernel that split items need, in key units of the
// tensor-core loop (one more dependent launch plus a few round trips)
constexpr double kMergeKeys = 768.0;
// most key chunks of any tensor-core item of a launch that runs the one-O
// variant of the kernel
constexpr int64_t kSharedOChunks = 12;

size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

int fanout_cap(const xgr_config &c) { return c.max_fanout > 0 ? c.max_fanout : c.vocab; }

int64_t partial_rows(const xgr_config &c) {
    return (int64_t)c.max_requests * c.beam_width * c.n_q_heads;
}

int partial_slots(const xgr_config &c) {
    if (c.max_partials > 0) return c.max_partials;
    const double per_slot = (double)partial_rows(c) * c.head_dim * 4.0;
    int s = (int)std::min(8.0, std::max(2.0, (1ull << 30) / per_slot));
    return s;
}

int64_t plan_item_cap(const xgr_config &c) {
    const int G = c.n_q_heads / c.n_kv_heads;
    const int64_t rows = 2ll * c.max_requests * c.beam_width * G;
    const int64_t tiles = (rows + kSmallRows - 1) / kSmallRows + c.max_shared + c.max_requests;
    return tiles * c.n_kv_heads + 8192;
}

struct Layout {
    size_t status, n_live, cum, node, anc, seq;
    size_t kstore, vstore, pool_k, pool_v;
    size_t trie_ptr, trie_tok, root_bits, node_bits;
    size_t node_bits_bytes;    // room for the pre-generated per-node bitsets of level 1
    int64_t trie_level_cap;    // ints per level in each of trie_ptr / trie_tok
    size_t mask_sync;
    size_t select_scratch;
    int64_t key_cap;             // selection keys per request
    size_t part_o, part_ml;
    int slots;
    size_t plan_items[2], plan_members[2], plan_nslots[2];
    size_t req_seg;              // [B][4] each request's prompt and suffix ranges (per-beam path)
    int64_t item_cap, member_cap;
    size_t total;
};

void make_layout(const xgr_config &c, Layout &L) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up(bytes);
        return o;
    };
    const int64_t B = c.max_requests, BW = c.beam_width, S = c.steps;
    const int64_t D = c.head_dim, Hkv = c.n_kv_heads;
    L.status = take(16);
    L.n_live = take(4 * B);
    L.cum = take(4 * B * BW);
    L.node = take(4 * B * BW);
    L.anc = take(4 * B * BW * S);
    L.seq = take(4 * B * BW * S);
    L.kstore = take(2 * Hkv * c.kv_tokens * D);
    L.vstore = take(2 * Hkv * c.kv_tokens * D);
    L.pool_k = take(2 * S * B * BW * Hkv * D);
    L.pool_v = take(2 * S * B * BW * Hkv * D);
    if (c.vocab > 0) {
        L.trie_level_cap = c.max_items + 2;
        L.trie_ptr = take(4 * S * L.trie_level_cap);
        L.trie_tok = take(4 * S * L.trie_level_cap);
        L.root_bits = take(4 * ((c.vocab + 31) / 32));
        // level 1 has at most min(V, items) nodes; its dense table is kept only
        // when it fits kNodeBitsMax
        const size_t nb = (size_t)std::min<int64_t>(c.vocab, c.max_items) * (size_t)((c.vocab + 31) / 32) * 4;
        L.node_bits_bytes = (c.steps >= 2 && nb <= kNodeBitsMax) ? nb : 0;
        L.node_bits = L.node_bits_bytes ? take(L.node_bits_bytes) : 0;

        L.mask_sync = take(8 * (B + 1));   // look-back words, then the two ticket words
        L.key_cap = BW * (int64_t)fanout_cap(c);
        L.select_scratch = take(select_scratch_bytes((int)B, (int)BW, L.key_cap));
    } else {
        L.trie_level_cap = 0;
        L.trie_ptr = L.trie_tok = L.root_bits = L.mask_sync = 0;
        L.node_bits = L.node_bits_bytes = 0;
        L.select_scratch = 0;
        L.key_cap = 0;
    }
    L.slots = partial_slots(c);
    L.part_o = take(4 * (size_t)L.slots * partial_rows(c) * D);
    L.part_ml = take(8 * (size_t)L.slots * partial_rows(c));
    L.item_cap = plan_item_cap(c);
    L.member_cap = 2 * B + 16;
    for (int p = 0; p < 2; ++p) {
        L.plan_items[p] = take(sizeof(WorkItem) * L.item_cap);
        L.plan_members[p] = take(4 * L.member_cap);
        L.plan_nslots[p] = take(4 * B);
    }
    L.req_seg = take(16 * B);
    L.total = off;
}

xgr_status check_config(const xgr_config *c) {
    if (!c) return XGR_ERR_ARG;
    if (c->max_requests < 1 || c->max_shared < 0 || c->kv_tokens < 0) return XGR_ERR_SHAPE;
    if (c->kv_tokens >= (1ll << 31)) return XGR_ERR_SHAPE;
    if (c->n_kv_heads >= 1 && (int64_t)c->n_kv_heads * c->kv_tokens >= (1ll << 31)) return XGR_ERR_SHAPE;
    if (c->beam_width < 1 || c->beam_width > 1024) return XGR_ERR_SHAPE;
    if (c->steps < 1 || c->steps > kMaxSteps) return XGR_ERR_SHAPE;
    if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads) return XGR_ERR_SHAPE;
    const int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return XGR_ERR_UNIMPLEMENTED;
    if (c->head_dim != 64 && c->head_dim != 128) return XGR_ERR_UNIMPLEMENTED;
    if (c->vocab < 0 || c->max_items < 0 || c->max_fanout < 0 || c->max_partials < 0)
        return XGR_ERR_SHAPE;
    if (c->vocab > 0) {
        if (c->top_k < c->beam_width || c->top_k > 1024) return XGR_ERR_SHAPE;
        if ((int64_t)c->beam_width * c->vocab >= (1ll << 32)) return XGR_ERR_SHAPE;
        if (c->max_items < 1) return XGR_ERR_SHAPE;
        if (c->vocab > kSelectMaxVocab) return XGR_ERR_UNIMPLEMENTED;
    }
    if ((int64_t)c->max_requests * c->beam_width * c->n_q_heads >= (1ll << 31)) return XGR_ERR_SHAPE;
    return XGR_OK;
}

bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

struct xgr_ctx {
    xgr_config cfg;
    Layout L;
    uint8_t *ws = nullptr;
    int device = 0, num_sms = 148;
    Dims dims;
    BeamState st;
    TrieView trie;
    bool has_trie = false;
    int level_fanout[kMaxSteps] = {};   // most children of one node of each trie level
    bool level_bits[kMaxSteps] = {};    // the level's per-node bitsets are pre-generated
    // prompt KV store bookkeeping (host)
    int64_t kv_used = 0;
    std::vector<int64_t> sid_off, sid_len;
    std::vector<int32_t> req_sid;
    std::vector<int64_t> suf_off, suf_len;
    bool plan_dirty = true;
    int planned_B = -1;
    int n_small[2] = {0, 0};   // small-row work items of each plan (then n_tc[] tensor-core ones)
    int n_tc[2] = {0, 0};
    int n_unfused[2] = {0, 0};   // requests the merge kernel still has to finish
    int tc_shared[2] = {0, 0};   // the tensor-core launch takes the one-O variant (short items)
    bool has_tc = false;       // tensor-core Shared stage available (D = 128, tensor maps built)
    CUtensorMap tmk, tmv;
    CUtensorMap tmq;             // Q tensor map of the last decode step, re-encoded when q or B changes
    const void *tmq_ptr = nullptr;
    int64_t tmq_rows = -1;
    // the last beam-state-writing or attention launch of this context: the
    // attention of step attn_step on attn_stream (-1: something else)
    int attn_step = -1;
    cudaStream_t attn_stream = nullptr;
    // decode state
    bool begun = false;
    int cur_step = 0;

    template <class T>
    T *at(size_t off) const { return reinterpret_cast<T *>(ws + off); }
};

namespace {

Partials partials_of(const xgr_ctx *c) {
    Partials p;
    p.o = c->at<float>(c->L.part_o);
    p.ml = c->at<float2>(c->L.part_ml);
    p.rows = partial_rows(c->cfg);
    return p;
}

// ---- Shared-stage plan: KV segments x kv heads x row tiles x key splits.
// plan 0: one live beam per request (step 0); plan 1: BW beams per request.
xgr_status build_plan(xgr_ctx *c, int which, int B) {
    const xgr_config &cf = c->cfg;
    const int nb = (which == 0) ? 1 : cf.beam_width;
    const int G = cf.n_q_heads / cf.n_kv_heads;
    struct Seg {
        int64_t off, len;
        std::vector<int> members;
    };
    std::vector<Seg> segs;
    std::vector<int> nseg(B, 0);
    for (int sid = 0; sid < cf.max_shared; ++sid) {
        if (c->sid_len[sid] <= 0) continue;
        Seg sg{c->sid_off[sid], c->sid_len[sid], {}};
        for (int r = 0; r < B; ++r)
            if (c->req_sid[r] == sid) sg.members.push_back(r);
        if (!sg.members.empty()) segs.push_back(std::move(sg));
    }
    for (int r = 0; r < B; ++r)
        if (c->suf_len[r] > 0) segs.push_back(Seg{c->suf_off[r], c->suf_len[r], {r}});
    for (auto &sg : segs)
        for (int r : sg.members) nseg[r]++;

    // kind of every segment: tensor-core tiles of 128 rows whenever D = 128
    // (few rows waste tensor work, but the loop still streams K/V faster than
    // the small-row kernel's scalar dot products), else the small-row kernel
    auto rows_of = [&](const Seg &sg) { return (int64_t)sg.members.size() * nb * G; };
    auto is_tc = [&](const Seg &sg) { return c->has_tc && rows_of(sg) > 0; };
    // split factor per kind: the fewest waves x keys per item (+ a fixed
    // per-item overhead in key units), over the resident CTAs of the GPU
    // A tensor-core segment left whole finishes its requests itself; splitting
    // it adds the merge kernel, unless some segment needs that kernel anyway.
    bool merge_anyway = false;
    for (auto &sg : segs) {
        if (!is_tc(sg)) merge_anyway = true;
        for (int r : sg.members) merge_anyway |= nseg[r] > 1;
    }
    auto pick_split = [&](bool tc) {
        int64_t base = 0, keys = 0, nseg_k = 0;
        for (auto &sg : segs) {
            if (is_tc(sg) != tc) continue;
            const int64_t R = tc ? kTcRows : kSmallRows;
            base += (rows_of(sg) + R - 1) / R * cf.n_kv_heads;
            keys += sg.len;
            ++nseg_k;
        }
        if (!nseg_k) return (int64_t)1;
        const double L = (double)keys / nseg_k;
        const int64_t cap = tc ? c->num_sms : 2ll * c->num_sms;
        const double over = tc ? 384.0 : 128.0;
        const double merge = (tc && !merge_anyway) ? kMergeKeys : 0.0;
        int64_t best = 1;
        double best_cost = 1e300;
        for (int64_t f = 1; f <= c->L.slots; ++f) {
            if (f > 1 && L / f < kMinChunk) break;
            const double waves = (double)((base * f + cap - 1) / cap);
            const double cost = waves * (L / f + over) + (f > 1 ? merge : 0.0);
            if (cost < best_cost * 0.999) {
                best_cost = cost;
                best = f;
            }
        }
        return best;
    };
    const int64_t f_tc = pick_split(true), f_small = pick_split(false);
    // Segments of very different lengths (a shared prefix beside its members'
    // private suffixes): the common split, sized by the average segment, leaves
    // the long ones as the launch's tail.  Where the merge kernel runs anyway, a
    // tensor-core segment longer than twice t_keys -- the average key load per
    // SM, or the common split's range when larger -- is split into items of at
    // most t_keys keys (measured on the prefix-shared workload: batches of one
    // 8192-token prefix and 16 suffixes 0.393 -> 0.225 ms per four; segments
    // only 1.4 x t_keys long measured slower split).
    int64_t t_keys = 0;
    if (merge_anyway) {
        int64_t work = 0, keys = 0, n = 0;
        for (auto &sg : segs) {
            if (!is_tc(sg)) continue;
            work += (rows_of(sg) + kTcRows - 1) / kTcRows * cf.n_kv_heads * sg.len;
            keys += sg.len;
            ++n;
        }
        if (n) {
            const int64_t per_sm = (work + c->num_sms - 1) / c->num_sms;
            const int64_t common = (keys / n + f_tc - 1) / f_tc;
            t_keys = (std::max<int64_t>({per_sm, common, kMinChunk}) + 127) / 128 * 128;
        }
    }

    std::vector<WorkItem> items_small, items_tc;
    std::vector<int32_t> members;
    std::vector<int32_t> nslots(B, 0);
    std::vector<char> fused(B, 0);
    for (auto &sg : segs) {
        const bool tc = is_tc(sg);
        const int64_t R = tc ? kTcRows : kSmallRows;
        const int64_t rows = rows_of(sg);
        const int64_t tiles = (rows + R - 1) / R;
        int max_seg = 1;
        for (int r : sg.members) max_seg = std::max(max_seg, nseg[r]);
        const int64_t slot_cap = std::max(1, c->L.slots / max_seg);
        const bool long_seg = tc && t_keys > 0 && sg.len > 2 * t_keys;
        const int64_t want = long_seg ? std::max<int64_t>(f_tc, (sg.len + t_keys - 1) / t_keys)
                                      : (tc ? f_tc : f_small);
        int64_t splits = std::min<int64_t>({want, slot_cap, (sg.len + kMinChunk - 1) / kMinChunk});
        splits = std::max<int64_t>(1, splits);
        int64_t chunk = (sg.len + splits - 1) / splits;
        chunk = (chunk + 127) / 128 * 128;
        splits = (sg.len + chunk - 1) / chunk;
        int slot0 = 0;
        for (int r : sg.members) slot0 = std::max(slot0, nslots[r]);
        if (slot0 + splits > c->L.slots) return XGR_ERR_CAPACITY;
        const int member_off = (int)members.size();
        for (int r : sg.members) members.push_back(r);
        auto &dst = tc ? items_tc : items_small;
        // a final item runs the Unshared and Merging stages itself: no split and
        // no other segment for any of its requests
        const bool final_seg = tc && splits == 1 && max_seg == 1;
        if (final_seg)
            for (int r : sg.members) fused[r] = 1;
        for (int g = 0; g < cf.n_kv_heads; ++g)
            for (int64_t sp = 0; sp < splits; ++sp)
                for (int64_t t = 0; t < tiles; ++t) {
                    WorkItem it{};
                    it.kv_off = (int32_t)sg.off;
                    it.key_begin = (int32_t)(sp * chunk);
                    it.key_end = (int32_t)std::min<int64_t>(sg.len, (sp + 1) * chunk);
                    it.g = g;
                    it.member_off = member_off;
                    it.n_members = (int32_t)sg.members.size();
                    it.row_begin = (int32_t)(t * R);
                    it.n_rows = (int32_t)std::min<int64_t>(R, rows - t * R);
                    it.slot = (int32_t)(slot0 + sp);
                    it.flags = (final_seg ? 1 : 0) | (sg.members.size() == 1 ? 2 : 0);
                    it.r0 = sg.members[0];
                    dst.push_back(it);
                }
        for (int r : sg.members) nslots[r] = (int32_t)(slot0 + splits);
    }
    int unfused = 0;
    for (int r = 0; r < B; ++r) {
        if (fused[r]) nslots[r] = -1;   // the merge kernel skips this request
        else ++unfused;
    }
    // One live beam per request (plan 0): when the tensor-core items finish every
    // request, zero-fill items in the same launch write the other beams' rows on
    // the SMs the attention leaves idle, so no merge kernel runs.
    bool dead_rows = nb == cf.beam_width;   // plan 1: the items' tiles cover every beam
    if (!dead_rows && unfused == 0 && !items_tc.empty()) {
        const int64_t dead = (int64_t)B * (cf.beam_width - 1);
        const int64_t idle = std::max<int64_t>(1, (int64_t)c->num_sms - (int64_t)items_tc.size() - B);
        const int zb = (int)std::max<int64_t>(8, (dead + idle - 1) / idle);   // beams per zero item
        const int64_t n_zero = (int64_t)B * ((cf.beam_width - 1 + zb - 1) / zb);
        if ((int64_t)(items_small.size() + items_tc.size()) + n_zero <= c->L.item_cap) {
            for (int r = 0; r < B; ++r)
                for (int b0 = 1; b0 < cf.beam_width; b0 += zb) {
                    WorkItem it{};
                    it.r0 = r;
                    it.row_begin = b0;
                    it.n_rows = std::min(zb, cf.beam_width - b0);
                    it.flags = 4;
                    items_tc.push_back(it);
                }
            dead_rows = true;
        }
    }
    if (!dead_rows && unfused == 0) unfused = 1;   // the merge kernel writes the dead rows
    std::vector<WorkItem> items(items_small);
    items.insert(items.end(), items_tc.begin(), items_tc.end());
    if ((int64_t)items.size() > c->L.item_cap || (int64_t)members.size() > c->L.member_cap)
        return XGR_ERR_CAPACITY;
    if (!items.empty() &&
        cudaMemcpy(c->at<WorkItem>(c->L.plan_items[which]), items.data(),
                   items.size() * sizeof(WorkItem), cudaMemcpyHostToDevice) != cudaSuccess)
        return XGR_ERR_CUDA;
    if (!members.empty() &&
        cudaMemcpy(c->at<int32_t>(c->L.plan_members[which]), members.data(),
                   members.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
        return XGR_ERR_CUDA;
    if (cudaMemcpy(c->at<int32_t>(c->L.plan_nslots[which]), nslots.data(), (size_t)B * 4,
                   cudaMemcpyHostToDevice) != cudaSuccess)
        return XGR_ERR_CUDA;
    c->n_small[which] = (int)items_small.size();
    c->n_tc[which] = (int)items_tc.size();
    // Launches of short items only (few key chunks each) run the one-O variant
    // of the tensor-core kernel (three S buffers: the tensor pipe does not
    // drain between chunks); a launch with any long item keeps an O per
    // softmax warpgroup, whose warpgroups never wait for each other (measured:
    // 8-chunk items faster with one O, 16- to 128-chunk items slower).
    {
        int64_t longest = 0, n = 0;
        for (const WorkItem &it : items_tc)
            if (!(it.flags & 4)) {
                longest = std::max<int64_t>(longest, (it.key_end - it.key_begin + 127) / 128);
                ++n;
            }
        c->tc_shared[which] = n > 0 && longest <= kSharedOChunks;
    }
    c->n_unfused[which] = unfused;
    return XGR_OK;
}

}  // namespace

extern "C" {

const char *xgr_status_string(xgr_status s) {
    switch (s) {
        case XGR_OK: return "ok";
        case XGR_ERR_ARG: return "invalid argument (null/misaligned pointer, unknown flag)";
        case XGR_ERR_SHAPE: return "size inconsistent with the configuration";
        case XGR_ERR_CAPACITY: return "capacity fixed at create exceeded";
        case XGR_ERR_STATE: return "call out of order";
        case XGR_ERR_CUDA: return "CUDA runtime error";
        case XGR_ERR_DEVICE: return "device status word set (index, NaN, mask or capacity fault)";
        case XGR_ERR_UNIMPLEMENTED: return "configuration not supported by this build";
        default: return "unknown status";
    }
}

xgr_status xgr_workspace_bytes(const xgr_config *cfg, size_t *bytes) {
    const xgr_status e = check_config(cfg);
    if (e) return e;
    if (!bytes) return XGR_ERR_ARG;
    Layout L;
    make_layout(*cfg, L);
    *bytes = L.total;
    return XGR_OK;
}

xgr_status xgr_create(const xgr_config *cfg, void *d_workspace, size_t bytes, xgr_ctx **out) {
    const xgr_status e = check_config(cfg);
    if (e) return e;
    if (!out || !d_workspace || (reinterpret_cast<uintptr_t>(d_workspace) & (kAlign - 1)))
        return XGR_ERR_ARG;
    Layout L;
    make_layout(*cfg, L);
    if (bytes < L.total) return XGR_ERR_CAPACITY;
    xgr_ctx *c = new (std::nothrow) xgr_ctx();
    if (!c) return XGR_ERR_CAPACITY;
    c->cfg = *cfg;
    c->L = L;
    c->ws = static_cast<uint8_t *>(d_workspace);
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
        delete c;
        return XGR_ERR_CUDA;
    }
    c->dims = Dims{cfg->max_requests, cfg->beam_width, cfg->top_k, cfg->steps, cfg->n_q_heads,
                   cfg->n_kv_heads, cfg->head_dim, cfg->vocab, cfg->n_q_heads / cfg->n_kv_heads};
    c->st.status = c->at<int32_t>(L.status);
    c->st.n_live = c->at<int32_t>(L.n_live);
    c->st.cum = c->at<float>(L.cum);
    c->st.node = c->at<int32_t>(L.node);
    c->st.anc = c->at<int32_t>(L.anc);
    c->st.seq = c->at<int32_t>(L.seq);
    c->sid_off.assign(cfg->max_shared, 0);
    c->sid_len.assign(cfg->max_shared, 0);
    c->req_sid.assign(cfg->max_requests, -1);
    c->suf_off.assign(cfg->max_requests, 0);
    c->suf_len.assign(cfg->max_requests, 0);
    std::memset(&c->trie, 0, sizeof(c->trie));
    // the store starts as zeros so that key rows read past the end of a segment
    // (a tile's tail, masked out of the softmax) are always finite
    const size_t store_bytes = (size_t)2 * cfg->n_kv_heads * cfg->kv_tokens * cfg->head_dim;
    if (cudaMemset(c->st.status, 0, 16) != cudaSuccess ||
        (store_bytes && (cudaMemset(c->at<uint8_t>(L.kstore), 0, store_bytes) != cudaSuccess ||
                         cudaMemset(c->at<uint8_t>(L.vstore), 0, store_bytes) != cudaSuccess)) ||
        cudaDeviceSynchronize() != cudaSuccess) {
        delete c;
        return XGR_ERR_CUDA;
    }
    if (cfg->head_dim == 128 && cfg->kv_tokens > 0) {
        const int64_t rows = (int64_t)cfg->n_kv_heads * cfg->kv_tokens;
        c->has_tc = make_kv_tensor_map(&c->tmk, c->at<void>(L.kstore), rows) == cudaSuccess &&
                    make_kv_tensor_map(&c->tmv, c->at<void>(L.vstore), rows) == cudaSuccess;
    }
    *out = c;
    return XGR_OK;
}

xgr_status xgr_destroy(xgr_ctx *ctx) {
    if (!ctx) return XGR_ERR_ARG;
    delete ctx;
    return XGR_OK;
}

xgr_status xgr_build_trie(xgr_ctx *c, const int32_t *h_items, int64_t n_items, int32_t item_len) {
    if (!c || !h_items) return XGR_ERR_ARG;
    const xgr_config &cf = c->cfg;
    if (cf.vocab <= 0) return XGR_ERR_STATE;
    if (item_len != cf.steps || n_items < 1) return XGR_ERR_SHAPE;
    if (n_items > cf.max_items) return XGR_ERR_CAPACITY;
    const int L = item_len;
    for (int64_t i = 0; i < n_items * L; ++i)
        if (h_items[i] < 0 || h_items[i] >= cf.vocab) return XGR_ERR_SHAPE;
    // sort item indices lexicographically, drop repeats
    std::vector<int64_t> idx(n_items);
    std::iota(idx.begin(), idx.end(), 0);
    auto less = [&](int64_t a, int64_t b) {
        return std::lexicographical_compare(h_items + a * L, h_items + a * L + L, h_items + b * L,
                                            h_items + b * L + L);
    };
    std::sort(idx.begin(), idx.end(), less);
    auto same = [&](int64_t a, int64_t b, int len) {
        return std::equal(h_items + a * L, h_items + a * L + len, h_items + b * L);
    };
    idx.erase(std::unique(idx.begin(), idx.end(), [&](int64_t a, int64_t b) { return same(a, b, L); }),
              idx.end());
    const int64_t N = (int64_t)idx.size();
    // level l: nodes = distinct prefixes of length l, children = distinct prefixes of length l+1
    TrieView tv;
    std::memset(&tv, 0, sizeof(tv));
    tv.levels = L;
    tv.n_nodes[0] = 1;
    const int fan = fanout_cap(cf);
    std::vector<int32_t> ptr, tok;
    for (int l = 0; l < L; ++l) {
        ptr.clear();
        tok.clear();
        int max_children = 0, cur_children = 0;
        for (int64_t i = 0; i < N; ++i) {
            const bool new_node = (i == 0) || !same(idx[i], idx[i - 1], l);
            const bool new_child = (i == 0) || !same(idx[i], idx[i - 1], l + 1);
            if (new_node) {
                ptr.push_back((int32_t)tok.size());
                cur_children = 0;
            }
            if (new_child) {
                tok.push_back(h_items[idx[i] * L + l]);
                max_children = std::max(max_children, ++cur_children);
            }
        }
        ptr.push_back((int32_t)tok.size());
        if (l >= 1 && max_children > fan) return XGR_ERR_CAPACITY;
        if ((int64_t)ptr.size() > c->L.trie_level_cap || (int64_t)tok.size() > c->L.trie_level_cap)
            return XGR_ERR_CAPACITY;
        int32_t *dptr = c->at<int32_t>(c->L.trie_ptr) + (int64_t)l * c->L.trie_level_cap;
        int32_t *dtok = c->at<int32_t>(c->L.trie_tok) + (int64_t)l * c->L.trie_level_cap;
        if (cudaMemcpy(dptr, ptr.data(), ptr.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
            cudaMemcpy(dtok, tok.data(), tok.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
            return XGR_ERR_CUDA;
        tv.ptr[l] = dptr;
        tv.tok[l] = dtok;
        c->level_fanout[l] = max_children;
        c->level_bits[l] = false;
        tv.n_nodes[l + 1] = (int32_t)tok.size();
        // xGR 2.2 "Hybrid dense/sparse storage": dense, pre-generated masks for
        // the first steps -- here level 1 (step 1) when its nodes have many
        // children: one bitset of valid next tokens per node
        const int n_nodes_l = (int)ptr.size() - 1;
        const size_t nwv = (size_t)((cf.vocab + 31) / 32);
        if (l == 1 && c->L.node_bits_bytes >= (size_t)n_nodes_l * nwv * 4 &&
            max_children <= kNodeBitsStride && (int64_t)tok.size() * 256 >= (int64_t)n_nodes_l * cf.vocab) {
            std::vector<uint32_t> tb((size_t)n_nodes_l * nwv, 0u);
            for (int nd = 0; nd < n_nodes_l; ++nd)
                for (int e = ptr[nd]; e < ptr[nd + 1]; ++e) tb[(size_t)nd * nwv + (tok[e] >> 5)] |= 1u << (tok[e] & 31);
            if (cudaMemcpy(c->at<uint32_t>(c->L.node_bits), tb.data(), tb.size() * 4, cudaMemcpyHostToDevice) !=
                cudaSuccess)
                return XGR_ERR_CUDA;
            c->level_bits[l] = true;
        }
        if (l == 0) {
            std::vector<uint32_t> bits((cf.vocab + 31) / 32, 0u);
            for (int32_t t : tok) bits[t >> 5] |= 1u << (t & 31);
            uint32_t *db = c->at<uint32_t>(c->L.root_bits);
            if (cudaMemcpy(db, bits.data(), bits.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
                return XGR_ERR_CUDA;
            tv.root_bits = db;
        }
    }
    c->trie = tv;
    c->has_trie = true;
    return XGR_OK;
}

xgr_status xgr_prefill_kv(xgr_ctx *c, int32_t request, int32_t shared_id, const void *d_k,
                          const void *d_v, int32_t len, int32_t kind, xgr_stream_t stream) {
    if (!c) return XGR_ERR_ARG;
    const xgr_config &cf = c->cfg;
    if (kind != XGR_KV_SHARED && kind != XGR_KV_SUFFIX) return XGR_ERR_ARG;
    if (request < 0 || request >= cf.max_requests) return XGR_ERR_SHAPE;
    if (kind == XGR_KV_SHARED && (shared_id < 0 || shared_id >= cf.max_shared)) return XGR_ERR_SHAPE;
    const bool load = (kind == XGR_KV_SUFFIX) || d_k != nullptr;
    if (load) {
        if (!aligned16(d_k) || !aligned16(d_v)) return XGR_ERR_ARG;
        if (len < 1) return XGR_ERR_SHAPE;
        if (c->kv_used + len > cf.kv_tokens) return XGR_ERR_CAPACITY;
        const int64_t off = c->kv_used;
        const size_t D = cf.head_dim;
        for (int g = 0; g < cf.n_kv_heads; ++g) {
            const size_t dst = ((size_t)g * cf.kv_tokens + off) * D;
            const size_t src = (size_t)g * len * D;
            if (cudaMemcpyAsync(c->at<__nv_bfloat16>(c->L.kstore) + dst,
                                static_cast<const __nv_bfloat16 *>(d_k) + src, (size_t)len * D * 2,
                                cudaMemcpyDeviceToDevice, stream) != cudaSuccess ||
                cudaMemcpyAsync(c->at<__nv_bfloat16>(c->L.vstore) + dst,
                                static_cast<const __nv_bfloat16 *>(d_v) + src, (size_t)len * D * 2,
                                cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
                return XGR_ERR_CUDA;
        }
        if (cudaStreamSynchronize(stream) != cudaSuccess) return XGR_ERR_CUDA;
        c->kv_used += len;
        if (kind == XGR_KV_SHARED) {
            c->sid_off[shared_id] = off;
            c->sid_len[shared_id] = len;
        } else {
            c->suf_off[request] = off;
            c->suf_len[request] = len;
        }
    } else if (c->sid_len[shared_id] <= 0) {
        return XGR_ERR_STATE;
    }
    if (kind == XGR_KV_SHARED) c->req_sid[request] = shared_id;
    c->plan_dirty = true;
    return XGR_OK;
}

xgr_status xgr_reset_kv(xgr_ctx *c) {
    if (!c) return XGR_ERR_ARG;
    c->kv_used = 0;
    std::fill(c->sid_len.begin(), c->sid_len.end(), 0);
    std::fill(c->req_sid.begin(), c->req_sid.end(), -1);
    std::fill(c->suf_len.begin(), c->suf_len.end(), 0);
    c->plan_dirty = true;
    c->begun = false;
    return XGR_OK;
}

xgr_status xgr_begin(xgr_ctx *c, int32_t n_requests, xgr_stream_t stream) {
    if (!c) return XGR_ERR_ARG;
    if (n_requests < 1 || n_requests > c->cfg.max_requests) return XGR_ERR_SHAPE;
    if (c->plan_dirty || c->planned_B != n_requests) {
        for (int p = 0; p < 2; ++p) {
            const xgr_status e = build_plan(c, p, n_requests);
            if (e) return e;
        }
        // each request's KV ranges, for the per-beam comparison path
        std::vector<int32_t> seg(4 * (size_t)n_requests);
        for (int r = 0; r < n_requests; ++r) {
            const int sid = c->req_sid[r];
            seg[4 * r] = sid >= 0 ? (int32_t)c->sid_off[sid] : 0;
            seg[4 * r + 1] = sid >= 0 ? (int32_t)c->sid_len[sid] : 0;
            seg[4 * r + 2] = (int32_t)c->suf_off[r];
            seg[4 * r + 3] = (int32_t)c->suf_len[r];
        }
        if (cudaMemcpy(c->at<int32_t>(c->L.req_seg), seg.data(), seg.size() * 4, cudaMemcpyHostToDevice) !=
            cudaSuccess)
            return XGR_ERR_CUDA;
        c->plan_dirty = false;
        c->planned_B = n_requests;
    }
    c->dims.B = n_requests;
    if (launch_begin(c->st, c->dims, c->cfg.max_requests, c->cfg.vocab == 0,
                     c->cfg.vocab > 0 ? c->at<uint64_t>(c->L.mask_sync) : nullptr, (cudaStream_t)stream) !=
        cudaSuccess)
        return XGR_ERR_CUDA;
    c->begun = true;
    c->cur_step = 0;
    c->attn_step = -1;
    return XGR_OK;
}

xgr_status xgr_decode_step(xgr_ctx *c, int32_t step, const void *d_q, const void *d_k_new,
                           const void *d_v_new, void *d_out, float *d_lse, xgr_stream_t stream) {
    if (!c) return XGR_ERR_ARG;
    if (!aligned16(d_q) || !aligned16(d_k_new) || !aligned16(d_v_new) || !aligned16(d_out) ||
        !aligned16(d_lse))
        return XGR_ERR_ARG;
    if (!c->begun || step != c->cur_step || step >= c->cfg.steps) return XGR_ERR_STATE;
    const int which = (step == 0) ? 0 : 1;
    const cudaStream_t s = (cudaStream_t)stream;
    SmallArgs sa;
    sa.items = c->at<WorkItem>(c->L.plan_items[which]);
    sa.members = c->at<int32_t>(c->L.plan_members[which]);
    sa.q = static_cast<const __nv_bfloat16 *>(d_q);
    sa.kstore = c->at<__nv_bfloat16>(c->L.kstore);
    sa.vstore = c->at<__nv_bfloat16>(c->L.vstore);
    sa.kv_tokens = c->cfg.kv_tokens;
    sa.dims = c->dims;
    sa.nb = (which == 0) ? 1 : c->cfg.beam_width;
    sa.n_live = c->st.n_live;
    sa.part = partials_of(c);
    {
        const cudaError_t e = launch_attn_small(sa, c->n_small[which], s);
        if (e != cudaSuccess) {
            debug_log("decode_step: small-row launch failed: %s", cudaGetErrorString(e));
            return XGR_ERR_CUDA;
        }
    }
    if (c->n_tc[which] > 0) {
        TcArgs ta;
        ta.items = sa.items + c->n_small[which];
        ta.members = sa.members;
        ta.q = sa.q;
        ta.kv_tokens = sa.kv_tokens;
        ta.dims = sa.dims;
        ta.nb = sa.nb;
        ta.n_live = sa.n_live;
        ta.part = sa.part;
        ta.status = c->st.status;
        ta.k_new = static_cast<const __nv_bfloat16 *>(d_k_new);
        ta.v_new = static_cast<const __nv_bfloat16 *>(d_v_new);
        ta.pool_k = c->at<__nv_bfloat16>(c->L.pool_k);
        ta.pool_v = c->at<__nv_bfloat16>(c->L.pool_v);
        ta.out = static_cast<__nv_bfloat16 *>(d_out);
        ta.lse = d_lse;
        ta.st = c->st;
        ta.Bcap = c->cfg.max_requests;
        ta.step = step;
        ta.shared_o = c->tc_shared[which];
        // Q tiles of single-request items are one TMA box: D x (query heads of
        // one kv head) x (128 / G beams) over q viewed as [B*BW][Hq][D]
        const int64_t q_rows = (int64_t)c->dims.B * c->cfg.beam_width;
        if (c->tmq_ptr != d_q || c->tmq_rows != q_rows) {
            if (make_q_tensor_map(&c->tmq, d_q, q_rows, c->cfg.n_q_heads, c->dims.G) != cudaSuccess) {
                c->tmq_ptr = nullptr;
                debug_log("decode_step: q tensor map failed");
                return XGR_ERR_CUDA;
            }
            c->tmq_ptr = d_q;
            c->tmq_rows = q_rows;
        }
        const cudaError_t e = launch_attn_tc(c->tmk, c->tmv, c->tmq, ta, c->n_tc[which], s);
        if (e != cudaSuccess) {
            debug_log("decode_step: tensor-core launch failed: %s", cudaGetErrorString(e));
            return XGR_ERR_CUDA;
        }
    }
    // every request finished by the tensor-core launch (its items cover every
    // beam's rows, the not-yet-live ones at step 0 by zero-fill items): no merge
    if (c->n_unfused[which] == 0) {
        if (c->cfg.vocab == 0) c->cur_step = step + 1;
        c->attn_step = step;
        c->attn_stream = s;
        return XGR_OK;
    }
    MergeArgs ma;
    ma.q = sa.q;
    ma.k_new = static_cast<const __nv_bfloat16 *>(d_k_new);
    ma.v_new = static_cast<const __nv_bfloat16 *>(d_v_new);
    ma.pool_k = c->at<__nv_bfloat16>(c->L.pool_k);
    ma.pool_v = c->at<__nv_bfloat16>(c->L.pool_v);
    ma.out = static_cast<__nv_bfloat16 *>(d_out);
    ma.lse = d_lse;
    ma.st = c->st;
    ma.dims = c->dims;
    ma.Bcap = c->cfg.max_requests;
    ma.step = step;
    ma.n_slots = c->at<int32_t>(c->L.plan_nslots[which]);
    ma.part = sa.part;
    {
        const cudaError_t e = launch_attn_merge(ma, s);
        if (e != cudaSuccess) {
            debug_log("decode_step: merge launch failed: %s", cudaGetErrorString(e));
            return XGR_ERR_CUDA;
        }
    }
    if (c->cfg.vocab == 0) c->cur_step = step + 1;   // attention-only: no selection step
    c->attn_step = step;
    c->attn_stream = s;
    return XGR_OK;
}

xgr_status xgr_per_beam_bytes(const xgr_ctx *c, size_t *bytes) {
    if (!c || !bytes) return XGR_ERR_ARG;
    *bytes = per_beam_block_bytes(c->cfg.max_requests, c->cfg.beam_width, c->cfg.n_kv_heads, c->cfg.head_dim);
    return XGR_OK;
}

xgr_status xgr_decode_step_per_beam(xgr_ctx *c, int32_t step, const void *d_q, const void *d_k_new,
                                    const void *d_v_new, void *d_out, float *d_lse, void *d_blocks,
                                    size_t blocks_bytes, xgr_stream_t stream) {
    if (!c) return XGR_ERR_ARG;
    if (!aligned16(d_q) || !aligned16(d_k_new) || !aligned16(d_v_new) || !aligned16(d_out) ||
        !aligned16(d_lse) || !aligned16(d_blocks))
        return XGR_ERR_ARG;
    if (!c->begun || step != c->cur_step || step >= c->cfg.steps) return XGR_ERR_STATE;
    if (c->cfg.head_dim != 128 || c->dims.G > 8 || (c->dims.G & (c->dims.G - 1)) || step + 1 > kPerBeamBlock)
        return XGR_ERR_UNIMPLEMENTED;
    const size_t need = per_beam_block_bytes(c->cfg.max_requests, c->cfg.beam_width, c->cfg.n_kv_heads,
                                             c->cfg.head_dim);
    if (blocks_bytes < need) return XGR_ERR_CAPACITY;
    const cudaStream_t s = (cudaStream_t)stream;
    PerBeamArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(d_q);
    a.k_new = static_cast<const __nv_bfloat16 *>(d_k_new);
    a.v_new = static_cast<const __nv_bfloat16 *>(d_v_new);
    a.kstore = c->at<__nv_bfloat16>(c->L.kstore);
    a.vstore = c->at<__nv_bfloat16>(c->L.vstore);
    a.blk_k = static_cast<__nv_bfloat16 *>(d_blocks);
    a.blk_v = a.blk_k + need / 4;   // (need / 2 bytes of K blocks, then V)
    a.out = static_cast<__nv_bfloat16 *>(d_out);
    a.lse = d_lse;
    a.req_seg = c->at<int32_t>(c->L.req_seg);
    a.n_live = c->st.n_live;
    a.st = c->st;
    a.status = c->st.status;
    a.dims = c->dims;
    a.Bcap = c->cfg.max_requests;
    a.step = step;
    a.kv_tokens = c->cfg.kv_tokens;
    if (launch_per_beam(a, s) != cudaSuccess) return XGR_ERR_CUDA;
    if (c->cfg.vocab == 0) c->cur_step = step + 1;   // attention-only: no selection step
    c->attn_step = step;
    c->attn_stream = s;
    return XGR_OK;
}

xgr_status xgr_build_mask(xgr_ctx *c, int32_t step, xgr_mask *out, xgr_stream_t stream) {
    (void)stream;   // every kind is a view: nothing is enqueued
    if (!c || !out) return XGR_ERR_ARG;
    if (!c->has_trie || !c->begun || step != c->cur_step || step >= c->cfg.steps)
        return XGR_ERR_STATE;
    std::memset(out, 0, sizeof(*out));
    out->step = step;
    out->n_rows = c->dims.B * c->dims.BW;
    out->n_words = (c->cfg.vocab + 31) / 32;
    if (step == 0) {
        out->kind = XGR_MASK_DENSE;
        out->bits = c->trie.root_bits;
        return XGR_OK;
    }
    out->kind = c->level_bits[step] ? XGR_MASK_NODE_BITS : XGR_MASK_TRIE_ROWS;
    out->bits = c->level_bits[step] ? c->at<uint32_t>(c->L.node_bits) : nullptr;
    out->row_node = c->st.node;
    out->node_ptr = c->trie.ptr[step];
    out->cols = c->trie.tok[step];
    out->cols_capacity = c->trie.n_nodes[step + 1];
    out->n_nodes = c->trie.n_nodes[step];
    out->row_stride = std::max(1, c->level_fanout[step]);
    return XGR_OK;
}

xgr_status xgr_mask_to_csr(xgr_ctx *c, const xgr_mask *mask, int32_t *d_row_ptr, int32_t *d_cols,
                           int64_t cols_capacity, xgr_stream_t stream) {
    if (!c || !mask || !aligned16(d_row_ptr) || !aligned16(d_cols) || cols_capacity < 1) return XGR_ERR_ARG;
    if (mask->kind != XGR_MASK_NODE_BITS && mask->kind != XGR_MASK_TRIE_ROWS) return XGR_ERR_ARG;
    if (!c->has_trie || !c->begun || mask->step != c->cur_step || mask->step < 1 ||
        mask->step >= c->cfg.steps)
        return XGR_ERR_STATE;
    const int step = mask->step;
    MaskArgs ma;
    ma.st = c->st;
    ma.trie = c->trie;
    ma.dims = c->dims;
    ma.step = step;
    ma.row_ptr = d_row_ptr;
    ma.cols = d_cols;
    ma.cap = cols_capacity;
    ma.flags = c->at<uint64_t>(c->L.mask_sync);
    ma.ticket = reinterpret_cast<uint32_t *>(ma.flags + c->cfg.max_requests);
    // CTAs per request sharing the copy: about 16K entries each
    const int64_t entries = (int64_t)c->cfg.beam_width * c->level_fanout[step];
    const int parts = (int)std::min<int64_t>(16, std::max<int64_t>(1, (entries + 16383) / 16384));
    if (launch_build_mask(ma, parts, (cudaStream_t)stream) != cudaSuccess) return XGR_ERR_CUDA;
    return XGR_OK;
}

xgr_status xgr_beam_select(xgr_ctx *c, int32_t step, const float *d_scores, int32_t flags,
                           const xgr_mask *mask, int32_t *d_parent, int32_t *d_token, float *d_cum,
                           int32_t *d_n_out, xgr_stream_t stream) {
    if (!c || !mask) return XGR_ERR_ARG;
    if (flags != XGR_SCORES_LOGPROB && flags != XGR_SCORES_LOGITS) return XGR_ERR_ARG;
    if (!aligned16(d_scores) || !aligned16(d_parent) || !aligned16(d_token) || !aligned16(d_cum) ||
        !aligned16(d_n_out))
        return XGR_ERR_ARG;
    if (!c->has_trie || !c->begun || step != c->cur_step || step >= c->cfg.steps)
        return XGR_ERR_STATE;
    if (mask->step != step) return XGR_ERR_STATE;
    if (step == 0) {
        if (mask->kind != XGR_MASK_DENSE || !mask->bits) return XGR_ERR_ARG;
    } else if (mask->kind == XGR_MASK_CSR) {
        if (!mask->row_ptr || !mask->cols) return XGR_ERR_ARG;
    } else if (mask->kind == XGR_MASK_TRIE_ROWS || mask->kind == XGR_MASK_NODE_BITS) {
        // node views of this context's own trie level and beam state only
        if (mask->row_node != c->st.node || mask->node_ptr != c->trie.ptr[step] ||
            mask->cols != c->trie.tok[step] || mask->n_nodes != c->trie.n_nodes[step] ||
            mask->row_stride != std::max(1, c->level_fanout[step]))
            return XGR_ERR_ARG;
        if (mask->kind == XGR_MASK_NODE_BITS &&
            (!c->level_bits[step] || mask->bits != c->at<uint32_t>(c->L.node_bits) ||
             mask->n_words != (c->cfg.vocab + 31) / 32))
            return XGR_ERR_ARG;
    } else {
        return XGR_ERR_ARG;
    }
    SelectArgs a;
    a.cum = c->st.cum;
    a.n_live = c->st.n_live;
    a.status = c->st.status;
    a.rewire = 1;
    a.st = c->st;
    a.trie = c->trie;
    a.dims = c->dims;
    a.step = step;
    a.logits = flags == XGR_SCORES_LOGITS;
    a.scores = d_scores;
    a.dense = step == 0;
    a.bits = mask->bits;
    a.mask_kind = mask->kind;
    a.row_ptr = mask->row_ptr;
    a.cols = mask->cols;
    a.row_node = mask->row_node;
    a.node_ptr = mask->node_ptr;
    a.node_tok = mask->cols;
    a.node_bits = mask->kind == XGR_MASK_NODE_BITS ? mask->bits : nullptr;
    a.n_nodes = mask->n_nodes;
    a.n_words = mask->n_words;
    a.row_stride = mask->row_stride;
    a.num_sms = c->num_sms;
    // right after this step's attention on the same stream, the kernel before
    // the selection wrote no beam state (the attention reads it only)
    a.prep_early = c->attn_step == step && c->attn_stream == (cudaStream_t)stream;
    select_scratch_carve(c->at<uint8_t>(c->L.select_scratch), c->cfg.max_requests,
                         c->cfg.beam_width, c->L.key_cap, a);
    a.parent = d_parent;
    a.token = d_token;
    a.cum_out = d_cum;
    a.n_out = d_n_out;
    c->attn_step = -1;
    if (launch_beam_select(a, (cudaStream_t)stream) != cudaSuccess) return XGR_ERR_CUDA;
    c->cur_step = step + 1;
    return XGR_OK;
}

xgr_status xgr_get_sequences(xgr_ctx *c, int32_t *d_seq, xgr_stream_t stream) {
    if (!c || !aligned16(d_seq)) return XGR_ERR_ARG;
    if (!c->begun) return XGR_ERR_STATE;
    if (launch_get_sequences(c->st, c->dims, d_seq, (cudaStream_t)stream) != cudaSuccess)
        return XGR_ERR_CUDA;
    return XGR_OK;
}

xgr_status xgr_device_status(xgr_ctx *c, xgr_stream_t stream, int32_t *host_code) {
    if (!c || !host_code) return XGR_ERR_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return XGR_ERR_CUDA;
    int32_t code = 0;
    if (cudaMemcpy(&code, c->st.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(c->st.status, 0, 4) != cudaSuccess)
        return XGR_ERR_CUDA;
    *host_code = code;
    return code ? XGR_ERR_DEVICE : XGR_OK;
}

}  // extern "C"

// sched_cht.cu -- the Chunked Hash Tree batch former (host code only).
//
// Feather page ("Requests of the same feather must flock together"),
// "Methodology", 1. Chunked Hash Tree: requests as cumulative hashes over
// fixed-size token chunks, a working set of the hashes of the batch being
// formed, and a min-heap of waiting requests keyed by their missing count, so
// that the best request to add is found in O(log W).  The heap is updated
// lazily: when a hash enters the working set, every waiting request that holds
// it gets its count lowered and a fresh heap entry; stale entries are skipped
// when they reach the top.  The batch's tip (its shared depth in chunks) is
// kept incrementally by a binary search against the first member's hashes.
// Readings of what the page leaves open are in include/xgr_sched.h.
#include <algorithm>
#include <cstdint>
#include <functional>
#include <new>
#include <queue>
#include <tuple>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "../../include/xgr_sched.h"

namespace {

// SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): its output function, applied to a running state.
inline uint64_t splitmix64(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

enum : uint8_t { kWaiting = 0, kInBatch = 1, kGone = 2 };

struct Req {
    int64_t id = 0, seq = 0;
    std::vector<uint64_t> h;   // cumulative hash after each full chunk
    int32_t missing = 0;       // chunks whose hash is not in the working set
    uint8_t state = kWaiting;
    int32_t n() const { return (int32_t)h.size(); }
};

}  // namespace

struct xgr_cht {
    int32_t chunk = 1;
    int64_t next_seq = 0;
    std::vector<Req> reqs;                                      // every request ever inserted
    std::unordered_map<int64_t, int32_t> live;                  // id -> index, waiting or in the batch
    std::unordered_map<uint64_t, std::vector<int32_t>> holders;  // hash -> requests holding it (lazy)
    std::unordered_set<uint64_t> ws;                            // the batch's working set
    std::vector<int32_t> batch;                                 // members in join order
    int32_t tip = 0;                                            // chunks shared by every member
    int32_t n_waiting = 0;
    using Entry = std::tuple<int32_t, int64_t, int32_t>;        // (missing, seq, index)
    std::priority_queue<Entry, std::vector<Entry>, std::greater<Entry>> by_missing;
    using Fifo = std::pair<int64_t, int32_t>;                   // (seq, index)
    std::priority_queue<Fifo, std::vector<Fifo>, std::greater<Fifo>> by_age;

    // chunks of r whose hashes are in the working set (a prefix: the set holds
    // every chunk hash of every member, so it is closed under prefixes)
    int32_t covered(const Req &r) const {
        int32_t lo = 0, hi = r.n();
        while (lo < hi) {
            const int32_t mid = (lo + hi + 1) / 2;
            if (ws.count(r.h[mid - 1])) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    }
    // leading chunks r shares with the batch's first member, at most the tip
    int32_t shared_with_tip(const Req &r) const {
        const Req &f = reqs[batch.front()];
        int32_t lo = 0, hi = std::min(tip, r.n());
        while (lo < hi) {
            const int32_t mid = (lo + hi + 1) / 2;
            if (r.h[mid - 1] == f.h[mid - 1]) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    }
    int32_t best() {   // index of the best waiting request, or -1
        if (n_waiting == 0) return -1;
        if (batch.empty()) {
            while (!by_age.empty() && reqs[by_age.top().second].state != kWaiting) by_age.pop();
            return by_age.empty() ? -1 : by_age.top().second;
        }
        while (!by_missing.empty()) {
            const auto [m, s, i] = by_missing.top();
            if (reqs[i].state == kWaiting && reqs[i].missing == m) return i;
            by_missing.pop();   // stale
        }
        return -1;
    }
    // The best waiting request whose depth_after reaches `floor` (smallest missing
    // count, then the earliest inserted), or -1.  Entries that fail the floor are
    // set aside while the heap is searched and pushed back afterwards, so a
    // request that shares nothing with the batch (a short or unrelated prompt,
    // whose missing count is small) does not end the batch while requests that
    // share its prefix still wait.
    int32_t best_passing(int32_t floor) {
        if (n_waiting == 0 || batch.empty()) return -1;
        std::vector<Entry> aside;
        int32_t found = -1;
        while (!by_missing.empty()) {
            const Entry e = by_missing.top();
            const int32_t i = std::get<2>(e);
            if (reqs[i].state != kWaiting || reqs[i].missing != std::get<0>(e)) {
                by_missing.pop();   // stale
                continue;
            }
            if (shared_with_tip(reqs[i]) >= floor) {
                found = i;
                break;
            }
            aside.push_back(e);
            by_missing.pop();
        }
        for (const Entry &e : aside) by_missing.push(e);
        return found;
    }
    void add(int32_t i) {
        Req &r = reqs[i];
        const int32_t from = covered(r);
        r.state = kInBatch;
        --n_waiting;
        if (batch.empty()) tip = r.n();
        batch.push_back(i);
        if (batch.size() > 1) tip = shared_with_tip(r);
        for (int32_t p = from; p < r.n(); ++p) {   // new hashes: the holders' counts drop
            if (!ws.insert(r.h[p]).second) continue;
            auto it = holders.find(r.h[p]);
            if (it == holders.end()) continue;
            for (int32_t j : it->second) {
                Req &o = reqs[j];
                if (o.state != kWaiting) continue;
                --o.missing;
                by_missing.emplace(o.missing, o.seq, j);
            }
        }
    }
    // drops departed requests from the tables (only between batches: no member
    // indices are held then)
    void compact() {
        std::vector<Req> keep;
        keep.reserve(live.size());
        for (auto &kv : live) {
            keep.push_back(std::move(reqs[kv.second]));
            kv.second = (int32_t)keep.size() - 1;
        }
        reqs.swap(keep);
        holders.clear();
        by_age = decltype(by_age)();
        for (int32_t i = 0; i < (int32_t)reqs.size(); ++i) {
            for (uint64_t x : reqs[i].h) holders[x].push_back(i);
            by_age.emplace(reqs[i].seq, i);
        }
    }
    void restart() {   // an empty batch: every waiting request misses all its chunks
        batch.clear();
        ws.clear();
        tip = 0;
        if (reqs.size() > 2 * live.size() + 1024) compact();
        by_missing = decltype(by_missing)();
        for (const auto &kv : live) {
            Req &r = reqs[kv.second];
            if (r.state != kWaiting) continue;
            r.missing = r.n();
            by_missing.emplace(r.missing, r.seq, kv.second);
        }
    }
    int32_t dispatch(int64_t *ids, int32_t cap) {
        const int32_t n = (int32_t)batch.size();
        for (int32_t k = 0; k < n; ++k) {
            Req &r = reqs[batch[k]];
            if (ids && k < cap) ids[k] = r.id;
            r.state = kGone;
            live.erase(r.id);
        }
        restart();
        return n;
    }
};

extern "C" {

xgr_status xgr_cht_create(int32_t chunk_tokens, xgr_cht **out) {
    if (!out) return XGR_ERR_ARG;
    *out = nullptr;
    if (chunk_tokens < 1) return XGR_ERR_SHAPE;
    xgr_cht *t = new (std::nothrow) xgr_cht();
    if (!t) return XGR_ERR_CAPACITY;
    t->chunk = chunk_tokens;
    *out = t;
    return XGR_OK;
}

xgr_status xgr_cht_destroy(xgr_cht *t) {
    if (!t) return XGR_ERR_ARG;
    delete t;
    return XGR_OK;
}

xgr_status xgr_cht_insert(xgr_cht *t, int64_t request_id, const int32_t *h_tokens, int64_t n_tokens) {
    if (!t || (n_tokens > 0 && !h_tokens) || request_id < 0) return XGR_ERR_ARG;
    if (n_tokens < 0) return XGR_ERR_SHAPE;
    if (t->live.count(request_id)) return XGR_ERR_ARG;
    Req r;
    r.id = request_id;
    r.seq = t->next_seq++;
    const int64_t full = n_tokens / t->chunk;
    r.h.reserve((size_t)full);
    uint64_t h = 0;
    for (int64_t c = 0; c < full; ++c) {
        for (int64_t k = 0; k < t->chunk; ++k) h = splitmix64(h ^ (uint32_t)h_tokens[c * t->chunk + k]);
        r.h.push_back(h);
    }
    const int32_t i = (int32_t)t->reqs.size();
    r.missing = r.n() - (t->batch.empty() ? 0 : t->covered(r));
    for (uint64_t x : r.h) t->holders[x].push_back(i);
    t->by_missing.emplace(r.missing, r.seq, i);
    t->by_age.emplace(r.seq, i);
    t->reqs.push_back(std::move(r));
    t->live[request_id] = i;
    ++t->n_waiting;
    return XGR_OK;
}

xgr_status xgr_cht_remove(xgr_cht *t, int64_t request_id) {
    if (!t) return XGR_ERR_ARG;
    auto it = t->live.find(request_id);
    if (it == t->live.end()) return XGR_ERR_ARG;
    Req &r = t->reqs[it->second];
    if (r.state != kWaiting) return XGR_ERR_STATE;
    r.state = kGone;
    t->live.erase(it);
    --t->n_waiting;
    return XGR_OK;
}

xgr_status xgr_cht_find_best(xgr_cht *t, int64_t *request_id, int32_t *missing, int32_t *depth_after,
                             int32_t *delta, int32_t *w) {
    if (!t || !request_id) return XGR_ERR_ARG;
    const int32_t i = t->best();
    *request_id = -1;
    if (missing) *missing = 0;
    if (depth_after) *depth_after = 0;
    if (delta) *delta = 0;
    if (w) *w = 0;
    if (i < 0) return XGR_OK;
    const Req &r = t->reqs[i];
    *request_id = r.id;
    const int32_t d = t->batch.empty() ? r.n() : t->shared_with_tip(r);
    if (missing) *missing = t->batch.empty() ? r.n() : r.missing;
    if (depth_after) *depth_after = d;
    if (delta) *delta = t->batch.empty() ? 0 : t->tip - d;
    if (w && d > 0) {
        const uint64_t key = r.h[d - 1];
        int32_t c = 0;
        auto it = t->holders.find(key);
        if (it != t->holders.end())
            for (int32_t j : it->second) c += (j != i && t->reqs[j].state == kWaiting) ? 1 : 0;
        *w = c;
    }
    return XGR_OK;
}

xgr_status xgr_cht_add_to_batch(xgr_cht *t, int64_t request_id) {
    if (!t) return XGR_ERR_ARG;
    auto it = t->live.find(request_id);
    if (it == t->live.end()) return XGR_ERR_ARG;
    if (t->reqs[it->second].state != kWaiting) return XGR_ERR_STATE;
    t->add(it->second);
    return XGR_OK;
}

xgr_status xgr_cht_dispatch(xgr_cht *t, int64_t *h_ids, int32_t cap, int32_t *n, int32_t *shared_chunks) {
    if (!t || (cap > 0 && !h_ids)) return XGR_ERR_ARG;
    if (shared_chunks) *shared_chunks = t->batch.empty() ? 0 : t->tip;
    const int32_t k = t->dispatch(h_ids, cap);
    if (n) *n = k;
    return XGR_OK;
}

xgr_status xgr_cht_counts(xgr_cht *t, int32_t *waiting, int32_t *in_batch) {
    if (!t) return XGR_ERR_ARG;
    if (waiting) *waiting = t->n_waiting;
    if (in_batch) *in_batch = (int32_t)t->batch.size();
    return XGR_OK;
}

xgr_status xgr_cht_form_batches(xgr_cht *t, int32_t max_batch, int32_t min_shared_chunks, int64_t *h_ids,
                                int64_t cap_ids, int32_t *h_sizes, int32_t *h_shared, int32_t cap_batches,
                                int32_t *n_batches) {
    if (!t || !h_ids || !h_sizes || !h_shared || !n_batches || max_batch < 1) return XGR_ERR_ARG;
    const int64_t total = (int64_t)t->n_waiting + (int64_t)t->batch.size();
    const int64_t most = (int64_t)t->n_waiting + (t->batch.empty() ? 0 : 1);   // one batch per request at most
    if (cap_ids < total || cap_batches < most) return XGR_ERR_CAPACITY;
    int64_t at = 0;
    int32_t nb = 0;
    auto close = [&]() {
        h_shared[nb] = t->tip;
        const int32_t k = t->dispatch(h_ids + at, (int32_t)std::min<int64_t>(cap_ids - at, INT32_MAX));
        h_sizes[nb++] = k;
        at += k;
    };
    if (!t->batch.empty()) close();
    while (t->n_waiting > 0) {
        t->add(t->best());   // the oldest waiting request seeds the batch
        while ((int32_t)t->batch.size() < max_batch) {
            const int32_t i = t->best_passing(min_shared_chunks);
            if (i < 0) break;
            t->add(i);
        }
        close();
    }
    *n_batches = nb;
    return XGR_OK;
}

}  // extern "C"

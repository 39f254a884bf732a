// kv_cache.cpp -- host-side manager of the two-tier paged KV cache (GPU pages + pinned host pages).
//
// The serving path's cache (NVIDIA blog "Deploying an HSTU Generative Recommender with NVIDIA
// Dynamo-Triton", section "Why serving large sequential recommenders is hard"): a paged GPU KV
// table with lookup, allocate, append and evict, LRU-like eviction of old users when GPU space
// runs short, and a host tier with onboard and offload.  The exact policy is written out in
// include/hstu.h above hstu_cache_create; this file implements it.
//
// Data structures (sized for pools of 10^5..10^6 pages and as many users):
//   - per tier, a bitmap of free pages (bit set = free) with a hint at the lowest word that may
//     hold a set bit, so "the k lowest free pages" is a scan of set bits from the hint;
//   - per tier, an ordered set of (stamp, user id) of its residents: the LRU order;
//   - a hash map from user id to its record (tier, stored length, stamp, page list).
// A prepare call first decides everything without touching the state (victims, which of them
// fit in the host tier, which host residents make room, the output sizes), checks the output
// capacities, and only then applies the decisions, so a failed call changes nothing.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <unordered_map>
#include <unordered_set>
#include <utility>
#include <vector>

#include "hstu.h"

namespace {

class PageBitmap {
public:
    explicit PageBitmap(int32_t n) : n_(n), words_((size_t)(n + 63) / 64, ~0ull), free_(n)
    {
        if (n % 64)
            words_.back() = (1ull << (n % 64)) - 1;
        if (n == 0)
            words_.clear();
    }
    int32_t free_count() const { return free_; }
    bool is_free(int32_t p) const { return (words_[p >> 6] >> (p & 63)) & 1ull; }

    // the k lowest free pages, ascending, marked used; the caller has checked k <= free_count()
    void take(int32_t k, std::vector<int32_t>& out)
    {
        size_t w = hint_;
        while (k > 0 && w < words_.size()) {
            uint64_t bits = words_[w];
            while (bits && k > 0) {
                const int b = __builtin_ctzll(bits);
                bits &= bits - 1;
                out.push_back((int32_t)(w * 64 + b));
                --k;
                --free_;
            }
            words_[w] = bits;   // the bits handed out are cleared, the rest stay free
            if (k > 0)
                ++w;
        }
        hint_ = w;
    }

    void give(const std::vector<int32_t>& pages)
    {
        for (int32_t p : pages) {
            words_[p >> 6] |= 1ull << (p & 63);
            hint_ = std::min(hint_, (size_t)(p >> 6));
        }
        free_ += (int32_t)pages.size();
    }

    // free pages below `limit`, ascending
    void free_below(int32_t limit, std::vector<int32_t>& out) const
    {
        for (size_t w = hint_; w < words_.size() && (int64_t)w * 64 < limit; ++w) {
            uint64_t bits = words_[w];
            while (bits) {
                const int b = __builtin_ctzll(bits);
                bits &= bits - 1;
                const int32_t p = (int32_t)(w * 64 + b);
                if (p >= limit)
                    return;
                out.push_back(p);
            }
        }
    }

    // everything below `live` used, everything from `live` on free
    void reset_prefix(int32_t live)
    {
        std::fill(words_.begin(), words_.end(), 0ull);
        for (int32_t p = live; p < n_; ++p)
            words_[p >> 6] |= 1ull << (p & 63);
        free_ = n_ - live;
        hint_ = (size_t)(live >> 6);
    }

private:
    int32_t n_;
    std::vector<uint64_t> words_;
    size_t hint_ = 0;   // every word below it is zero (no free page)
    int32_t free_;
};

struct UserRec {
    int32_t tier = HSTU_TIER_MISS;
    int32_t n = 0;
    int64_t stamp = 0;
    std::vector<int32_t> pages;
};

using LruKey = std::pair<int64_t, int64_t>;   // (stamp, user id)

}  // namespace

struct hstu_kv_cache {
    int32_t G, Hp, P, M;
    PageBitmap gpu_free, host_free;
    std::set<LruKey> gpu_lru, host_lru;
    std::unordered_map<int64_t, UserRec> users;
    int64_t clock = 0;
    std::mutex mu;

    hstu_kv_cache(int32_t g, int32_t hp, int32_t p, int32_t m) : G(g), Hp(hp), P(p), M(m), gpu_free(g), host_free(hp) {}

    int64_t pages_for(int64_t n) const { return (n + P - 1) / P; }
    PageBitmap& bitmap(int32_t tier) { return tier == HSTU_TIER_GPU ? gpu_free : host_free; }
    std::set<LruKey>& lru(int32_t tier) { return tier == HSTU_TIER_GPU ? gpu_lru : host_lru; }

    void take(int32_t tier, int32_t k, std::vector<int32_t>& out)
    {
        if (k <= 0)
            return;
        bitmap(tier).take(k, out);
    }
};

namespace {

// One victim's fate, decided before anything changes.
struct VictimPlan {
    int64_t id;
    bool placed;                      // offloaded to the host tier (else dropped)
    std::vector<int64_t> host_drops;  // host residents dropped to make room, oldest first
};

}  // namespace

extern "C" {

int hstu_cache_create(int32_t gpu_pages, int32_t host_pages, int32_t page_size, int32_t max_pages_per_user,
                      hstu_kv_cache** out)
{
    if (!out || gpu_pages < 0 || host_pages < 0 || page_size < 1 || max_pages_per_user < 1)
        return HSTU_ERR_INVALID_ARG;
    if ((int64_t)page_size * max_pages_per_user >= ((int64_t)1 << 31))
        return HSTU_ERR_INVALID_ARG;   // stored lengths are int32
    *out = nullptr;
    try {
        *out = new hstu_kv_cache(gpu_pages, host_pages, page_size, max_pages_per_user);
    } catch (...) {
        return HSTU_ERR_INVALID_ARG;
    }
    return HSTU_OK;
}

void hstu_cache_destroy(hstu_kv_cache* c) { delete c; }

int hstu_cache_lookup(hstu_kv_cache* c, const int64_t* ids, int32_t n, int32_t* tier_out, int32_t* len_out)
{
    if (!c || n < 0 || (n > 0 && (!ids || !tier_out || !len_out)))
        return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    for (int32_t i = 0; i < n; ++i) {
        auto it = c->users.find(ids[i]);
        tier_out[i] = it == c->users.end() ? HSTU_TIER_MISS : it->second.tier;
        len_out[i] = it == c->users.end() ? 0 : it->second.n;
    }
    return HSTU_OK;
}

int hstu_cache_prepare(hstu_kv_cache* c, const int64_t* ids, const int32_t* append, int32_t B,
                       int32_t* tier_before_out, int32_t* cached_out, int32_t* rows_out, int32_t* offload_out,
                       int32_t offload_cap, int32_t* n_offload, int32_t* onboard_out, int32_t onboard_cap,
                       int32_t* n_onboard, int64_t* dropped_out, int32_t dropped_cap, int32_t* n_dropped)
{
    if (!c || B < 0 || !n_offload || !n_onboard || !n_dropped || offload_cap < 0 || onboard_cap < 0 ||
        dropped_cap < 0)
        return HSTU_ERR_INVALID_ARG;
    if (B > 0 && (!ids || !append || !tier_before_out || !cached_out || !rows_out))
        return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);

    // ---- validation and the batch's GPU page demand
    std::unordered_set<int64_t> batch;
    batch.reserve((size_t)B * 2);
    std::vector<int32_t> need((size_t)B);
    int64_t demand = 0;
    for (int32_t b = 0; b < B; ++b) {
        if (append[b] < 0 || !batch.insert(ids[b]).second)
            return HSTU_ERR_INVALID_ARG;
        auto it = c->users.find(ids[b]);
        const int64_t n = it == c->users.end() ? 0 : it->second.n;
        const int64_t k = c->pages_for(n + append[b]);
        if (k > c->M)
            return HSTU_ERR_INVALID_ARG;
        need[b] = (int32_t)k;
        const int64_t have =
            (it != c->users.end() && it->second.tier == HSTU_TIER_GPU) ? (int64_t)it->second.pages.size() : 0;
        demand += k - have;
    }

    // ---- GPU victims: residents outside the batch, oldest first, until the demand fits
    std::vector<int64_t> victims;   // ascending (stamp, id)
    int64_t obtainable = c->gpu_free.free_count();
    for (auto it = c->gpu_lru.begin(); it != c->gpu_lru.end() && obtainable < demand; ++it) {
        if (batch.count(it->second))
            continue;
        victims.push_back(it->second);
        obtainable += (int64_t)c->users[it->second].pages.size();
    }
    if (obtainable < demand)
        return HSTU_ERR_CACHE_FULL;

    // ---- host placement, newest victim first; host residents are dropped from the oldest end
    std::vector<VictimPlan> plans;
    plans.reserve(victims.size());
    int64_t host_free = c->host_free.free_count();
    auto hcur = c->host_lru.begin();   // host residents before hcur are already dropped (or in the batch)
    int64_t count_offload = 0, count_drop = 0;
    for (size_t vi = victims.size(); vi-- > 0;) {
        const int64_t vid = victims[vi];
        const UserRec& v = c->users[vid];
        const LruKey vkey{v.stamp, vid};
        const int64_t k = (int64_t)v.pages.size();
        VictimPlan plan{vid, false, {}};
        int64_t avail = host_free;
        for (auto it = hcur; it != c->host_lru.end() && *it < vkey && avail < k; ++it)
            if (!batch.count(it->second))
                avail += (int64_t)c->users[it->second].pages.size();
        if (avail >= k) {
            while (host_free < k) {
                // the oldest host resident outside the batch (older than the victim: the
                // availability check above guarantees one exists before vkey)
                while (batch.count(hcur->second))
                    ++hcur;
                plan.host_drops.push_back(hcur->second);
                host_free += (int64_t)c->users[hcur->second].pages.size();
                ++hcur;
            }
            host_free -= k;
            plan.placed = true;
            count_offload += k;
        } else {
            ++count_drop;
        }
        count_drop += (int64_t)plan.host_drops.size();
        plans.push_back(std::move(plan));
    }
    int64_t count_onboard = 0;
    for (int32_t b = 0; b < B; ++b) {
        auto it = c->users.find(ids[b]);
        if (it != c->users.end() && it->second.tier == HSTU_TIER_HOST)
            count_onboard += (int64_t)it->second.pages.size();
    }
    *n_offload = (int32_t)count_offload;
    *n_onboard = (int32_t)count_onboard;
    *n_dropped = (int32_t)count_drop;
    if (count_offload > offload_cap || count_onboard > onboard_cap || count_drop > dropped_cap)
        return HSTU_ERR_OUTPUT_CAPACITY;
    if ((count_offload > 0 && !offload_out) || (count_onboard > 0 && !onboard_out) ||
        (count_drop > 0 && !dropped_out))
        return HSTU_ERR_INVALID_ARG;

    // ---- apply
    const int64_t stamp = ++c->clock;
    int32_t no = 0, nd = 0;
    std::vector<int32_t> gpu_freed, got;
    for (const VictimPlan& plan : plans) {
        for (int64_t hid : plan.host_drops) {
            UserRec& h = c->users[hid];
            c->host_free.give(h.pages);
            c->host_lru.erase({h.stamp, hid});
            c->users.erase(hid);
            dropped_out[nd++] = hid;
        }
        UserRec& v = c->users[plan.id];
        gpu_freed.insert(gpu_freed.end(), v.pages.begin(), v.pages.end());
        c->gpu_lru.erase({v.stamp, plan.id});
        if (!plan.placed) {
            c->users.erase(plan.id);
            dropped_out[nd++] = plan.id;
            continue;
        }
        got.clear();
        c->take(HSTU_TIER_HOST, (int32_t)v.pages.size(), got);
        for (size_t i = 0; i < got.size(); ++i) {
            offload_out[2 * no] = v.pages[i];
            offload_out[2 * no + 1] = got[i];
            ++no;
        }
        v.pages = got;
        v.tier = HSTU_TIER_HOST;
        c->host_lru.insert({v.stamp, plan.id});
    }
    c->gpu_free.give(gpu_freed);

    int32_t nb = 0;
    std::vector<int32_t> host_to_free;
    for (int32_t b = 0; b < B; ++b) {
        auto it = c->users.find(ids[b]);
        if (it == c->users.end()) {
            tier_before_out[b] = HSTU_TIER_MISS;
            it = c->users.emplace(ids[b], UserRec{}).first;
            it->second.tier = HSTU_TIER_GPU;
            c->take(HSTU_TIER_GPU, need[b], it->second.pages);
        } else if (it->second.tier == HSTU_TIER_GPU) {
            tier_before_out[b] = HSTU_TIER_GPU;
            c->gpu_lru.erase({it->second.stamp, ids[b]});
            c->take(HSTU_TIER_GPU, need[b] - (int32_t)it->second.pages.size(), it->second.pages);
        } else {
            tier_before_out[b] = HSTU_TIER_HOST;
            UserRec& u = it->second;
            c->host_lru.erase({u.stamp, ids[b]});
            got.clear();
            c->take(HSTU_TIER_GPU, need[b], got);
            for (size_t i = 0; i < u.pages.size(); ++i) {
                onboard_out[2 * nb] = u.pages[i];
                onboard_out[2 * nb + 1] = got[i];
                ++nb;
            }
            host_to_free.insert(host_to_free.end(), u.pages.begin(), u.pages.end());
            u.pages = got;
            u.tier = HSTU_TIER_GPU;
        }
        UserRec& u = it->second;
        cached_out[b] = u.n;
        u.n += append[b];
        u.stamp = stamp;
        c->gpu_lru.insert({stamp, ids[b]});
        int32_t* row = rows_out + (int64_t)b * c->M;
        for (int32_t j = 0; j < c->M; ++j)
            row[j] = j < (int32_t)u.pages.size() ? u.pages[j] : -1;
    }
    c->host_free.give(host_to_free);
    return HSTU_OK;
}

int hstu_cache_evict(hstu_kv_cache* c, int64_t id, int32_t* tier_out)
{
    if (!c || !tier_out)
        return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    auto it = c->users.find(id);
    if (it == c->users.end()) {
        *tier_out = HSTU_TIER_MISS;
        return HSTU_OK;
    }
    UserRec& u = it->second;
    *tier_out = u.tier;
    c->bitmap(u.tier).give(u.pages);
    c->lru(u.tier).erase({u.stamp, id});
    c->users.erase(it);
    return HSTU_OK;
}

int hstu_cache_compact(hstu_kv_cache* c, int32_t* moves_out, int32_t capacity, int32_t* n_moves)
{
    if (!c || !n_moves || capacity < 0)
        return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    const int32_t live = c->G - c->gpu_free.free_count();
    std::vector<int32_t> dsts;
    c->gpu_free.free_below(live, dsts);
    *n_moves = (int32_t)dsts.size();
    if ((int32_t)dsts.size() > capacity)
        return HSTU_ERR_OUTPUT_CAPACITY;
    if (!dsts.empty() && !moves_out)
        return HSTU_ERR_INVALID_ARG;
    // the live pages at ids >= live, ascending, are the used (not free) ids in [live, G)
    std::vector<int32_t> remap;
    if (!dsts.empty())
        remap.assign((size_t)c->G, -1);
    size_t i = 0;
    for (int32_t p = live; p < c->G && i < dsts.size(); ++p) {
        if (c->gpu_free.is_free(p))
            continue;
        moves_out[2 * i] = p;
        moves_out[2 * i + 1] = dsts[i];
        remap[p] = dsts[i];
        ++i;
    }
    if (!dsts.empty())
        for (auto& kv : c->users)
            if (kv.second.tier == HSTU_TIER_GPU)
                for (int32_t& p : kv.second.pages)
                    if (remap[p] >= 0)
                        p = remap[p];
    c->gpu_free.reset_prefix(live);
    return HSTU_OK;
}

int hstu_cache_page_rows(hstu_kv_cache* c, const int64_t* ids, int32_t n, int32_t* rows_out)
{
    if (!c || n < 0 || (n > 0 && (!ids || !rows_out)))
        return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    for (int32_t i = 0; i < n; ++i) {
        int32_t* row = rows_out + (int64_t)i * c->M;
        auto it = c->users.find(ids[i]);
        const std::vector<int32_t>* pages =
            (it != c->users.end() && it->second.tier == HSTU_TIER_GPU) ? &it->second.pages : nullptr;
        for (int32_t j = 0; j < c->M; ++j)
            row[j] = (pages && j < (int32_t)pages->size()) ? (*pages)[j] : -1;
    }
    return HSTU_OK;
}

int hstu_cache_stats(hstu_kv_cache* c, int64_t* s)
{
    if (!c || !s)
        return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    s[0] = c->gpu_free.free_count();
    s[1] = c->host_free.free_count();
    s[2] = (int64_t)c->gpu_lru.size();
    s[3] = (int64_t)c->host_lru.size();
    s[4] = c->clock;
    return HSTU_OK;
}

}  // extern "C"

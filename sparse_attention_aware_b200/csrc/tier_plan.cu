// Host-side slot planning for a tiered KV cache (no device code).
//
// Method: "语言模型能自己决定该看哪里吗？" (a DA step only hides context, so the
// pages no step reads can wait in an outer tier and come back when a
// declaration names them again) and "百万上下文，模型终于会挑重点了", section
// "对百万上下文产品意味着什么" (the KV cache as tiered storage, focus regions
// loaded on demand).  Before each step the host pages it reads are mapped onto
// a fixed pool of device slots; this runs once per decode step on the host, so
// it is plain C++ over the caller's arrays, O(pages wanted + slots).  The
// library keeps nothing between calls: page marks and working lists live in
// the caller's scratch buffer.
#include <algorithm>

#include "sa.h"

namespace {

// scratch layout (int32 words): [0] mark generation, [1, 1 + host_pages) page
// marks, then four lists of `slots` entries (distinct wanted, missing, slots
// to fill, evictable slots)
struct Scratch {
    uint32_t *gen;
    uint32_t *mark;
    int32_t *distinct, *missing, *cand, *evictable;
};

}  // namespace

extern "C" SA_API int64_t sa_tier_plan_scratch_ints(int64_t host_pages, int32_t slots)
{
    if (host_pages < 1 || slots < 1) return 0;
    return 1 + host_pages + 4 * (int64_t)slots;
}

extern "C" SA_API sa_status sa_tier_plan(int32_t *slot_of, int64_t host_pages, int32_t *page_in,
                                         int64_t *last_use, int32_t slots, int64_t tick, const int32_t *wanted,
                                         int32_t n_wanted, const int32_t *keep, int32_t n_keep, int32_t *pairs,
                                         int32_t *evicted, int32_t *counts, int32_t *scratch, int64_t scratch_ints)
{
    if (!slot_of || !page_in || !last_use || !pairs || !evicted || !counts || !scratch)
        return SA_ERR_INVALID_ARGUMENT;
    if (slots < 1 || host_pages < 1 || n_wanted < 0 || n_keep < 0) return SA_ERR_INVALID_ARGUMENT;
    if (scratch_ints < sa_tier_plan_scratch_ints(host_pages, slots)) return SA_ERR_WORKSPACE;
    if ((n_wanted > 0 && !wanted) || (n_keep > 0 && !keep)) return SA_ERR_INVALID_ARGUMENT;
    for (int32_t i = 0; i < n_wanted; ++i)
        if (wanted[i] < 0 || wanted[i] >= host_pages) return SA_ERR_INVALID_ARGUMENT;
    for (int32_t i = 0; i < n_keep; ++i)
        if (keep[i] < 0 || keep[i] >= host_pages) return SA_ERR_INVALID_ARGUMENT;

    Scratch t;
    t.gen = reinterpret_cast<uint32_t *>(scratch);
    t.mark = t.gen + 1;
    t.distinct = scratch + 1 + host_pages;
    t.missing = t.distinct + slots;
    t.cand = t.missing + slots;
    t.evictable = t.cand + slots;
    // a new mark generation (a zero-filled buffer has never marked anything)
    uint32_t gen = *t.gen + 1;
    if (gen == 0) {
        std::fill(t.mark, t.mark + host_pages, 0u);
        gen = 1;
    }
    *t.gen = gen;
    auto mark = [&](int32_t p) {   // returns whether p was marked already
        const bool was = t.mark[p] == gen;
        t.mark[p] = gen;
        return was;
    };

    // distinct wanted pages in order of first occurrence
    int32_t nd = 0;
    for (int32_t i = 0; i < n_wanted; ++i) {
        if (mark(wanted[i])) continue;
        if (nd == slots) return SA_ERR_CAPACITY;
        t.distinct[nd++] = wanted[i];
    }
    // pages that may not leave their slots: this step's and the step in flight's
    for (int32_t i = 0; i < n_keep; ++i) mark(keep[i]);

    int32_t need = 0;
    for (int32_t i = 0; i < nd; ++i)
        if (slot_of[t.distinct[i]] < 0) t.missing[need++] = t.distinct[i];

    // slots to fill: free ones in ascending order, then the least recently
    // used slots holding a page that is neither wanted nor kept (ties to the
    // lower slot)
    int32_t nc = 0;
    for (int32_t s = 0; s < slots && nc < need; ++s)
        if (page_in[s] < 0) t.cand[nc++] = s;
    if (nc < need) {
        int32_t ne = 0;
        for (int32_t s = 0; s < slots; ++s)
            if (page_in[s] >= 0 && t.mark[page_in[s]] != gen) t.evictable[ne++] = s;
        const int32_t more = need - nc;
        if (ne < more) return SA_ERR_CAPACITY;
        auto older = [&](int32_t x, int32_t y) {
            return last_use[x] < last_use[y] || (last_use[x] == last_use[y] && x < y);
        };
        std::partial_sort(t.evictable, t.evictable + more, t.evictable + ne, older);
        std::copy(t.evictable, t.evictable + more, t.cand + nc);
        nc += more;
    }

    // commit
    for (int32_t i = 0; i < nd; ++i)
        if (slot_of[t.distinct[i]] >= 0) last_use[slot_of[t.distinct[i]]] = tick;
    int32_t m = 0;
    for (int32_t i = 0; i < need; ++i) {
        const int32_t s = t.cand[i], p = t.missing[i], old = page_in[s];
        if (old >= 0) {
            slot_of[old] = -1;
            evicted[m++] = old;
        }
        page_in[s] = p;
        slot_of[p] = s;
        last_use[s] = tick;
        pairs[2 * i] = p;
        pairs[2 * i + 1] = s;
    }
    counts[0] = need;
    counts[1] = m;
    counts[2] = nd - need;
    counts[3] = nd;
    return SA_OK;
}

// Host-side slot planning for a tiered KV cache (no device code).
//
// Method: "语言模型能自己决定该看哪里吗？" (a DA step only hides context, so the
// pages no step reads can wait in an outer tier and come back when a
// declaration names them again) and "百万上下文，模型终于会挑重点了", section
// "对百万上下文产品意味着什么" (the KV cache as tiered storage, focus regions
// loaded on demand).  Before each step the host pages it reads are mapped onto
// a fixed pool of device slots; this runs once per decode step on the host, so
// it is plain C++ over the caller's state arrays: O(pages wanted + slots), no
// allocation after the first call of a thread.
#include <algorithm>
#include <vector>

#include "sa.h"

namespace {

// Generation-stamped marks over host pages (one array per host thread).
struct PageMarks {
    std::vector<uint32_t> stamp;
    uint32_t gen = 0;
    void begin(size_t n)
    {
        if (stamp.size() < n) {
            stamp.assign(n, 0u);
            gen = 0;
        }
        if (++gen == 0) {   // wrapped: clear once
            std::fill(stamp.begin(), stamp.end(), 0u);
            gen = 1;
        }
    }
    bool marked(size_t p) const { return stamp[p] == gen; }
    bool mark(size_t p)   // returns whether p was marked already
    {
        const bool was = stamp[p] == gen;
        stamp[p] = gen;
        return was;
    }
};

struct PlanScratch {
    PageMarks marks;
    std::vector<int32_t> distinct, missing, cand, evictable;
};

thread_local PlanScratch t_scratch;

}  // namespace

extern "C" SA_API sa_status sa_tier_plan(int32_t *slot_of, int64_t host_pages, int32_t *page_in,
                                         int64_t *last_use, int32_t slots, int64_t tick, const int32_t *wanted,
                                         int32_t n_wanted, const int32_t *keep, int32_t n_keep, int32_t *pairs,
                                         int32_t *evicted, int32_t *counts)
{
    if (!slot_of || !page_in || !last_use || !pairs || !evicted || !counts) return SA_ERR_INVALID_ARGUMENT;
    if (slots < 1 || host_pages < 1 || n_wanted < 0 || n_keep < 0) return SA_ERR_INVALID_ARGUMENT;
    if ((n_wanted > 0 && !wanted) || (n_keep > 0 && !keep)) return SA_ERR_INVALID_ARGUMENT;
    for (int32_t i = 0; i < n_wanted; ++i)
        if (wanted[i] < 0 || wanted[i] >= host_pages) return SA_ERR_INVALID_ARGUMENT;
    for (int32_t i = 0; i < n_keep; ++i)
        if (keep[i] < 0 || keep[i] >= host_pages) return SA_ERR_INVALID_ARGUMENT;

    PlanScratch &t = t_scratch;
    t.marks.begin((size_t)host_pages);
    // distinct wanted pages in order of first occurrence
    t.distinct.clear();
    for (int32_t i = 0; i < n_wanted; ++i)
        if (!t.marks.mark((size_t)wanted[i])) t.distinct.push_back(wanted[i]);
    if ((int64_t)t.distinct.size() > slots) return SA_ERR_CAPACITY;
    // pages that may not leave their slots: this step's and the step in flight's
    for (int32_t i = 0; i < n_keep; ++i) t.marks.mark((size_t)keep[i]);

    t.missing.clear();
    for (const int32_t p : t.distinct)
        if (slot_of[p] < 0) t.missing.push_back(p);
    const size_t need = t.missing.size();

    // slots to fill: free ones in ascending order, then the least recently
    // used slots holding a page that is neither wanted nor kept (ties to the
    // lower slot)
    t.cand.clear();
    for (int32_t s = 0; s < slots && t.cand.size() < need; ++s)
        if (page_in[s] < 0) t.cand.push_back(s);
    if (t.cand.size() < need) {
        t.evictable.clear();
        for (int32_t s = 0; s < slots; ++s)
            if (page_in[s] >= 0 && !t.marks.marked((size_t)page_in[s])) t.evictable.push_back(s);
        const size_t more = need - t.cand.size();
        if (t.evictable.size() < more) return SA_ERR_CAPACITY;
        auto older = [&](int32_t x, int32_t y) {
            return last_use[x] < last_use[y] || (last_use[x] == last_use[y] && x < y);
        };
        std::partial_sort(t.evictable.begin(), t.evictable.begin() + (ptrdiff_t)more, t.evictable.end(), older);
        t.cand.insert(t.cand.end(), t.evictable.begin(), t.evictable.begin() + (ptrdiff_t)more);
    }

    // commit
    for (const int32_t p : t.distinct)
        if (slot_of[p] >= 0) last_use[slot_of[p]] = tick;
    int32_t m = 0;
    for (size_t i = 0; i < need; ++i) {
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
    counts[0] = (int32_t)need;
    counts[1] = m;
    counts[2] = (int32_t)(t.distinct.size() - need);
    counts[3] = (int32_t)t.distinct.size();
    return SA_OK;
}

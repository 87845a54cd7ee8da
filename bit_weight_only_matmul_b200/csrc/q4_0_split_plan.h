// q4_0_split_plan.h -- the host-side plan of the decode kernel's split mode,
// free of CUDA so that the CPU tests can check it.
//
// A launch of few items (128 weight rows x all K of one problem each) runs
// its CTAs in clusters of cl.  Items of at least cl stages that are longer
// than the mean load of a CTA are cut into cl pieces, one per CTA of a
// cluster (rank r takes stages piece_begin(n, r, cl) .. piece_begin(n, r+1,
// cl) - 1), and dealt to the clusters; the other items stay whole and are
// dealt to single CTAs.  Every deal puts the next item, longest first, onto
// the least loaded cluster or CTA.  Each CTA's list holds its cluster's split
// items first, in the same order on every CTA of the cluster (their partial
// sums meet in rank 0), then its own whole items.
#pragma once

#include <algorithm>
#include <cstdint>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#if defined(__CUDACC__)
#define Q4_SPLIT_HD __host__ __device__
#else
#define Q4_SPLIT_HD
#endif

namespace q4split {

constexpr int kMaxItems = 1024;              // items per launch in split mode
constexpr int kMaxSplitCtas = 256;           // CTAs per launch in split mode
constexpr int kMaxSched = 2 * kMaxItems;     // schedule entries per launch
constexpr uint16_t kSplitFlag = 0x8000;      // entry flag: a piece of a split item

// First stage of piece r (0 <= r <= cl) of an n-stage item cut into cl
// pieces: ceil(n r / cl).  Pieces differ in length by at most one, and none
// is empty when n >= cl.
Q4_SPLIT_HD inline int piece_begin(int n, int r, int cl) { return (n * r + cl - 1) / cl; }

// One problem as the plan sees it: items item_begin .. item_begin + items - 1,
// each of `stages` stages.  Problems come sorted by stages, largest first.
struct PlanProblem {
    int stages, item_begin, items;
};

struct Schedule {
    std::vector<std::vector<uint16_t>> split_of;   // per cluster: its split items
    std::vector<std::vector<uint16_t>> whole_of;   // per CTA: its whole items
    long max_load = 0;                             // stages on the busiest CTA
    int entries = 0;                               // list entries over all CTAs
};

inline void plan(const PlanProblem *p, int count, int clusters, int cl, Schedule &out) {
    const int ctas = cl * clusters;
    long total = 0;
    for (int i = 0; i < count; ++i) total += static_cast<long>(p[i].items) * p[i].stages;
    const long mean = (total + ctas - 1) / ctas;
    auto is_split = [&](int n) { return n >= cl && n > mean; };
    using Load = std::pair<long, int>;
    out.split_of.assign(clusters, {});
    out.whole_of.assign(ctas, {});
    out.entries = 0;
    std::vector<long> load(ctas, 0);
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> cq;
    for (int c = 0; c < clusters; ++c) cq.push({0, c});
    for (int i = 0; i < count; ++i) {
        const int n = p[i].stages;
        if (!is_split(n)) continue;
        for (int k = 0; k < p[i].items; ++k) {
            Load l = cq.top();
            cq.pop();
            out.split_of[l.second].push_back(static_cast<uint16_t>(p[i].item_begin + k));
            out.entries += cl;
            l.first += (n + cl - 1) / cl;
            for (int r = 0; r < cl; ++r) load[cl * l.second + r] = l.first;
            cq.push(l);
        }
    }
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> tq;
    for (int b = 0; b < ctas; ++b) tq.push({load[b], b});
    for (int i = 0; i < count; ++i) {
        const int n = p[i].stages;
        if (is_split(n)) continue;
        for (int k = 0; k < p[i].items; ++k) {
            Load l = tq.top();
            tq.pop();
            out.whole_of[l.second].push_back(static_cast<uint16_t>(p[i].item_begin + k));
            ++out.entries;
            l.first += n;
            load[l.second] = l.first;
            tq.push(l);
        }
    }
    out.max_load = ctas > 0 ? *std::max_element(load.begin(), load.end()) : 0;
}

// The CTAs' lists: CTA b runs sched[begin[b] .. begin[b+1]).  begin holds
// cl * clusters + 1 entries, sched holds sc.entries; returns sc.entries.
inline int write(const Schedule &sc, int clusters, int cl, uint16_t *begin, uint16_t *sched) {
    const int ctas = cl * clusters;
    int pos = 0;
    for (int b = 0; b < ctas; ++b) {
        begin[b] = static_cast<uint16_t>(pos);
        for (uint16_t it : sc.split_of[b / cl]) sched[pos++] = static_cast<uint16_t>(it | kSplitFlag);
        for (uint16_t it : sc.whole_of[b]) sched[pos++] = it;
    }
    begin[ctas] = static_cast<uint16_t>(pos);
    return pos;
}

}  // namespace q4split

// CPU checks of the decode kernel's split-mode plan (csrc/q4_0_split_plan.h),
// walked the way the kernel walks it: CTA b is rank b % cl of its cluster,
// runs the entries of its list in order, and of a split n-stage item takes
// stages piece_begin(n, rank, cl) .. piece_begin(n, rank + 1, cl) - 1.
//
// For every case: every stage of every item is worked exactly once; no piece
// is empty; the split items of a cluster open the list of each of its CTAs,
// in the same order; the loads the walk gives stay within the plan's
// max_load, which stays within greedy list scheduling's bound (planned work
// per CTA + the costliest single deal).  Prints "ok <cases>" or the first
// failure, and exits non-zero on a failure.
#include <algorithm>
#include <cstdio>
#include <functional>
#include <random>
#include <string>
#include <vector>

#include "q4_0_split_plan.h"

namespace {

struct Case {
    std::string name;
    std::vector<std::pair<int, int>> probs;   // (stages, items), stages non-increasing
    int clusters, cl;
};

bool fail(const Case &c, const char *what, long a = 0, long b = 0) {
    std::printf("FAIL %s (clusters %d, cl %d): %s [%ld, %ld]\n", c.name.c_str(), c.clusters, c.cl, what, a, b);
    return false;
}

// false on a failed check; *skipped when the launcher would not split this case
bool check(const Case &c, bool *skipped) {
    *skipped = false;
    std::vector<q4split::PlanProblem> pp;
    std::vector<int> stages_of;   // per item
    int items = 0;
    for (const auto &pr : c.probs) {
        pp.push_back({pr.first, items, pr.second});
        for (int k = 0; k < pr.second; ++k) stages_of.push_back(pr.first);
        items += pr.second;
    }
    if (items > q4split::kMaxItems || c.cl * c.clusters > q4split::kMaxSplitCtas) {
        *skipped = true;
        return true;
    }
    q4split::Schedule sc;
    q4split::plan(pp.data(), static_cast<int>(pp.size()), c.clusters, c.cl, sc);
    if (sc.entries > q4split::kMaxSched) {   // the launcher falls back to plain mode
        *skipped = true;
        return true;
    }
    const int ctas = c.cl * c.clusters;
    std::vector<uint16_t> begin(ctas + 1), sched(std::max(sc.entries, 1));
    const int n = q4split::write(sc, c.clusters, c.cl, begin.data(), sched.data());
    if (n != sc.entries || begin[ctas] != n) return fail(c, "entry count", n, sc.entries);

    std::vector<std::vector<int>> cover(items);
    for (int i = 0; i < items; ++i) cover[i].assign(stages_of[i], 0);
    long walked_max = 0, planned_total = 0, costliest = 0;
    for (int b = 0; b < ctas; ++b) {
        if (begin[b] > begin[b + 1]) return fail(c, "list bounds", begin[b], begin[b + 1]);
        const int rank = b % c.cl;
        long load = 0;
        bool whole_seen = false;
        for (int e = begin[b]; e < begin[b + 1]; ++e) {
            const int item = sched[e] & (q4split::kSplitFlag - 1);
            const bool split = (sched[e] & q4split::kSplitFlag) != 0;
            if (item >= items) return fail(c, "item index", item, items);
            const int ns = stages_of[item];
            int s0 = 0, s1 = ns;
            if (split) {
                if (whole_seen) return fail(c, "split entry after a whole one", b, e);
                if (ns < c.cl) return fail(c, "split item shorter than the cluster", ns, c.cl);
                s0 = q4split::piece_begin(ns, rank, c.cl);
                s1 = q4split::piece_begin(ns, rank + 1, c.cl);
                // every CTA of the cluster lists the same split item at the same place
                const int b0 = b - rank;
                for (int r = 0; r < c.cl; ++r) {
                    const int other = begin[b0 + r] + (e - begin[b]);
                    if (other >= begin[b0 + r + 1] || sched[other] != sched[e])
                        return fail(c, "split lists differ across the cluster", b, r);
                }
            } else {
                whole_seen = true;
            }
            if (s1 <= s0) return fail(c, "empty piece", s0, s1);
            for (int s = s0; s < s1; ++s) ++cover[item][s];
            load += s1 - s0;
        }
        walked_max = std::max(walked_max, load);
    }
    for (int i = 0; i < items; ++i)
        for (int s = 0; s < stages_of[i]; ++s)
            if (cover[i][s] != 1) return fail(c, "stage not worked exactly once", i, cover[i][s]);

    // planned work: a split item costs ceil(n/cl) on each CTA of its cluster
    for (int b = 0; b < c.clusters; ++b)
        for (uint16_t it : sc.split_of[b]) {
            const long cost = (stages_of[it] + c.cl - 1) / c.cl;
            planned_total += cost * c.cl;
            costliest = std::max(costliest, cost);
        }
    for (int b = 0; b < ctas; ++b)
        for (uint16_t it : sc.whole_of[b]) {
            planned_total += stages_of[it];
            costliest = std::max<long>(costliest, stages_of[it]);
        }
    if (walked_max > sc.max_load) return fail(c, "walk exceeds the planned max load", walked_max, sc.max_load);
    const long bound = (planned_total + ctas - 1) / ctas + costliest;
    if (sc.max_load > bound) return fail(c, "max load above the list-scheduling bound", sc.max_load, bound);
    return true;
}

// decoder-layer linear sets at 256 k per stage and 128 rows per item
const std::vector<std::pair<int, int>> kLayer = {{32, 24}, {12, 40}, {12, 24}, {12, 128}};

}  // namespace

int main() {
    std::vector<Case> cases;
    cases.push_back({"layer", kLayer, 74, 2});
    cases.push_back({"layer, fewer clusters", kLayer, 60, 2});
    std::vector<std::pair<int, int>> flow = {{32, 72}, {12, 120}, {12, 72}, {12, 384}};
    cases.push_back({"flow head", flow, 74, 2});
    for (int cl : {4, 6, 8})
        for (int clusters : {14, 18, 20, 24, 37})
            if (cl * clusters <= 148) {
                cases.push_back({"gemv", {{12, 24}}, clusters, cl});
                cases.push_back({"grouped few items", {{32, 2}, {8, 1}, {7, 8}, {1, 3}}, clusters, cl});
            }
    cases.push_back({"one item shorter than the cluster", {{3, 1}}, 1, 4});
    cases.push_back({"one item, pieces of one", {{6, 1}}, 1, 6});
    cases.push_back({"uneven pieces", {{7, 8}}, 8, 4});

    std::mt19937 rng(12345);
    for (int t = 0; t < 400; ++t) {
        const int cl = std::vector<int>{2, 4, 6, 8}[rng() % 4];
        const int clusters = 1 + static_cast<int>(rng() % (q4split::kMaxSplitCtas / cl));
        const int count = 1 + static_cast<int>(rng() % 8);
        std::vector<int> st;
        for (int i = 0; i < count; ++i) st.push_back(1 + static_cast<int>(rng() % 40));
        std::sort(st.begin(), st.end(), std::greater<int>());
        std::vector<std::pair<int, int>> probs;
        for (int s : st) probs.push_back({s, 1 + static_cast<int>(rng() % 150)});
        cases.push_back({"random " + std::to_string(t), probs, clusters, cl});
    }

    int checked = 0;
    for (const Case &c : cases) {
        bool skipped = false;
        if (!check(c, &skipped)) return 1;
        checked += skipped ? 0 : 1;
    }
    std::printf("ok %d\n", checked);
    return checked > 0 ? 0 : 1;
}

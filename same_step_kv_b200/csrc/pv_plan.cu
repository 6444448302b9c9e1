// Host-side work planner for the attention kernel.
//
// One CTA computes one unit: two 128-row query tiles of one (stream, head)
// against a contiguous range of 128-key tiles.  When there are too few query
// blocks to fill the GPU (one 880-token chunk has 4 query blocks per head, 96
// over 24 heads, against 148 SMs), the key range of each block is split and
// the parts are merged by the last CTA to finish (split-KV).  The planner
// picks the split counts by simulating the hardware's greedy dispatch of CTAs
// in grid order on n_sm SMs and keeping the plan with the shortest makespan.
#include <algorithm>
#include <map>
#include <mutex>
#include <queue>
#include <vector>

#include "pv_internal.h"

namespace pv {
namespace {

// Relative cost of one unit: key tiles times the query tiles it carries
// (a lone tile cannot overlap its softmax with a second tile's MMAs, so it
// costs more than half), plus a fixed prologue/epilogue charge and the merge.
double unit_cost(int tiles, bool two_tiles, bool split) {
    return tiles * (two_tiles ? 2.0 : 1.3) + 6.0 + (split ? 3.0 : 0.0);
}

struct Cand {
    std::vector<int> n_split;
    double makespan;
    long long units;
};

double simulate(const AttnStreamDesc* st, const int* order, int n_streams, int heads, int n_sm,
                const std::vector<int>& n_split) {
    std::priority_queue<double, std::vector<double>, std::greater<double>> sm;
    for (int i = 0; i < n_sm; ++i) sm.push(0.0);
    double makespan = 0;
    for (int oi = 0; oi < n_streams; ++oi) {
        const int i = order[oi];
        const AttnStreamDesc& s = st[i];
        const int ns = n_split[i];
        for (int h = 0; h < heads; ++h)
            for (int qb = 0; qb < s.n_qb; ++qb) {
                const bool two = s.n_q - qb * kQBlock > kQRows;
                for (int sp = 0; sp < ns; ++sp) {
                    const int tiles = (sp + 1) * s.n_kt / ns - sp * s.n_kt / ns;
                    const double t = sm.top() + unit_cost(tiles, two, ns > 1);
                    sm.pop();
                    sm.push(t);
                    makespan = std::max(makespan, t);
                }
            }
    }
    return makespan;
}

struct PlanKey {
    std::vector<int> shape;  // heads, n_sm, caps, then (n_q, n_k) per stream
    bool operator<(const PlanKey& o) const { return shape < o.shape; }
};

std::mutex g_plan_mu;
std::map<PlanKey, std::vector<int>> g_plan_cache;

}  // namespace

int plan_attention(AttnStreamDesc* st, int n_streams, int heads, int n_sm, int part_capacity,
                   int cnt_capacity, int* order) {
    long long base_units = 0, counters = 0;
    for (int i = 0; i < n_streams; ++i) {
        st[i].n_qb = (st[i].n_q + kQBlock - 1) / kQBlock;
        st[i].n_kt = (st[i].n_k + kKeyTile - 1) / kKeyTile;
        base_units += (long long)heads * st[i].n_qb;
        counters += (long long)heads * st[i].n_qb * kQTilesPerCta;
    }
    if (counters > cnt_capacity) return -1;
    // Longest units first, so that the greedy dispatch approximates LPT.
    for (int i = 0; i < n_streams; ++i) order[i] = i;
    std::stable_sort(order, order + n_streams,
                     [&](int a, int b) { return st[a].n_kt > st[b].n_kt; });

    PlanKey key;
    key.shape = {heads, n_sm, part_capacity, cnt_capacity};
    for (int i = 0; i < n_streams; ++i) {
        key.shape.push_back(st[i].n_q);
        key.shape.push_back(st[i].n_k);
    }
    std::vector<int> best;
    {
        std::lock_guard<std::mutex> lock(g_plan_mu);
        auto it = g_plan_cache.find(key);
        if (it != g_plan_cache.end()) best = it->second;
    }
    if (best.empty()) {
        best.assign(n_streams, 1);
        // With at least two full waves of unsplit units, splitting only adds merges.
        if (base_units < 2LL * n_sm) {
            int max_kt = 0;
            for (int i = 0; i < n_streams; ++i) max_kt = std::max(max_kt, st[i].n_kt);
            double best_t = simulate(st, order, n_streams, heads, n_sm, best);
            for (int n = 2; n <= kMaxSplit; ++n) {
                const int target = (max_kt + n - 1) / n;  // key tiles per part
                if (target < 4) break;
                std::vector<int> cand(n_streams);
                long long parts = 0;
                for (int i = 0; i < n_streams; ++i) {
                    cand[i] = std::min(std::max(1, (st[i].n_kt + target - 1) / target), kMaxSplit);
                    cand[i] = std::min(cand[i], st[i].n_kt);
                    if (cand[i] > 1) parts += (long long)heads * st[i].n_qb * kQTilesPerCta * cand[i];
                }
                if (parts > part_capacity) break;
                const double t = simulate(st, order, n_streams, heads, n_sm, cand);
                if (t < best_t * 0.98) {
                    best_t = t;
                    best = cand;
                }
            }
        }
        std::lock_guard<std::mutex> lock(g_plan_mu);
        if (g_plan_cache.size() > 256) g_plan_cache.clear();
        g_plan_cache[key] = best;
    }
    int unit = 0, part = 0, cnt = 0;
    for (int oi = 0; oi < n_streams; ++oi) {
        const int i = order[oi];
        st[i].n_split = best[i];
        st[i].unit0 = unit;
        unit += heads * st[i].n_qb * st[i].n_split;
    }
    for (int i = 0; i < n_streams; ++i) {
        st[i].cnt0 = cnt;
        cnt += heads * st[i].n_qb * kQTilesPerCta;
        st[i].part0 = part;
        if (st[i].n_split > 1) part += heads * st[i].n_qb * kQTilesPerCta * st[i].n_split;
    }
    if (part > part_capacity) return -1;
    return unit;
}

}  // namespace pv

// Host-side work planner for the attention kernel.
//
// The work of one launch is a list of items, one per (stream, head, 256-row
// query block), each a run of n_kt 128-key tiles.  Within a stream the items
// are laid out query-block-major (all heads of block 0, then block 1, ...),
// so that CTAs working on the same head's blocks at the same time share the
// K/V tiles through L2.  Laid end to end the items form `total` key tiles,
// and CTA c of `grid` takes one contiguous range of them.  Two ways to
// choose the ranges:
//  - stream-K: bounds[c] = c * total / grid.  Every SM gets the same number
//    of key tiles whatever the mix of lengths; an item that straddles CTAs
//    is finished by the last of them to arrive, which merges the parts.  A
//    CTA holds at most two partial parts (its first and its last segment) per
//    query tile, so the partial workspace is 4 slots per CTA.
//  - item-aligned: every bound is an item boundary, so no item is split and
//    nothing is merged; the boundaries are placed as near the stream-K ones
//    as the items allow (a table of first items, 16-bit to keep the kernel
//    parameters small; beyond 65,535 items, equal item counts).  Used when items are short next to a CTA's share
//    (then rounding to items costs little and merges would cost more), or
//    when the workspace has no room for the partials.
#include <algorithm>
#include <vector>

#include "pv_internal.h"

namespace pv {

constexpr long long kItemOverhead = 1;  // key-tile equivalents of one segment's fixed work

int plan_attention(AttnParams& p, int n_sm, int part_capacity, int cnt_capacity) {
    long long total = 0;
    int items = 0, max_kt = 0;
    for (int i = 0; i < p.n_streams; ++i) {
        AttnStreamDesc& s = p.st[i];
        s.n_qb = (s.n_q + kQBlock - 1) / kQBlock;
        s.n_kt = (s.n_k + kKeyTile - 1) / kKeyTile;
        s.item0 = items;
        s.cost0 = total;
        items += p.heads * s.n_qb;
        total += (long long)p.heads * s.n_qb * s.n_kt;
        if (s.n_qb > 0) max_kt = std::max(max_kt, s.n_kt);
    }
    if ((long long)items * kQTilesPerCta > cnt_capacity || total <= 0) return -1;
    const int sms = std::max(1, std::min(n_sm, kMaxGrid));
    p.total = total;
    p.n_items = items;
    const long long grid_sk = std::min<long long>(sms, total);
    const bool short_items = total / grid_sk >= 2LL * max_kt;
    if (4 * grid_sk <= part_capacity && !short_items) {
        p.item_aligned = 0;
        p.grid = (int)grid_sk;
        return p.grid;
    }
    p.grid = std::min(sms, items);
    if (items > 0xFFFF) {
        p.item_aligned = 2;  // equal item counts, computed on the device
        return p.grid;
    }
    // item-aligned: each CTA starts at the item whose start is nearest its
    // share of the cost, keeping at least one item per CTA.  An item costs
    // its key tiles plus kItemOverhead: a segment's fixed work (Q load,
    // first-tile softmax, output) measures at about one key-tile iteration.
    p.item_aligned = 1;
    std::vector<long long> start;  // cost before item k
    start.reserve(items + 1);
    long long cost = 0;
    for (int i = 0; i < p.n_streams; ++i)
        for (int k = 0; k < p.heads * p.st[i].n_qb; ++k) {
            start.push_back(cost);
            cost += p.st[i].n_kt + kItemOverhead;
        }
    start.push_back(cost);
    int prev = 0;
    p.first_item[0] = 0;
    for (int c = 1; c < p.grid; ++c) {
        const long long want = (long long)c * cost / p.grid;
        int k = (int)(std::lower_bound(start.begin(), start.end(), want) - start.begin());
        if (k > 0 && want - start[k - 1] < start[k] - want) --k;
        k = std::max(k, prev + 1);
        k = std::min(k, items - (p.grid - c));
        p.first_item[c] = (uint16_t)k;
        prev = k;
    }
    p.first_item[p.grid] = (uint16_t)items;
    return p.grid;
}

}  // namespace pv

// Host-side work planner for the attention kernel.
//
// The work of one launch is a list of items, one per (stream, head, 256-row
// query block), each a run of n_kt 128-key tiles.  Within a stream the items
// are laid out query-block-major (all heads of block 0, then block 1, ...),
// so that CTAs working on the same head's blocks at the same time share the
// K/V tiles through L2.  Laid end to end the items form `total` key tiles.
// Two ways to share them out:
//  - stream-K: CTA c of `grid` takes the key tiles [c * total / grid,
//    (c + 1) * total / grid).  Every SM gets the same number of key tiles
//    whatever the mix of lengths; an item that straddles CTAs is finished by
//    the last of them to arrive, which merges the parts.  A CTA holds at
//    most two partial parts (its first and its last segment) per query tile,
//    so the partial workspace is 4 slots per CTA.
//  - whole items at run time: each CTA's producer takes the next item from
//    a counter in global memory (atomicAdd) and hands it to the CTA's other
//    warps, until the list is exhausted; nothing is split or merged.  The
//    streams are put in decreasing order of key tiles first, so the longest
//    items go first and the short ones fill in at the end (the longest-first
//    list schedule).  Used when items are short next to a CTA's share (a
//    static cut into whole items then leaves CTAs up to an item apart: the
//    fixed cost of an item is ~1.6 key-tile iterations, so short items are
//    uneven), or when the workspace has no room for the partials.
#include <algorithm>
#include <vector>

#include "pv_internal.h"

namespace pv {

int plan_attention(AttnParams& p, int n_sm, int part_capacity, int cnt_capacity) {
    auto lay_out = [&]() {
        long long total = 0;
        int items = 0;
        for (int i = 0; i < p.n_streams; ++i) {
            AttnStreamDesc& s = p.st[i];
            s.n_qb = (s.n_q + kQBlock - 1) / kQBlock;
            s.n_kt = (s.n_k + kKeyTile - 1) / kKeyTile;
            s.item0 = items;
            s.cost0 = total;
            items += p.heads * s.n_qb;
            total += (long long)p.heads * s.n_qb * s.n_kt;
        }
        p.n_items = items;
        p.total = total;
    };
    lay_out();
    int max_kt = 0;
    for (int i = 0; i < p.n_streams; ++i)
        if (p.st[i].n_qb > 0) max_kt = std::max(max_kt, p.st[i].n_kt);
    const long long items = p.n_items, total = p.total;
    if (std::max<long long>(items * kQTilesPerCta, 2) > cnt_capacity || total <= 0) return -1;
    const int sms = std::max(1, std::min(n_sm, kMaxGrid));
    const long long grid_sk = std::min<long long>(sms, total);
    const bool short_items = total / grid_sk >= 2LL * max_kt;
    if (4 * grid_sk <= part_capacity && !short_items) {
        p.item_aligned = 0;
        p.grid = (int)grid_sk;
        return p.grid;
    }
    // whole items at run time, longest streams first
    std::stable_sort(p.st, p.st + p.n_streams, [](const AttnStreamDesc& a, const AttnStreamDesc& b) {
        return a.n_kt > b.n_kt;
    });
    lay_out();
    p.item_aligned = 1;
    p.grid = (int)std::min<long long>(sms, items);
    return p.grid;
}

}  // namespace pv

// Host-side work planner for the attention kernel: a stream-K schedule.
//
// The work of one launch is a list of items, one per (stream, head, 256-row
// query block), each a run of n_kt 128-key tiles.  Laid end to end they
// form total = sum(n_kt) key tiles; CTA c of `grid` (one per SM) takes the
// contiguous range [c*total/grid, (c+1)*total/grid).  Every SM therefore
// gets the same number of key tiles whatever the mix of chunk lengths, and an
// item that straddles CTAs is finished by the last of them to arrive, which
// merges the parts.  A CTA holds at most two partial parts (its first and its
// last segment) per query tile, so the partial workspace is 4 slots per CTA.
#include <algorithm>

#include "pv_internal.h"

namespace pv {

int plan_attention(AttnParams& p, int n_sm, int part_capacity, int cnt_capacity) {
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
    if ((long long)items * kQTilesPerCta > cnt_capacity || total <= 0) return -1;
    const int sms = std::max(1, std::min(n_sm, kMaxGrid));
    p.total = total;
    p.n_items = items;
    const long long grid = std::min<long long>(sms, total);
    if (4 * grid <= part_capacity) {
        p.item_aligned = 0;
        p.grid = (int)grid;
    } else {
        p.item_aligned = 1;
        p.grid = std::min(sms, items);
    }
    return p.grid;
}

}  // namespace pv

// eva_vq_plan.h -- the grid of lookup-path calls flagged independent
// (host-only, plain C++17: the CPU tests compile it with g++).
//
// A call that waits for its predecessor is planned for latency: Gs slice
// groups (one thread-block cluster) x Gt row groups, every cluster resident
// in one wave.  Calls flagged independent overlap with their neighbours, so a
// layer costs the CTA slots it holds times how long it holds them, and every
// CTA pays the same fixed part (x~ staging, image build, cluster reduction)
// whatever its share of the work.  Their grid therefore
//   - uses clusters of at most 8 CTAs: half the latency plan's Gs when it is
//     larger (8-CTA clusters fill 144 of a B200's 148 SMs, 16-CTA clusters
//     112);
//   - takes as few row groups as a preferred per-CTA tile count allows
//     (`soft_tiles`), never more tiles per CTA than the running-sum layout
//     holds (`hard_tiles`);
//   - never has more CTAs than the latency plan;
//   - fits the footprint budget `fit` (two CTAs per SM, or the latency
//     plan's own footprint when that is larger).
#pragma once
#include <algorithm>
#include <cstddef>

namespace eva {

// smem(tiles, gs): dynamic shared memory of one CTA with `tiles` row tiles in
// clusters of gs.  On success writes the grid and its footprint and returns
// true; returns false (keep the latency plan) when no grid qualifies.
template <typename SmemFn>
bool independent_grid(int T, int lat_gs, int lat_gt, int hard_tiles, int soft_tiles, size_t fit, SmemFn smem,
                      int *gs_out, int *gt_out, size_t *smem_out) {
    if (T < 1 || lat_gs < 1 || lat_gt < 1 || hard_tiles < 1 || soft_tiles < 1) return false;
    const int gs = lat_gs > 8 ? (lat_gs + 1) / 2 : lat_gs;
    const int gt_hi = std::min(T, std::max(1, lat_gs * lat_gt / gs));
    const int gt_hard = (T + hard_tiles - 1) / hard_tiles;
    int gt = std::max((T + soft_tiles - 1) / soft_tiles, gt_hard);
    if (gt > gt_hi) gt = std::max(gt_hi, gt_hard);
    for (; gt <= gt_hi; ++gt) {
        const size_t sm = smem((T + gt - 1) / gt, gs);
        if (sm <= fit) {
            *gs_out = gs;
            *gt_out = gt;
            *smem_out = sm;
            return true;
        }
    }
    return false;
}

}  // namespace eva

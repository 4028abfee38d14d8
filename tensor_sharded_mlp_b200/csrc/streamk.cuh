// streamk.cuh -- even split of a weight stream over the CTAs of a grid.
//
// A packed weight part is a sequence of (tile, k-block) blocks, tile-major,
// which the tile-blocked layout stores in exactly that order.  Iteration
// it = tile * KB + kb.  CTA c of G processes iterations
// [c * total / G, (c + 1) * total / G): one contiguous run of memory of
// (almost) the same length for every CTA.  A tile whose iterations fall to
// several CTAs is "split": each writes its fp32 partial sums to its own slot
// and the last one to arrive (one atomic counter per tile; nobody waits) adds
// the slots in slot order -- a fixed order, so results are deterministic.
#pragma once

#include <algorithm>

namespace tpmlp {

__host__ __device__ __forceinline__ long long share_begin(long long c, long long total, long long G) {
    return c * total / G;
}
// CTA whose share holds iteration `it`.
__host__ __device__ __forceinline__ int share_owner(long long it, long long total, long long G) {
    return (int)(((it + 1) * G - 1) / total);
}

struct StreamKGeom {
    int tiles, KB, grid, slots;   // slots: most CTAs sharing one tile
    long long total;
};

inline StreamKGeom streamk_geom(long long tiles, long long KB, int max_grid) {
    StreamKGeom g;
    g.tiles = (int)tiles;
    g.KB = (int)KB;
    g.total = tiles * KB;
    g.grid = (int)std::min<long long>(max_grid, g.total);
    g.slots = 1;
    for (long long t = 0; t < tiles; ++t) {
        const int c0 = share_owner(t * KB, g.total, g.grid);
        const int c1 = share_owner(t * KB + KB - 1, g.total, g.grid);
        g.slots = std::max(g.slots, c1 - c0 + 1);
    }
    return g;
}

}  // namespace tpmlp

// Grouped launches of the streaming kernels: several units (matrix batches of
// different shapes, one format) in one launch, so a model's small
// projections share one wave of resident blocks instead of paying a launch's
// ramp-up and tail each.
//
// Every unit gets a range of the launch's 1-D block index: its column tiles
// (cblocks, each `cw` unit columns wide, cw <= blockDim.x) times its row
// blocks (rblocks of rpb rows).  The resident blocks of one wave are split
// over the units so that the longest block, in rows, is as short as it can be.
#pragma once
#include "walk.cuh"

namespace tq {

constexpr int BATCH_MAX = TQ_MAX_BATCH;

struct BatchSlot {
    int64_t block0;    // first block of the unit
    int64_t cblocks;   // column tiles
    int64_t cw;        // unit columns per tile
    int64_t rblocks;   // row blocks
    int64_t rpb;       // rows per row block
};

// `cols[i]` unit columns and `rows[i]` rows (all matrices' rows, flattened)
// of unit i; `slots` = blocks of one wave.  Returns the block count and the
// widest tile (the launch's blockDim.x, a multiple of 32).  Every unit gets at
// least one row block per column tile; the count is at most `slots` when
// that leaves room for it.
inline int64_t batch_split(int n, const int64_t* cols, const int64_t* rows, int64_t slots, BatchSlot* out,
                           int64_t* width) {
    // Tiles of at most `best` columns, balanced within each unit; the block
    // is as wide as the widest unit's tile, so narrower tiles idle lanes.
    // One unit: best = 256.  Several: the widest `best` (a multiple of 32)
    // whose idle lanes, over all units' rows, are within 3 % of the fewest.
    auto tile = [&](int64_t w, int i, int64_t* cb, int64_t* cw) {
        *cb = (cols[i] + w - 1) / w;
        *cw = ((cols[i] + *cb - 1) / *cb + 31) / 32 * 32;
    };
    int64_t best = 256;
    if (n > 1) {
        double frac[8], lo = 1e300;
        double work = 0.0;
        for (int i = 0; i < n; ++i) work += static_cast<double>(rows[i]) * static_cast<double>(cols[i]);
        for (int t = 0; t < 8; ++t) {
            const int64_t w = 256 - 32 * t;
            int64_t cb[BATCH_MAX], cw[BATCH_MAX], W = 32;
            for (int i = 0; i < n; ++i) {
                tile(w, i, &cb[i], &cw[i]);
                W = cw[i] > W ? cw[i] : W;
            }
            double idle = 0.0;
            for (int i = 0; i < n; ++i)
                idle += static_cast<double>(rows[i]) * static_cast<double>(cb[i] * W - cols[i]);
            frac[t] = idle / work;
            lo = frac[t] < lo ? frac[t] : lo;
        }
        for (int t = 0; t < 8; ++t)
            if (frac[t] <= lo + 0.03) { best = 256 - 32 * t; break; }
    }
    *width = 32;
    for (int i = 0; i < n; ++i) {
        tile(best, i, &out[i].cblocks, &out[i].cw);
        *width = out[i].cw > *width ? out[i].cw : *width;
    }
    // Rows per block: the fewest R such that every unit's blocks, cblocks x
    // ceil(rows / R), fit in the wave (all units' blocks run at once, so the
    // longest block sets the launch's time); without room for one row block
    // per column tile, one row block per unit.
    int64_t rmax = 1;
    for (int i = 0; i < n; ++i) rmax = rows[i] > rmax ? rows[i] : rmax;
    auto blocks_at = [&](int64_t R) {
        int64_t t = 0;
        for (int i = 0; i < n; ++i) t += out[i].cblocks * ((rows[i] + R - 1) / R);
        return t;
    };
    int64_t R = 1, rhi = rmax;   // blocks_at(rmax) is the fewest possible
    while (R < rhi) {
        const int64_t mid = R + (rhi - R) / 2;
        if (blocks_at(mid) <= slots) rhi = mid;
        else R = mid + 1;
    }
    int64_t b = 0;
    for (int i = 0; i < n; ++i) {
        const int64_t rb = (rows[i] + R - 1) / R;   // the unit's row blocks, balanced within it
        out[i].rpb = (rows[i] + rb - 1) / rb;
        out[i].rblocks = (rows[i] + out[i].rpb - 1) / out[i].rpb;
        out[i].block0 = b;
        b += out[i].rblocks * out[i].cblocks;
    }
    return b;
}

// The unit that block `bid` belongs to (a scan of at most BATCH_MAX block
// ranges; the same for every thread of the block).
template <typename U>
__device__ __forceinline__ int batch_unit(const U* u, int n, int64_t bid) {
    int i = 0;
#pragma unroll 1
    while (i + 1 < n && bid >= u[i + 1].s.block0) ++i;
    return i;
}

}  // namespace tq

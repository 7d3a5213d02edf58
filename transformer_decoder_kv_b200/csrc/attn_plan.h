// Host-side launch plan of the split-K decode attention kernel, shared by the decode step,
// dec_attention and dec_attention_noalloc so that equal arguments give equal launches (and
// so equal split boundaries, summation orders and bits).
#pragma once

#include <algorithm>
#include <cmath>

#include "attention.cuh"

namespace dec {

// Most splits of one (stream, head) row; sizes the partial-state scratch.
constexpr int kAttnMaxSplits = 32;

// Split count of a launch over `rows` (stream, head) rows of at most `max_tiles` 64-key
// tiles, when every row is split the same way: fewest (waves x tiles per CTA), two CTAs
// resident per SM, at most `cap` splits.
inline int attn_choose_splits(int num_sms, int rows, int max_tiles, int cap = kAttnMaxSplits) {
    if (max_tiles <= 1) return 1;
    const int slots = num_sms * 2;
    int best = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= std::min(cap, max_tiles); ++s) {
        const int tps = (max_tiles + s - 1) / s;
        const int eff = (max_tiles + tps - 1) / tps;
        if (eff != s) continue;
        const double waves = std::ceil(double(rows) * s / slots);
        const double cost = waves * (tps + 1.5) + (s > 1 ? 0.5 : 0.0);
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

// Fixed tiles per split of the decode step for a handle holding up to `rows_cap` (stream,
// head) rows of at most `max_keys` keys: each row's split boundaries then depend on its own
// length only. Few rows and short caches favour two tiles per split (double-buffered), more
// rows or longer caches four or eight (measured on B200 with HBM-resident caches); never more
// than kAttnMaxSplits splits over the longest row.
inline int attn_tiles_per_split(int rows_cap, int max_keys) {
    const int tiles_cap = (max_keys + kAttnTile - 1) / kAttnTile;
    const int t = rows_cap <= 32 ? 1 : (rows_cap <= 256 && tiles_cap <= 8) ? 2 : (rows_cap <= 1023 ? 4 : 8);
    return std::max(t, (tiles_cap + kAttnMaxSplits - 1) / kAttnMaxSplits);
}

// Shared-memory stages at a fixed tile count per split: one (more resident CTAs) at 1 and 4
// tiles per split, two at 2 and 8 or more (the fastest of each on B200).
inline int attn_stages_for(int tps) { return (tps == 2 || tps >= 8) ? 2 : 1; }

inline size_t attn_smem_bytes(int stages) {
    return size_t(stages) * 2 * kAttnTile * kHeadDim * sizeof(float);
}

// Grid splits and stages of one launch. tps > 0: the step's fixed tiles per split; 0: every
// row split the same way by attn_choose_splits (three stages).
struct AttnLaunch {
    int S, tps, stages;
};
inline AttnLaunch attn_launch_plan(int num_sms, int rows, int max_keys, int tps) {
    const int max_tiles = std::max(1, (max_keys + kAttnTile - 1) / kAttnTile);
    AttnLaunch p;
    if (tps > 0) {
        p.tps = tps;
        p.S = std::max(1, (max_tiles + tps - 1) / tps);
        p.stages = attn_stages_for(tps);
    } else {
        p.tps = 0;
        p.S = attn_choose_splits(num_sms, rows, max_tiles);
        p.stages = kAttnStages;
    }
    return p;
}

}  // namespace dec

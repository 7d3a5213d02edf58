// Host-side plan of a split decode step: the rows of a step of kSplitMinBatch rows or more run
// as chains over equal parts of the batch, each on its own stream (run_step in dec.cu).
#pragma once

#include <algorithm>

namespace dec {

// Below this many rows a projection runs on the CUDA cores; the tensor-core paths start here.
constexpr int kMmaMinBatch = 8;
// Decode steps of this many rows or more run as chains; each chain has at least kMmaMinBatch
// rows, so each stays on the tensor-core paths. Measured on B200: C2 (16 rows) as two chains
// of 8, 0.600 -> 0.568 ms/step.
constexpr int kSplitMinBatch = 16;
// Most chains a step runs as. Measured on B200: two free-running chains C4 5.67 -> 5.40 and C5
// 7.21 -> 5.96 ms/step against two chains whose attentions alternated; four chains C4 5.41,
// C5 6.19.
constexpr int kMaxChains = 2;

// Rows of each chain of a split step: equal multiples of kMmaMinBatch (B / n rounded down),
// the last one taking the rest; r0[c] .. r0[c + 1] - 1 are chain c's rows (r0 holds
// kMaxChains + 1 entries). Returns the chain count (at least 1 for B >= 1); every chain of a
// step of kSplitMinBatch rows or more has at least kMmaMinBatch rows.
inline int chain_bounds(int B, int* r0) {
    const int n = std::max(1, std::min(kMaxChains, B / kMmaMinBatch));
    const int base = std::max(1, (B / n) / kMmaMinBatch * kMmaMinBatch);
    for (int c = 0; c < n; ++c) r0[c] = c * base;
    r0[n] = B;
    return n;
}

}  // namespace dec

// Warp-level match of equal values by ballots (row-id pass, mat-vec routing).
#pragma once

namespace moe {

// Lanes of the warp holding the same value as this lane, from one ballot per
// bit of the value (bits 0..nb; values are ids in [0, 2^nb) or -1, which bit nb
// tells apart).  A warp match instruction serialises over the distinct values
// present, and a 32-slot step of routing ids holds ~30 of them.
__device__ __forceinline__ unsigned match_by_ballots(int v, int nb) {
    unsigned m = 0xffffffffu;
    for (int b = 0; b <= nb; ++b) {
        const int bit = (v >> b) & 1;
        const unsigned bb = __ballot_sync(0xffffffffu, bit);
        m &= bit ? bb : ~bb;
    }
    return m;
}

}  // namespace moe

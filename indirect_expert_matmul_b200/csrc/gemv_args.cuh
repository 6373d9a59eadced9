// Argument block of the expert mat-vec kernel (gemv.cu).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kGvMaxSlots = 1024;   // the mat-vec path handles n_tokens*k up to this
constexpr int kGvNT = 8;            // tokens per pass over a weight chunk
constexpr int kHdrCnt0 = 16;        // header words [16, 64): split-K arrival counters
constexpr int kGvMaxGroups = 48;    // (expert, row tile) groups that may be split

struct GemvSide {
    const uint8_t* W0;  // prepared weights (single, or gate)
    const uint8_t* W1;  // up (dual) or null
    WLayout L;
    const void* x;      // activations: rows of L.n_in elements
    int x_type;         // MOE_BF16 / MOE_F16 / MOE_F32
    int x_per_slot;     // routed x row: 1 -> slot t*k+s, 0 -> token t
    float* out;         // single: out[slot][n] (routed) or out[t][n] (shared)
    __nv_bfloat16* h;   // dual: h[slot][n] (routed) or h[t][n] (shared)
    float* part;        // split-K partial sums [chunk][slot][n_out_pad][1 + dual], or null (no split)
    int kc;             // k-steps per chunk (filled by launch_gemv)
    int chunks;         // ceil(kt_count / kc)
    int group0;         // first counter index of this side's (expert, row tile) groups
};

struct GemvArgs {
    GemvSide routed, shared;
    int has_shared;
    int dual;
    const int32_t* ids;  // [n_tokens][k]
    int n_tokens, k, n_experts;
    int max_distinct;    // min(n_tokens*k, n_experts)
    int pdl_secondary;   // launched as a programmatic dependent: wait before reading activations
    int* hdr;
    // launch plan (filled by launch_gemv)
    int sk;              // k-steps per ring stage
    int ns;              // ring stages
    int xw;              // activation window, in k-steps (a multiple of sk)
    uint32_t stage_bytes, x_bytes, red_bytes, tab_words, bm_words;
};

moe_status launch_gemv(const GemvArgs& a, cudaStream_t stream);
// Reset the split fields of a side (no split); launch_gemv chooses the split.
void gemv_plan_side(GemvSide& s, int dual);

}  // namespace moe
